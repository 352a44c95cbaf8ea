"""The TopK rule given a guess of its boundary keys (t_full for full | rest, t_skip for kept |
skipped): the guess only changes how the kernels find the boundaries, never the result. Every
case compares the mask's tiers, lists and counts with the oracle bit for bit, and the one-launch
masked GEMV with and without the guess bit for bit.

`guess_path` restates, on the host, how the kernels use a guess (a window of 2048 bins around it,
the bin of rank K, the keys of that bin), so each case can assert which branch it exercises: a
miss, a whole bin, a one-key bin, a gathered bin, a bin too crowded to rank, or an invalid guess.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tiered_weight_gemv_b200 import spax, synth

pytestmark = pytest.mark.gpu

CAND = 32  # keys of one bin the kernels rank; more falls back to the full selection
BINS = 2048  # bins of one window


def _f32(v) -> np.float32:
    return np.float32(v)


def window(h):
    """(lo, sh) of a guess h, or None when h is not usable (keys [lo, lo + (BINS << sh)))."""
    hb = int(np.array([h], np.float32).view(np.uint32)[0])
    if not 1 <= hb <= 0x7F7FFFFF:
        return None
    a = int(np.array([_f32(h) * _f32(0.875)], np.float32).view(np.uint32)[0])
    b = int(np.array([_f32(h) * _f32(1.125)], np.float32).view(np.uint32)[0])
    if a == 0:
        return None
    r = b - a
    return a, (0 if r <= BINS else ((r - 1) // BINS).bit_length())


def guess_path(x: np.ndarray, K: int, h) -> str:
    """Which branch one boundary of rank K takes with guess h."""
    keys = np.asarray(x, np.float32).view(np.uint32).astype(np.int64) & 0x7FFFFFFF
    d = keys.size
    if K == 0 or K == d:
        return "edge"
    w = window(h)
    if w is None:
        return "invalid"
    lo, sh = w
    hi = lo + (BINS << sh)
    A = int(np.sum(keys >= hi))
    inside = keys[(keys >= lo) & (keys < hi)]
    if not (A < K <= A + inside.size):
        return "miss"
    cnt = np.bincount((inside - lo) >> sh, minlength=BINS)
    above = A
    for b in range(BINS - 1, -1, -1):
        if above < K <= above + cnt[b]:
            rem, c = K - above, int(cnt[b])
            if rem == c:
                return "bin"
            if sh == 0:
                return "onekey"
            return "crowded" if c > CAND else "gather"
        above += int(cnt[b])
    raise AssertionError("rank not found")


def kth_key(x: np.ndarray, K: int) -> float:
    """|x| of rank K (1-based, largest first)."""
    return float(np.sort(np.abs(np.asarray(x, np.float32)))[::-1][K - 1])


class Mask:
    def __init__(self, d):
        self.d = d
        self.tier = torch.empty(d, dtype=torch.uint8, device="cuda")
        self.fidx = torch.empty(d, dtype=torch.int32, device="cuda")
        self.aidx = torch.empty(d, dtype=torch.int32, device="cuda")
        self.counts = torch.empty(4, dtype=torch.int32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def check(self, x: np.ndarray, kf: int, ka: int, tf, ts, ctx=""):
        prm = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka, t_full=tf, t_skip=ts)
        self.status.zero_()
        spax.spax_build_mask(torch.from_numpy(x).cuda(), prm, self.tier, self.fidx, self.aidx,
                             self.counts, self.status)
        torch.cuda.synchronize()
        st, t_o, f_o, a_o, c_o = oracle.tiers(x, oracle.MODE_TOPK, k_full=kf, k_approx=ka)
        c = self.counts.cpu().numpy()
        assert self.status.item() == 0 and st == 0, ctx
        assert np.array_equal(c, c_o), ctx
        assert np.array_equal(self.tier.cpu().numpy(), t_o), ctx
        assert np.array_equal(self.fidx[: c[0]].cpu().numpy(), f_o), ctx
        assert np.array_equal(self.aidx[: c[1]].cpu().numpy(), a_o), ctx


def _laplace(d, seed):
    return synth.laplace((d,), seed, 41).numpy()


def _clustered(d, seed):
    """Laplace with 20 copies of 1.0 and 6 of the next float up, spread over the columns: ranks
    inside the cluster land in a bin that holds more keys than the rank takes."""
    x = _laplace(d, seed)
    rng = np.random.default_rng(seed)
    pos = rng.choice(d, 26, replace=False)
    up = np.nextafter(np.float32(1.0), np.float32(2.0))
    x[pos[:20]] = np.float32(1.0) * np.where(rng.random(20) < 0.5, 1, -1).astype(np.float32)
    x[pos[20:]] = up
    return x


def _subnormal(d, seed):
    """Subnormal magnitudes (bit patterns 1..3000, random signs): windows of single-key bins."""
    rng = np.random.default_rng(seed)
    bits = rng.integers(1, 3000, d).astype(np.uint32) | (rng.integers(0, 2, d).astype(np.uint32) << 31)
    return bits.view(np.float32).copy()


def _few_values(d, seed):
    """Only four distinct magnitudes: every bin of a rank holds hundreds of equal keys."""
    rng = np.random.default_rng(seed)
    return (rng.integers(1, 5, d) * 0.25).astype(np.float32) * np.where(rng.random(d) < 0.5, 1, -1).astype(np.float32)


@pytest.mark.parametrize("d", [7, 1000, 4096, 8192, 11008, 28672, 32768])
def test_guess_laplace_all_branches(d):
    m = Mask(d)
    x = _laplace(d, d)
    seen = set()
    for fk, ak in [(0.25, 0.25), (0.1, 0.5), (0.4, 0.1), (0.05, 0.05)]:
        kf, ka = int(fk * d + 0.5), int(ak * d + 0.5)
        if kf + ka > d:
            continue
        for scale in (1.0, 1.03, 0.97, 1.2, 0.8, 2.0, 0.5):
            tf = kth_key(x, kf) * scale if kf else 1.0
            ts = kth_key(x, kf + ka) * scale if kf + ka else 1.0
            seen.add(guess_path(x, kf, tf))
            seen.add(guess_path(x, kf + ka, ts))
            m.check(x, kf, ka, tf, ts, f"d={d} kf={kf} ka={ka} scale={scale}")
    if d >= 1000:
        assert {"miss", "bin"} <= seen, seen
    if d in (1000, 4096, 28672):
        assert "gather" in seen, seen


def test_guess_invalid_and_edge_values():
    d = 4096
    m = Mask(d)
    x = _laplace(d, 5)
    for tf, ts in [(0.0, 0.0), (-1.0, 0.7), (float("nan"), 0.7), (float("inf"), 0.7),
                   (1.5, float("-inf")), (1e-45, 1e-45), (3e38, 3e38), (1.4, 0.69)]:
        for kf, ka in [(0, 0), (d, 0), (0, d), (1, 1), (d - 1, 1), (1024, 1024), (2048, 0)]:
            m.check(x, kf, ka, tf, ts, f"kf={kf} ka={ka} tf={tf} ts={ts}")
    assert guess_path(x, 1024, float("nan")) == "invalid"
    assert guess_path(x, 0, 0.7) == "edge"


def test_guess_gathered_bin():
    d = 4096
    m = Mask(d)
    x = _clustered(d, 11)
    above = int(np.sum(np.abs(x) > 1.0))  # includes the 6 keys just above 1.0
    hits = set()
    for r in (1, 3, 10, 19):
        K = above + r  # rank inside the 20 equal keys
        p = guess_path(x, K, 1.0)
        hits.add(p)
        m.check(x, K, 0, 1.0, 1.0, f"K={K}")  # both boundaries at rank K
        m.check(x, K - 2, 2, 1.0, 1.0, f"K={K} split")
        m.check(x, 100, K - 100, 0.6 * 2, 1.0, f"K={K} approx boundary")
    assert "gather" in hits, hits


def test_guess_crowded_bin_falls_back():
    d = 11008
    m = Mask(d)
    x = _few_values(d, 3)
    for kf, ka in [(d // 4, d // 4), (d // 3, d // 3), (100, 200)]:
        tf = kth_key(x, kf)
        ts = kth_key(x, kf + ka)
        assert guess_path(x, kf + ka, ts) in ("crowded", "bin"), guess_path(x, kf + ka, ts)
        m.check(x, kf, ka, tf, ts, f"kf={kf} ka={ka}")


def test_guess_one_key_bins():
    d = 4096
    m = Mask(d)
    x = _subnormal(d, 9)
    paths = set()
    for kf, ka in [(1000, 1000), (512, 2048), (2000, 1), (1, 4000)]:
        tf = kth_key(x, kf)
        ts = kth_key(x, kf + ka)
        assert window(tf)[1] == 0
        paths.add(guess_path(x, kf, tf))
        paths.add(guess_path(x, kf + ka, ts))
        m.check(x, kf, ka, tf, ts, f"kf={kf} ka={ka}")
    assert "onekey" in paths, paths


def test_guess_nonfinite_sets_status():
    d = 3000
    x = synth.laplace((d,), 1, 1).numpy()
    for bad in (float("nan"), float("inf")):
        xb = x.copy()
        xb[17] = bad
        m = Mask(d)
        prm = spax.mask_params(spax.MASK_TOPK, k_full=300, k_approx=300,
                               t_full=kth_key(x, 300), t_skip=kth_key(x, 600))
        spax.spax_build_mask(torch.from_numpy(xb).cuda(), prm, m.tier, m.fidx, m.aidx, m.counts,
                             m.status)
        torch.cuda.synchronize()
        assert m.status.item() == spax.ERR_NONFINITE
        assert not m.tier.any() and not m.counts.any()


@pytest.mark.parametrize("d_out,d_in", [(4096, 4096), (4096, 11008), (6144, 4096)])
def test_masked_gemv_guess_bitexact(d_out, d_in):
    """The one-launch masked GEMV gives the same tiers, lists, counts and y, bit for bit, with a
    hitting, a missing and no guess (several tokens of each)."""
    W = synth.weight(d_out, d_in, 3, 5, device="cuda")
    pm = spax.alloc_packed(d_out, d_in, spax.FULL_BF16)
    spax.spax_pack_weights(W, spax.FULL_BF16, pm)
    ws = spax.alloc_workspace(spax.OP_TIERED_GEMV, d_out, d_in)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kf, ka = d_in // 4, d_in // 4
    for tok in range(4):
        x = _clustered(d_in, 100 + tok) if tok == 3 else _laplace(d_in, 100 + tok)
        xd = torch.from_numpy(x).cuda()
        outs = []
        for tf, ts in [(0.0, 0.0), (kth_key(x, kf), kth_key(x, kf + ka)),
                       (kth_key(x, kf) * 1.05, kth_key(x, kf + ka) * 0.96),
                       (kth_key(x, kf) * 3, kth_key(x, kf + ka) / 3)]:
            prm = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka, t_full=tf, t_skip=ts)
            y = torch.full((d_out,), float("nan"), device="cuda")
            tier = torch.full((d_in,), 7, dtype=torch.uint8, device="cuda")
            fi = torch.full((d_in,), -1, dtype=torch.int32, device="cuda")
            ai = torch.full((d_in,), -1, dtype=torch.int32, device="cuda")
            c = torch.full((4,), -1, dtype=torch.int32, device="cuda")
            spax.spax_masked_gemv(pm, xd, prm, y, st, ws, tier=tier, full_idx=fi, approx_idx=ai,
                                  counts=c)
            torch.cuda.synchronize()
            assert st.item() == 0
            outs.append([t.cpu().numpy() for t in (tier, fi, ai, c, y)])
        _, t_o, f_o, a_o, c_o = oracle.tiers(x, oracle.MODE_TOPK, k_full=kf, k_approx=ka)
        assert np.array_equal(outs[0][0], t_o) and np.array_equal(outs[0][3], c_o)
        for o in outs[1:]:
            for a, b in zip(outs[0], o):
                assert np.array_equal(a, b), f"token {tok}: guessed result differs"


@pytest.mark.parametrize("d", [4096, 11008])
def test_guess_miss_stress(d):
    """Many tokens whose guesses all miss (twice and half the true keys, both boundaries or one):
    the windowed pass gives way to the full selection in the same launch, which must start from a
    clean histogram every time. Mask and one-launch masked GEMV against the oracle, bit for bit."""
    m = Mask(d)
    d_out = 1024
    W = synth.weight(d_out, d, 4, 6, device="cuda")
    pm = spax.alloc_packed(d_out, d, spax.FULL_BF16)
    spax.spax_pack_weights(W, spax.FULL_BF16, pm)
    ws = spax.alloc_workspace(spax.OP_TIERED_GEMV, d_out, d)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kf, ka = int(0.3 * d + 0.5), int(0.3 * d + 0.5)
    for tok in range(24):
        x = _laplace(d, 500 + tok)
        f = (2.0, 0.5, 1.0)[tok % 3]
        g = (1.0, 2.0, 0.5)[tok % 3]
        tf, ts = kth_key(x, kf) * f, kth_key(x, kf + ka) * g
        assert "miss" in (guess_path(x, kf, tf), guess_path(x, kf + ka, ts))
        m.check(x, kf, ka, tf, ts, f"token {tok}")
        prm = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka, t_full=tf, t_skip=ts)
        tier = torch.empty(d, dtype=torch.uint8, device="cuda")
        y = torch.empty(d_out, device="cuda")
        spax.spax_masked_gemv(pm, torch.from_numpy(x).cuda(), prm, y, st, ws, tier=tier)
        torch.cuda.synchronize()
        assert st.item() == 0
        _, t_o, _, _, _ = oracle.tiers(x, oracle.MODE_TOPK, k_full=kf, k_approx=ka)
        assert np.array_equal(tier.cpu().numpy(), t_o), f"masked GEMV token {tok}"


def _masked(pm, d_out, d_in, x, prm, ws, norms=None, swiglu=False):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.full((d_out,), float("nan"), device="cuda")
    tier = torch.full((d_in,), 7, dtype=torch.uint8, device="cuda")
    fi = torch.full((d_in,), -1, dtype=torch.int32, device="cuda")
    ai = torch.full((d_in,), -1, dtype=torch.int32, device="cuda")
    c = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    kw = dict(tier=tier, full_idx=fi, approx_idx=ai, counts=c)
    if swiglu:
        spax.spax_masked_gemv_swiglu(pm, x, prm, y, st, ws, **kw)
    elif norms is not None:
        spax.spax_masked_gemv_wina(pm, x, norms, prm, y, st, ws, **kw)
    else:
        spax.spax_masked_gemv(pm, x, prm, y, st, ws, **kw)
    torch.cuda.synchronize()
    assert st.item() == 0
    return [t.cpu().numpy() for t in (tier, fi, ai, c, y)]


@pytest.mark.parametrize("d_out,d_in,fmt,src", [(4096, 4096, 0, "x"), (4096, 11008, 0, "x"),
                                                (4096, 4096, 1, "x"), (4096, 4096, 0, "wina"),
                                                (4096, 11008, 0, "swiglu"),
                                                (8192, 20480, 0, "swiglu")])
def test_scaled_guess_follows_token_scale(d_out, d_in, fmt, src):
    """MASK_TOPK_SCALED: the guesses are multiples of the token's mean key, calibrated once on a
    unit-scale token. Tokens scaled by 0.25 to 7.5 (SwiGLU: u scaled, so x = silu(g) * u scales
    with it): on the host model of the window, the scaled
    guess hits every token while the same guess taken as absolute keys misses the far scales; on
    the GPU, the scaled rule gives the tiers, lists, counts and y of the unguessed TopK rule bit
    for bit (and the oracle's tiers), through spax_build_mask and the masked GEMV. The sources:
    plain x, the WINA score, and SwiGLU through the plain instance (4096 x 11008: x stays in shared
    memory) and through its own instance (8192 x 20480)."""
    W = synth.weight(d_out, d_in, 7, 9, device="cuda")
    pm = spax.alloc_packed(d_out, d_in, fmt)
    spax.spax_pack_weights(W, fmt, pm)
    ws = spax.alloc_workspace(spax.OP_TIERED_GEMV, d_out, d_in)
    norms = None
    if src == "wina":
        norms = torch.empty(d_in, device="cuda")
        spax.spax_column_norms(W, norms)
    del W
    kf, ka = int(0.3 * d_in + 0.5), int(0.3 * d_in + 0.5)

    def keys_of(v):  # the rule's keys on the host (fp32)
        v = np.asarray(v, np.float32)
        if src == "wina":
            return np.abs(v) * norms.cpu().numpy()
        if src == "swiglu":
            return np.abs(oracle.swiglu(v[:d_in].astype(np.float64), v[d_in:].astype(np.float64)).astype(np.float32))
        return np.abs(v)

    n_in = 2 * d_in if src == "swiglu" else d_in
    x0 = synth.laplace((n_in,), 70, 3).numpy()
    k0 = keys_of(x0)
    mean0 = float(np.mean(k0, dtype=np.float64))
    rel_f, rel_s = kth_key(k0, kf) / mean0, kth_key(k0, kf + ka) / mean0
    m = Mask(d_in) if src == "x" else None
    missed_abs = 0
    for i, scale in enumerate([0.25, 0.5, 1.0, 2.0, 4.0, 7.5]):
        x = synth.laplace((n_in,), 71 + i, 3).numpy()
        if src == "swiglu":  # x = silu(g) * u scales with u alone
            x[d_in:] *= np.float32(scale)
        else:
            x *= np.float32(scale)
        k = keys_of(x)
        mean = float(np.mean(k, dtype=np.float64))
        assert guess_path(k, kf, rel_f * mean) != "miss" and guess_path(k, kf + ka, rel_s * mean) != "miss"
        missed_abs += "miss" in (guess_path(k, kf, rel_f * mean0), guess_path(k, kf + ka, rel_s * mean0))
        xd = torch.from_numpy(x).cuda()
        plain = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka)
        scaled = spax.mask_params(spax.MASK_TOPK_SCALED, k_full=kf, k_approx=ka, t_full=rel_f,
                                  t_skip=rel_s)
        a = _masked(pm, d_out, d_in, xd, plain, ws, norms, src == "swiglu")
        b = _masked(pm, d_out, d_in, xd, scaled, ws, norms, src == "swiglu")
        for u, v in zip(a, b):
            assert np.array_equal(u, v), f"scale {scale}: the scaled guess changed the result"
        if src == "x":
            _, t_o, _, _, c_o = oracle.tiers(x, oracle.MODE_TOPK, k_full=kf, k_approx=ka)
            assert np.array_equal(b[0], t_o) and np.array_equal(b[3], c_o)
            m.status.zero_()
            spax.spax_build_mask(xd, scaled, m.tier, m.fidx, m.aidx, m.counts, m.status)
            torch.cuda.synchronize()
            assert m.status.item() == 0 and np.array_equal(m.tier.cpu().numpy(), t_o)
            assert np.array_equal(m.counts.cpu().numpy(), c_o)
    assert missed_abs >= 2  # the absolute guess misses the far scales


def test_scaled_guess_edge_values():
    """MASK_TOPK_SCALED with no usable guess (0, NaN, a negative multiple), an all-zero token and a
    non-finite token: the results of the unguessed TopK rule, and SPAX_ERR_NONFINITE for the
    last."""
    d = 4096
    m = Mask(d)
    kf, ka = 1000, 1000
    x = _laplace(d, 90)
    _, t_o, f_o, a_o, c_o = oracle.tiers(x, oracle.MODE_TOPK, k_full=kf, k_approx=ka)
    for tf, ts in [(0.0, 0.0), (float("nan"), 1.0), (-1.0, -2.0), (1e30, 1e-30)]:
        prm = spax.mask_params(spax.MASK_TOPK_SCALED, k_full=kf, k_approx=ka, t_full=tf, t_skip=ts)
        m.status.zero_()
        spax.spax_build_mask(torch.from_numpy(x).cuda(), prm, m.tier, m.fidx, m.aidx, m.counts,
                             m.status)
        torch.cuda.synchronize()
        assert m.status.item() == 0 and np.array_equal(m.tier.cpu().numpy(), t_o)
        assert np.array_equal(m.counts.cpu().numpy(), c_o)
    prm = spax.mask_params(spax.MASK_TOPK_SCALED, k_full=kf, k_approx=ka, t_full=1.2, t_skip=0.4)
    z = np.zeros(d, np.float32)
    _, t_z, _, _, c_z = oracle.tiers(z, oracle.MODE_TOPK, k_full=kf, k_approx=ka)
    m.status.zero_()
    spax.spax_build_mask(torch.from_numpy(z).cuda(), prm, m.tier, m.fidx, m.aidx, m.counts, m.status)
    torch.cuda.synchronize()
    assert m.status.item() == 0 and np.array_equal(m.tier.cpu().numpy(), t_z)
    assert np.array_equal(m.counts.cpu().numpy(), c_z)
    xn = x.copy()
    xn[17] = np.inf
    m.status.zero_()
    spax.spax_build_mask(torch.from_numpy(xn).cuda(), prm, m.tier, m.fidx, m.aidx, m.counts, m.status)
    torch.cuda.synchronize()
    assert m.status.item() == spax.ERR_NONFINITE
