"""Pins of the CPU oracle against things other than itself (no GPU needed).

Each test checks the oracle against brute force on tiny inputs, a closed form, an invariant, a
library routine, or a number the pages state (tests/golden/pages_facts.json), chosen so that a
plausible mistake (a dropped term, a wrong sign or index, a transposed operand, a wrong rounding)
fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from tiered_weight_gemv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_facts.json")


def facts():
    with open(GOLDEN) as f:
        return json.load(f)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_matches_torch(oracle_lib):
    vals = [0.0, -0.0, 1.0, 1.00390625, 1.01171875, -1.00390625, 3.0e38, 1e-40, -1e-45,
            float("inf"), -float("inf"), 0.1, 1 / 3, 65504.0, 2.0 ** -126, 6.0e-39]
    rng = np.random.default_rng(0)
    vals += list(rng.standard_normal(2000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 2000))
    for v in vals:
        v32 = np.float32(v)
        want = int(bf16_bits(torch.tensor([float(v32)], dtype=torch.float32).to(torch.bfloat16))[0])
        assert oracle_lib.f32_to_bf16_bits(float(v32)) == want, v
        assert oracle_lib.bf16_bits_to_f32(want) == float(
            torch.tensor([want], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
        )


# ----------------------------------------------------------------------------- tier rule

def brute_rank(x):
    """r(j) = #{i: |x_i| > |x_j|} + #{i < j: |x_i| == |x_j|}, O(d^2) counting."""
    a = [abs(float(np.float32(v))) for v in x]
    d = len(a)
    return [sum(1 for i in range(d) if a[i] > a[j]) + sum(1 for i in range(j) if a[i] == a[j])
            for j in range(d)]


def tiny_inputs():
    rng = np.random.default_rng(1)
    cases = []
    for d in (1, 2, 3, 7, 16, 33, 64):
        cases.append(rng.laplace(size=d).astype(np.float32))
        # heavy ties: few distinct magnitudes with both signs, plus signed zeros
        v = rng.integers(-3, 4, size=d).astype(np.float32) * 0.5
        v[rng.integers(0, d)] = -0.0
        cases.append(v)
    cases.append(np.zeros(9, np.float32))
    cases.append(np.array([-0.0, 0.0, -0.0, 0.0], np.float32))
    return cases


@pytest.mark.parametrize("case", range(len(tiny_inputs())))
def test_topk_matches_brute_force_ranks(oracle_lib, case):
    x = tiny_inputs()[case]
    d = x.size
    r = brute_rank(x)
    for kf in sorted({0, 1, d // 3, d // 2, d}):
        for ka in sorted({0, 1, (d - kf) // 2, d - kf}):
            if kf + ka > d:
                continue
            st, tier, fi, ai, counts = oracle_lib.tiers(x, oracle_lib.MODE_TOPK, k_full=kf,
                                                        k_approx=ka)
            assert st == 0
            want = [2 if r[j] < kf else (1 if r[j] < kf + ka else 0) for j in range(d)]
            assert tier.tolist() == want
            assert fi.tolist() == [j for j in range(d) if want[j] == 2]
            assert ai.tolist() == [j for j in range(d) if want[j] == 1]
            assert counts.tolist() == [kf, ka, 0, 0]


def test_tier_monotone_and_counts(oracle_lib):
    for seed in range(5):
        x = synth.laplace((1000,), seed, 11).numpy()
        st, tier, fi, ai, counts = oracle_lib.tiers(x, oracle_lib.MODE_TOPK, k_full=300,
                                                    k_approx=250)
        a = np.abs(x)
        # |x_i| > |x_j|  =>  tier(i) >= tier(j)   (SpAx Abstract: skip closest to zero)
        order = np.argsort(-a, kind="stable")
        assert np.all(np.diff(tier[order].astype(int)) <= 0)
        assert (tier == 2).sum() == 300 and (tier == 1).sum() == 250
        assert counts[0] + counts[1] + (tier == 0).sum() == x.size


def test_topk_permutation_equivariant(oracle_lib):
    rng = np.random.default_rng(3)
    x = rng.laplace(size=500).astype(np.float32)  # continuous: no ties
    perm = rng.permutation(500)
    _, t0, *_ = oracle_lib.tiers(x, oracle_lib.MODE_TOPK, k_full=100, k_approx=150)
    _, t1, *_ = oracle_lib.tiers(x[perm], oracle_lib.MODE_TOPK, k_full=100, k_approx=150)
    assert np.array_equal(t1, t0[perm])


def test_threshold_counts_match_sorted_search(oracle_lib):
    rng = np.random.default_rng(4)
    x = rng.laplace(size=4096).astype(np.float32)
    srt = np.sort(np.abs(x))
    for ts, tf in [(0.0, 0.0), (0.5, 1.0), (0.7, 0.7), (1e-3, 50.0), (float(srt[100]), float(srt[3000]))]:
        st, tier, fi, ai, counts = oracle_lib.tiers(x, oracle_lib.MODE_THRESHOLD, t_skip=ts,
                                                    t_full=tf)
        n1 = int(np.searchsorted(srt, np.float32(ts), side="left"))
        n2 = int(np.searchsorted(srt, np.float32(tf), side="left"))
        assert (counts[2], counts[3]) == (n1, n2)
        assert (tier == 0).sum() == n1 and (tier == 1).sum() == n2 - n1
        assert counts[0] == x.size - n2 and counts[1] == n2 - n1


def band_brute(n, d, s_bp, delta_bp):
    """The m in {0..d} with |m/d - s| <= δ nearest to n (exact rationals); None if none."""
    s, dl = Fraction(s_bp, 10000), Fraction(delta_bp, 10000)
    ok = [m for m in range(d + 1) if abs(Fraction(m, d) - s) <= dl]
    if not ok:
        return None
    return min(ok, key=lambda m: (abs(m - n), m))


def test_guided_band_clip_brute_force(oracle_lib):
    rng = np.random.default_rng(5)
    for trial in range(60):
        d = int(rng.integers(50, 400))
        x = (rng.laplace(size=d) * math.exp(rng.uniform(-1.5, 1.5))).astype(np.float32)
        s1 = int(rng.integers(500, 8000))
        s2 = s1 + int(rng.integers(300, 10000 - s1 + 1)) if s1 < 9700 else 10000
        s2 = min(s2, 10000)
        ts, tf = 0.6, 1.2
        st, tier, fi, ai, counts = oracle_lib.tiers(x, oracle_lib.MODE_GUIDED, t_skip=ts,
                                                    t_full=tf, s_skip_bp=s1, s_below_full_bp=s2,
                                                    delta_bp=100)
        n1 = int((np.abs(x) < np.float32(ts)).sum())
        n2 = int((np.abs(x) < np.float32(tf)).sum())
        m1 = band_brute(n1, d, s1, 100)
        m2 = max(band_brute(n2, d, s2, 100), m1)
        assert (tier == 0).sum() == m1
        assert (tier == 1).sum() == m2 - m1
        assert (counts[2], counts[3]) == (n1, n2)
        # tiers are a TopK by the rank order (brute-force ranks)
        r = brute_rank(x)
        kf = d - m2
        assert tier.tolist() == [2 if r[j] < kf else (1 if r[j] < d - m1 else 0) for j in range(d)]


def test_guided_realised_sparsity_within_delta(oracle_lib):
    f = facts()
    delta = f["guided_delta"]["value"]
    assert f["guided_realised_band_at_0_5"]["max_abs_deviation"] == delta
    for target in f["target_sparsities"]["values"]:
        s1 = int(round(target * 10000))
        s2 = s1 + (10000 - s1) // 2
        calib = synth.laplace((64, 4096), 9, 1).numpy()
        st, ts, tf = oracle_lib.calibrate(calib, s1, s2)
        scales = synth.log_uniform((200,), 9, 2, 0.5, 2.0).numpy()
        toks = synth.laplace((200, 4096), 9, 3).numpy() * scales[:, None].astype(np.float32)
        clipped = 0
        for t in range(200):
            st, tier, fi, ai, counts = oracle_lib.tiers(
                toks[t], oracle_lib.MODE_GUIDED, t_skip=ts, t_full=tf, s_skip_bp=s1,
                s_below_full_bp=s2, delta_bp=int(round(delta * 10000)))
            realised = (tier == 0).mean()
            assert abs(realised - target) <= delta + 1e-12
            assert abs((tier != 2).mean() - s2 / 1e4) <= delta + 1e-12
            clipped += counts[2] != (tier == 0).sum()
        assert clipped > 0  # the clip path was exercised


def test_guided_in_band_equals_threshold(oracle_lib):
    rng = np.random.default_rng(6)
    x = rng.laplace(size=4096).astype(np.float32)
    srt = np.sort(np.abs(x))
    ts, tf = float(srt[2048]), float(srt[3072])  # n1 = 2048 (s=0.5), n2 = 3072 (s=0.75)
    _, tg, *_ = oracle_lib.tiers(x, oracle_lib.MODE_GUIDED, t_skip=ts, t_full=tf, s_skip_bp=5000,
                                 s_below_full_bp=7500, delta_bp=100)
    _, tt, *_ = oracle_lib.tiers(x, oracle_lib.MODE_THRESHOLD, t_skip=ts, t_full=tf)
    assert np.array_equal(tg, tt)


def test_nonfinite_is_an_error(oracle_lib):
    for bad in (np.nan, np.inf, -np.inf):
        x = np.ones(10, np.float32)
        x[3] = bad
        st, tier, fi, ai, counts = oracle_lib.tiers(x, oracle_lib.MODE_TOPK, k_full=3)
        assert st == oracle_lib.ERR_NONFINITE and not tier.any() and not counts.any()


# ----------------------------------------------------------------------------- quantisers

def bf16_of(v: float) -> float:
    return float(torch.tensor([v], dtype=torch.float32).to(torch.bfloat16).float())


def groups_for_test():
    rng = np.random.default_rng(7)
    out = []
    for _ in range(200):
        w = torch.tensor(rng.standard_normal(128) * 0.02 * 10.0 ** rng.uniform(-3, 2),
                         dtype=torch.float32).to(torch.bfloat16)
        out.append(bf16_bits(w))
    out.append(bf16_bits(torch.full((128,), 0.0137, dtype=torch.bfloat16)))   # constant
    out.append(bf16_bits(torch.zeros(128, dtype=torch.bfloat16)))             # zero
    v = torch.zeros(128, dtype=torch.bfloat16)
    v[5] = -0.5
    out.append(bf16_bits(v))                                                  # one outlier
    return out


def test_quant2_brute_force(oracle_lib):
    for wb in groups_for_test():
        w = np.array([oracle_lib.bf16_bits_to_f32(int(h)) for h in wb])
        q, sb, mb = oracle_lib.quant2_group(wb)
        s, m = oracle_lib.bf16_bits_to_f32(sb), oracle_lib.bf16_bits_to_f32(mb)
        assert m == w.min()                                    # min stored exactly
        assert s == bf16_of(np.float32(np.float32(w.max()) - np.float32(w.min())) / np.float32(3))
        assert q.min() >= 0 and q.max() <= 3
        levels = m + np.arange(4) * s
        for wi, qi in zip(w, q):
            err = np.abs(wi - levels)
            best = np.flatnonzero(err == err.min())
            if s == 0:
                assert qi == 0
            elif best.size == 1:
                assert qi == best[0], (wi, levels)
            if m <= wi <= m + 3 * s:
                assert abs(wi - levels[qi]) <= s / 2 * (1 + 1e-6)
        if w.max() == w.min():
            assert np.all(levels[q] == w)                      # constant group is exact


def test_quant4_brute_force(oracle_lib):
    for wb in groups_for_test():
        w = np.array([oracle_lib.bf16_bits_to_f32(int(h)) for h in wb])
        q, sb = oracle_lib.quant4_group(wb)
        s = oracle_lib.bf16_bits_to_f32(sb)
        assert s == bf16_of(np.float32(np.abs(w).max()) / np.float32(7))
        assert q.min() >= -8 and q.max() <= 7
        levels = np.arange(-8, 8) * s
        for wi, qi in zip(w, q):
            err = np.abs(wi - levels)
            best = np.flatnonzero(err == err.min())
            if s == 0:
                assert qi == 0
            elif best.size == 1:
                assert qi == best[0] - 8
        if s > 0:
            assert np.max(np.abs(w - q * s)) <= s / 2 + s * 2.0 ** -7


# ----------------------------------------------------------------------------- packed layout

def decode_pools(full, approx, fmt, d_out, d_in):
    """Independent numpy decoder of the documented layout -> dense fp64 [d_out, d_in] matrices."""
    nrec2 = -(-d_out // 512)
    A = approx.reshape(d_in, nrec2, 144)
    codes = A[:, :, :128]
    q = np.stack([(codes >> (2 * k)) & 3 for k in range(4)], axis=-1).reshape(d_in, nrec2 * 512)
    sm = A[:, :, 128:].copy().view(np.uint32).reshape(d_in, nrec2 * 4)
    scale = (sm & 0xFFFF).astype(np.uint32) << 16
    mn = sm & 0xFFFF0000
    scale = np.repeat(scale.view(np.float32).astype(np.float64), 128, axis=1)
    mn = np.repeat(mn.view(np.float32).astype(np.float64), 128, axis=1)
    Wa = (mn + q * scale)[:, :d_out].T
    if fmt == 0:
        Wf = (full.view(np.uint16).astype(np.uint32) << 16).view(np.float32).reshape(d_in, d_out)
        Wf = Wf.astype(np.float64).T
    else:
        nrec4 = -(-d_out // 1024)
        F = full.reshape(d_in, nrec4, 528)
        nib = np.stack([F[:, :, :512] & 15, F[:, :, :512] >> 4], axis=-1).reshape(d_in, nrec4 * 1024)
        sc = (F[:, :, 512:].copy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
        sc = np.repeat(sc.reshape(d_in, nrec4 * 8).astype(np.float64), 128, axis=1)
        Wf = ((nib.astype(np.float64) - 8) * sc)[:, :d_out].T
    return Wf, Wa


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(128, 5), (640, 33), (1152, 17), (2048, 8)])
def test_pack_layout_and_values(oracle_lib, fmt, d_out, d_in):
    W = synth.weight(d_out, d_in, 0, 20 + fmt)
    Wb = bf16_bits(W)
    full, approx = oracle_lib.pack(Wb, fmt)
    assert full.size == d_in * oracle_lib.full_col_bytes(d_out, fmt)
    assert approx.size == d_in * oracle_lib.approx_col_bytes(d_out)
    Wf, Wa = decode_pools(full, approx, fmt, d_out, d_in)
    Wd = W.double().numpy()
    if fmt == 0:
        assert np.array_equal(Wf, Wd)            # bf16 pool is W^T exactly
    for j in range(d_in):
        for g in range(d_out // 128):
            grp = Wb[g * 128:(g + 1) * 128, j]
            q2, sb, mb = oracle_lib.quant2_group(grp)
            s, m = oracle_lib.bf16_bits_to_f32(sb), oracle_lib.bf16_bits_to_f32(mb)
            assert np.array_equal(Wa[g * 128:(g + 1) * 128, j], m + q2 * np.float64(s))
            if fmt == 1:
                q4, s4 = oracle_lib.quant4_group(grp)
                s4 = oracle_lib.bf16_bits_to_f32(s4)
                assert np.array_equal(Wf[g * 128:(g + 1) * 128, j], q4 * np.float64(s4))
    # point accessors agree with the decoder
    fcb, acb = oracle_lib.full_col_bytes(d_out, fmt), oracle_lib.approx_col_bytes(d_out)
    for (r, j) in [(0, 0), (d_out - 1, d_in - 1), (127, d_in // 2), (d_out // 2 + 3, 1 % d_in)]:
        assert oracle_lib.full_value(full[j * fcb:(j + 1) * fcb], fmt, r) == Wf[r, j]
        assert oracle_lib.approx_value(approx[j * acb:(j + 1) * acb], r) == Wa[r, j]
    # padding rows of the last records
    nrec2 = -(-d_out // 512)
    if nrec2 * 512 > d_out:
        A = approx.reshape(d_in, nrec2, 144)
        pad_groups = list(range((d_out % 512) // 128, 4))
        for g in pad_groups:
            assert not A[:, -1, 128 + 4 * g:132 + 4 * g].any()
        assert not A[:, -1, (d_out % 512) // 4:128].any()


# ----------------------------------------------------------------------------- products

@pytest.mark.parametrize("fmt", [0, 1])
def test_tiered_product_closed_forms(oracle_lib, fmt):
    d_out, d_in = 384, 200
    W = synth.weight(d_out, d_in, 1, 30)
    Wb = bf16_bits(W)
    x = synth.laplace((d_in,), 1, 31).numpy()
    full, approx = oracle_lib.pack(Wb, fmt)
    Wf, Wa = decode_pools(full, approx, fmt, d_out, d_in)
    # all skipped -> exactly zero
    y0 = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, np.zeros(d_in, np.uint8))
    assert np.all(y0 == 0.0)
    # all full -> the dense product of the full pool (bf16: the dense product of W)
    yf = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, np.full(d_in, 2, np.uint8))
    ref = Wf @ x.astype(np.float64)
    assert np.allclose(yf, ref, rtol=1e-12, atol=1e-12)
    if fmt == 0:
        assert np.allclose(yf, W.double().numpy() @ x.astype(np.float64), rtol=1e-12, atol=1e-12)
        assert np.allclose(oracle_lib.dense_gemv(Wb, x), yf, rtol=1e-12, atol=1e-12)
    # mixed tiers -> Σ over full columns of the full pool + Σ over approx columns of the 2-bit pool
    rng = np.random.default_rng(8)
    tier = rng.integers(0, 3, d_in).astype(np.uint8)
    y = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, tier)
    xd = x.astype(np.float64)
    ref = Wf[:, tier == 2] @ xd[tier == 2] + Wa[:, tier == 1] @ xd[tier == 1]
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([0, 5, 383, 128, 127], np.int32)
    assert np.array_equal(oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, tier, rows),
                          y[rows])


def test_four_level_columns_make_approx_exact(oracle_lib):
    # Every 128-row group on a grid w = m + k*s with bf16 m, s and all four levels present:
    # the 2-bit approximation is exact, so all-approx equals the dense product.
    d_out, d_in = 256, 24
    rng = np.random.default_rng(9)
    W = np.zeros((d_out, d_in), np.float32)
    for j in range(d_in):
        for g in range(2):
            s = 2.0 ** -int(rng.integers(6, 10))
            m = -int(rng.integers(0, 60)) * s  # (k - a) * s with |k - a| < 64: exact in bf16
            k = rng.integers(0, 4, 128)
            k[:4] = [0, 1, 2, 3]
            W[g * 128:(g + 1) * 128, j] = m + k * s
    Wt = torch.tensor(W).to(torch.bfloat16)
    assert torch.equal(Wt.float(), torch.tensor(W))
    full, approx = oracle_lib.pack(bf16_bits(Wt), 0)
    x = synth.laplace((d_in,), 2, 1).numpy()
    ya = oracle_lib.tiered_gemv(full, approx, 0, d_out, d_in, x, np.ones(d_in, np.uint8))
    assert np.allclose(ya, W.astype(np.float64) @ x.astype(np.float64), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- calibration

def test_calibration_laplace_closed_form(oracle_lib):
    # |Laplace(0,1)| ~ Exp(1): the s-quantile is -ln(1 - s).
    X = synth.laplace((512, 4096), 3, 1).numpy()
    for s1, s2 in [(3000, 6500), (5000, 7500), (7000, 8500)]:
        st, t1, t2 = oracle_lib.calibrate(X, s1, s2)
        assert st == 0
        assert abs(t1 - (-math.log(1 - s1 / 1e4))) < 3e-3
        assert abs(t2 - (-math.log(1 - s2 / 1e4))) < 3e-3


def test_calibration_order_statistic(oracle_lib):
    rng = np.random.default_rng(10)
    for M in (1, 2, 7, 100, 1001):
        X = rng.laplace(size=M).astype(np.float32)
        X[rng.integers(0, M)] = 0.0
        a = np.abs(X)
        for s in (0, 1, 2500, 5000, 9999, 10000):
            st, t, _ = oracle_lib.calibrate(X, s, s)
            k = min(int(Fraction(s, 10000) * M + Fraction(1, 2)), M - 1)
            # t is the k-th smallest (0-based): fewer than k+1 values below, at least k+1 <= t
            assert (a < t).sum() <= k < (a <= t).sum()


# ----------------------------------------------------------------------------- block budgets

def test_block_budgets_invariants(oracle_lib):
    f = facts()
    lo, hi = f["block_budget_clamp"]["lo"], f["block_budget_clamp"]["hi"]
    b = np.arange(32)
    sens = 1.0 + 3.0 * np.exp(-b / 4.0)
    for s in f["target_sparsities"]["values"]:
        u = oracle_lib.block_budgets(sens, s, 0.0, lo, hi)
        assert np.allclose(u, s, atol=0, rtol=0) or np.allclose(u, s, atol=1e-15)
        for lam in (0.2, 0.5, 0.8, 3.0):
            out = oracle_lib.block_budgets(sens, s, lam, lo, hi)
            assert abs(out.mean() - s) < 1e-9
            assert out.min() >= lo and out.max() <= hi
            # more sensitive -> not more sparsity
            order = np.argsort(sens)
            assert np.all(np.diff(out[order]) <= 1e-15)
            # independent solve: bisection on the shift c of the clamped mean
            a = s * (1 - lam * (sens / sens.mean() - 1))
            lo_c, hi_c = lo - a.max(), hi - a.min()
            for _ in range(200):
                mid = 0.5 * (lo_c + hi_c)
                if np.clip(a + mid, lo, hi).mean() < s:
                    lo_c = mid
                else:
                    hi_c = mid
            assert np.allclose(out, np.clip(a + 0.5 * (lo_c + hi_c), lo, hi), atol=1e-9)


# ----------------------------------------------------------------------------- byte account

def test_weight_bytes_account(oracle_lib):
    # full columns × d_out × 2 B + approx columns × d_out × 0.25 B + scales (bf16 scale + min)
    assert oracle_lib.weight_bytes(4096, 0, 1024, 1024) == 1024 * 4096 * 2 + 1024 * 4096 // 4 + 1024 * 32 * 4
    assert oracle_lib.weight_bytes(4096, 0, 0, 0) == 0
    # int4 full tier: d_out/2 bytes of codes + a bf16 scale per 128 rows
    assert oracle_lib.weight_bytes(8192, 1, 10, 0) == 10 * (4096 + 64 * 2)
    # the account equals the packed pools' column sizes when d_out fills whole records
    for d_out in (1024, 4096, 14336):
        assert oracle_lib.weight_bytes(d_out, 0, 0, 1) == oracle_lib.approx_col_bytes(d_out)
        assert oracle_lib.weight_bytes(d_out, 0, 1, 0) == oracle_lib.full_col_bytes(d_out, 0)
        assert oracle_lib.weight_bytes(d_out, 1, 1, 0) == oracle_lib.full_col_bytes(d_out, 1)


def test_openmp_build_gives_the_same_products(oracle_lib):
    # The multi-core build only hands independent row chunks to threads: every output is the
    # same sum in the same order, so the two builds agree bit for bit (ragged chunk included).
    d_out, d_in = 640, 300
    W = synth.weight(d_out, d_in, 1, 40)
    x = synth.laplace((d_in,), 1, 41).numpy()
    tier = np.random.default_rng(10).integers(0, 3, d_in).astype(np.uint8)
    rows = np.array([639, 0, 300, 257, 256, 255], np.int32)
    for fmt in (0, 1):
        full, approx = oracle_lib.pack(bf16_bits(W), fmt)
        y1 = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, tier)
        r1 = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, tier, rows)
        try:
            assert oracle_lib.use_openmp(True) >= 1
            yn = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, tier)
            rn = oracle_lib.tiered_gemv(full, approx, fmt, d_out, d_in, x, tier, rows)
        finally:
            oracle_lib.use_openmp(False)
        assert np.array_equal(y1, yn) and np.array_equal(r1, rn) and np.array_equal(r1, y1[rows])


def test_swiglu_closed_forms(oracle_lib):
    # silu(0) = 0; silu(g) - silu(-g) = g (sigma(g) + sigma(-g) = 1); silu(g) = g/2 (1 + tanh(g/2))
    # (a different closed form of the same function); the gate scales linearly in u.
    g = np.array([0.0, 1e-8, 0.3, -0.3, 1.0, -2.5, 7.0, -12.0, 30.0, -30.0])
    ones = np.ones_like(g)
    s = oracle_lib.swiglu(g, ones)
    assert s[0] == 0.0
    assert np.allclose(s - oracle_lib.swiglu(-g, ones), g, rtol=1e-14, atol=1e-14)
    mid = np.abs(g) <= 8  # the tanh form cancels in the negative tail; there use g e^g / (1 + e^g)
    assert np.allclose(s[mid], (g / 2 * (1 + np.tanh(g / 2)))[mid], rtol=1e-13, atol=1e-300)
    assert np.allclose(s, g * np.exp(g) / (1 + np.exp(g)), rtol=1e-14, atol=1e-300)
    u = np.linspace(-3, 3, g.size)
    assert np.allclose(oracle_lib.swiglu(g, u), s * u, rtol=1e-15, atol=0)
    # far tails: silu(g) -> g for large g, -> g e^g (tiny, negative) for very negative g
    assert oracle_lib.swiglu(40.0, 1.0) == 40.0
    assert -1e-15 < oracle_lib.swiglu(-40.0, 1.0) < 0.0


def test_column_norms_definition(oracle_lib):
    # the definition written out in Python on a small matrix (fp64 sum in row order, sqrt, fp32)
    rng = np.random.default_rng(21)
    W = torch.tensor(rng.normal(0, 0.05, (37, 11)), dtype=torch.float32).to(torch.bfloat16)
    Wb = bf16_bits(W)
    n = oracle_lib.column_norms(Wb)
    Wf = W.float().double().numpy()
    for j in range(11):
        acc = 0.0
        for r in range(37):
            acc += Wf[r, j] * Wf[r, j]
        assert n[j] == np.float32(math.sqrt(acc))
    # closed forms: a column of one value c has norm |c| sqrt(d_out); a zero column has norm 0
    C = torch.zeros(64, 3, dtype=torch.bfloat16)
    C[:, 0] = 0.375
    C[:, 1] = -2.0
    n = oracle_lib.column_norms(bf16_bits(C))
    assert n[0] == np.float32(0.375 * 8.0) and n[1] == np.float32(16.0) and n[2] == 0.0


def test_wina_scores_rank_by_norm_and_magnitude(oracle_lib):
    # equal norms give the |x| tiers; equal |x| gives the tiers of the norms (column order on ties)
    rng = np.random.default_rng(22)
    x = synth.laplace((500,), 2, 5).numpy()
    ones = np.full(500, 4.0, np.float32)  # a power of two: the products keep the order exactly
    kf, ka = 120, 150
    _, t_x, *_ = oracle_lib.tiers(x, oracle_lib.MODE_TOPK, k_full=kf, k_approx=ka)
    _, t_s, *_ = oracle_lib.tiers(oracle_lib.wina_scores(x, ones), oracle_lib.MODE_TOPK,
                                  k_full=kf, k_approx=ka)
    assert np.array_equal(t_x, t_s)
    norms = rng.uniform(0.1, 2.0, 500).astype(np.float32)
    _, t_n, *_ = oracle_lib.tiers(oracle_lib.wina_scores(np.full(500, -0.5, np.float32), norms),
                                  oracle_lib.MODE_TOPK, k_full=kf, k_approx=ka)
    rank = np.argsort(-norms, kind="stable")
    want = np.zeros(500, np.uint8)
    want[rank[:kf]] = 2
    want[rank[kf:kf + ka]] = 1
    assert np.array_equal(t_n, want)
    # the score is the fp32 product itself
    s = oracle_lib.wina_scores(np.array([-3.0, 0.1], np.float32), np.array([0.5, 3.0], np.float32))
    assert s[0] == np.float32(1.5) and s[1] == np.float32(0.1) * np.float32(3.0)
