"""GPU parity of every kernel against the CPU oracle, through the C ABI (needs a B200).

Tier codes, compacted lists, counts and packed pools must be bit-exact; y must be within
rel L2 <= 2e-3 and max abs <= 1e-2 * max|y| of the fp64 oracle on identical dequantised values.
Sizes span several row tiles and a ragged last tile, every split of the columns over CTAs, and the
degenerate cases (no column, one column, every column in one tier, ties, zeros, d_in = 1).
"""
import numpy as np
import pytest
import torch

from conftest import cuda_ok

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

if cuda_ok():
    import oracle
    from tiered_weight_gemv_b200 import spax, synth
    from gpu_helpers import GpuMatrix, bf16_bits, check_token, check_y


@pytest.fixture(scope="module", autouse=True)
def _built(oracle_lib):
    return oracle_lib


def _w(d_out, d_in, tid):
    return synth.weight(d_out, d_in, 0, tid, device="cuda")


# ----------------------------------------------------------------------------- packer

@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(128, 1), (640, 33), (1152, 70), (4096, 257), (22016, 40)])
def test_pack_bitexact(fmt, d_out, d_in):
    W = _w(d_out, d_in, 100 + d_out % 97)
    gm = GpuMatrix(W, fmt)
    torch.cuda.synchronize()
    full_o, approx_o = oracle.pack(bf16_bits(W), fmt)
    assert np.array_equal(gm.pm.full.cpu().numpy(), full_o)
    assert np.array_equal(gm.pm.approx.cpu().numpy(), approx_o)


def test_pack_special_values():
    # constant groups, signed zeros, one outlier, tiny and huge magnitudes
    d_out, d_in = 512, 64
    W = torch.zeros(d_out, d_in, dtype=torch.bfloat16)
    W[:, 1] = 0.0137
    W[:, 2] = -0.0
    W[::2, 3] = -0.0
    W[5, 4] = -0.5
    W[:, 5] = torch.linspace(-1e-30, 1e-30, d_out).to(torch.bfloat16)
    W[:, 6] = torch.linspace(-3e30, 2e30, d_out).to(torch.bfloat16)
    W[:, 7:] = synth.weight(d_out, d_in - 7, 1, 5)
    W = W.cuda()
    for fmt in (0, 1):
        gm = GpuMatrix(W, fmt)
        torch.cuda.synchronize()
        full_o, approx_o = oracle.pack(bf16_bits(W), fmt)
        assert np.array_equal(gm.pm.full.cpu().numpy(), full_o)
        assert np.array_equal(gm.pm.approx.cpu().numpy(), approx_o)


# ----------------------------------------------------------------------------- mask

def _mask_inputs(d, seed):
    x = synth.laplace((d,), seed, 7)
    ties = (torch.round(synth.laplace((d,), seed, 8) * 2) / 2).to(torch.float32)
    ties[:: max(1, d // 5)] = -0.0
    return {"laplace": x, "ties": ties, "zeros": torch.zeros(d)}


def _mask_cases(d):
    k = [(0, 0), (d, 0), (0, d), (d // 4, d // 4), (d // 3, d - d // 3), (1, 1), (max(0, d - 1), 1 if d > 0 else 0)]
    out = [spax.mask_params(spax.MASK_TOPK, k_full=a, k_approx=b) for a, b in k if a + b <= d]
    out += [spax.mask_params(spax.MASK_THRESHOLD, t_skip=ts, t_full=tf)
            for ts, tf in [(0.0, 0.0), (0.5, 1.0), (0.7, 0.7), (0.0, float("inf"))]]
    out += [spax.mask_params(spax.MASK_GUIDED, t_skip=ts, t_full=tf, s_skip_bp=s1,
                             s_below_full_bp=s2, delta_bp=100)
            for ts, tf, s1, s2 in [(0.69, 1.39, 5000, 7500), (0.36, 0.69, 3000, 6500),
                                   (2.0, 3.0, 7000, 8500), (0.0, 0.0, 5000, 5000)]]
    return out


@pytest.mark.parametrize("d", [1, 7, 1000, 4096, 11008, 28672, 32768])
def test_mask_bitexact(d):
    from gpu_helpers import oracle_params
    dev = "cuda"
    tier = torch.empty(d, dtype=torch.uint8, device=dev)
    fidx = torch.empty(d, dtype=torch.int32, device=dev)
    aidx = torch.empty(d, dtype=torch.int32, device=dev)
    counts = torch.empty(4, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for name, x in _mask_inputs(d, d).items():
        xd = x.to(dev)
        for prm in _mask_cases(d):
            spax.spax_build_mask(xd, prm, tier, fidx, aidx, counts, status)
            torch.cuda.synchronize()
            op = oracle_params(prm)
            st, t_o, f_o, a_o, c_o = oracle.tiers(x.numpy(), op.pop("mode"), **op)
            c = counts.cpu().numpy()
            ctx = f"{name} mode={prm.mode} kf={prm.k_full} ka={prm.k_approx} ts={prm.t_skip}"
            assert status.item() == 0
            assert np.array_equal(c, c_o), ctx
            assert np.array_equal(tier.cpu().numpy(), t_o), ctx
            assert np.array_equal(fidx[: c[0]].cpu().numpy(), f_o), ctx
            assert np.array_equal(aidx[: c[1]].cpu().numpy(), a_o), ctx


def test_mask_nonfinite_sets_status():
    d = 3000
    for bad in (float("nan"), float("inf"), -float("inf")):
        x = synth.laplace((d,), 1, 1).cuda()
        x[1234] = bad
        tier = torch.full((d,), 7, dtype=torch.uint8, device="cuda")
        fidx = torch.empty(d, dtype=torch.int32, device="cuda")
        aidx = torch.empty(d, dtype=torch.int32, device="cuda")
        counts = torch.full((4,), 9, dtype=torch.int32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        spax.spax_build_mask(x, spax.mask_params(spax.MASK_TOPK, k_full=10, k_approx=10), tier,
                             fidx, aidx, counts, status)
        torch.cuda.synchronize()
        assert status.item() == spax.ERR_NONFINITE
        assert not tier.any() and not counts.any()


def test_mask_host_errors():
    x = torch.zeros(100, device="cuda")
    t = torch.empty(100, dtype=torch.uint8, device="cuda")
    i = torch.empty(100, dtype=torch.int32, device="cuda")
    c = torch.empty(4, dtype=torch.int32, device="cuda")
    s = torch.zeros(1, dtype=torch.int32, device="cuda")
    bad = [spax.mask_params(spax.MASK_TOPK, k_full=60, k_approx=41),
           spax.mask_params(spax.MASK_TOPK, k_full=-1),
           spax.mask_params(spax.MASK_THRESHOLD, t_skip=1.0, t_full=0.5),
           spax.mask_params(spax.MASK_THRESHOLD, t_skip=-1.0, t_full=0.5),
           spax.mask_params(spax.MASK_GUIDED, t_skip=0.1, t_full=0.2, s_skip_bp=6000, s_below_full_bp=5000),
           spax.mask_params(9)]
    for prm in bad:
        with pytest.raises(spax.SpaxError) as e:
            spax.spax_build_mask(x, prm, t, i, i, c, s)
        assert e.value.status == spax.ERR_ARG
    big = torch.zeros(spax.MASK_MAX_DIN + 1, device="cuda")
    bt = torch.empty(big.numel(), dtype=torch.uint8, device="cuda")
    bi = torch.empty(big.numel(), dtype=torch.int32, device="cuda")
    with pytest.raises(spax.SpaxError) as e:
        spax.spax_build_mask(big, spax.mask_params(spax.MASK_TOPK), bt, bi, bi, c, s)
    assert e.value.status == spax.ERR_SHAPE


# ----------------------------------------------------------------------------- tiered GEMV

SPLITS = [(0.25, 0.25), (1.0, 0.0), (0.0, 1.0), (0.0, 0.0), (0.3, 0.0), (0.0, 0.3), (0.1, 0.6),
          (0.5, 0.4)]


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(128, 1), (1152, 300), (4096, 1024), (6144, 700), (22016, 256)])
def test_tiered_gemv_parity(fmt, d_out, d_in):
    W = _w(d_out, d_in, 200 + d_out % 89)
    gm = GpuMatrix(W, fmt)
    pools = oracle.pack(bf16_bits(W), fmt)
    x = synth.laplace((d_in,), d_out, 9).cuda()
    for f, a in SPLITS:
        kf = int(f * d_in + 0.5)
        ka = min(int(a * d_in + 0.5), d_in - kf)
        prm = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka)
        check_token(gm, pools, x, prm)


def test_tiered_gemv_deterministic():
    W = _w(4096, 4096, 300)
    gm = GpuMatrix(W, 0)
    x = synth.laplace((4096,), 3, 3).cuda()
    prm = spax.mask_params(spax.MASK_TOPK, k_full=1024, k_approx=1024)
    ys = [gm.token(x, prm)["y"] for _ in range(4)]
    for y in ys[1:]:
        assert np.array_equal(y.view(np.uint32), ys[0].view(np.uint32))


def test_tiered_gemv_many_columns_per_cta():
    # more selected columns per CTA than its shared-memory metadata holds: several chunks
    d_out, d_in = 16384, 20000
    W = _w(d_out, d_in, 301)
    gm = GpuMatrix(W, 0)
    S, R = spax.spax_gemv_plan(spax.OP_TIERED_GEMV, d_out, d_in)
    assert d_in / S > 1024
    pools = oracle.pack(bf16_bits(W), 0)
    x = synth.laplace((d_in,), 4, 4).cuda()
    rows = np.arange(0, d_out, 97, dtype=np.int32)
    check_token(gm, pools, x, spax.mask_params(spax.MASK_TOPK, k_full=0, k_approx=d_in), rows)
    check_token(gm, pools, x, spax.mask_params(spax.MASK_TOPK, k_full=d_in // 2, k_approx=d_in // 2), rows)


def test_tiered_gemv_bad_lists_set_status():
    W = _w(1024, 512, 302)
    gm = GpuMatrix(W, 0)
    x = synth.laplace((512,), 5, 5).cuda()
    # counts out of range: treated as empty, status INDEX
    gm.counts.copy_(torch.tensor([600, 0, 0, 0], dtype=torch.int32))
    gm.status.zero_()
    spax.spax_tiered_gemv(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status, gm.ws)
    torch.cuda.synchronize()
    assert gm.status.item() == spax.ERR_INDEX and not gm.y.any()
    # one index out of range: that column contributes zero, status INDEX
    gm.fidx[:3].copy_(torch.tensor([5, 100000, 7], dtype=torch.int32))
    gm.counts.copy_(torch.tensor([3, 0, 0, 0], dtype=torch.int32))
    gm.status.zero_()
    spax.spax_tiered_gemv(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status, gm.ws)
    torch.cuda.synchronize()
    assert gm.status.item() == spax.ERR_INDEX
    tier = np.zeros(512, np.uint8)
    tier[[5, 7]] = 2
    pools = oracle.pack(bf16_bits(W), 0)
    y_ref = oracle.tiered_gemv(*pools, 0, 1024, 512, x.cpu().numpy(), tier)
    check_y(gm.y.cpu().numpy(), y_ref)
    # the workspace is still consistent afterwards: a normal call is correct
    check_token(gm, pools, x, spax.mask_params(spax.MASK_TOPK, k_full=100, k_approx=100))


def test_gemv_host_errors():
    W = _w(1024, 512, 303)
    gm = GpuMatrix(W, 0)
    x = torch.zeros(512, device="cuda")
    small_ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(spax.SpaxError) as e:
        spax.spax_tiered_gemv(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status, small_ws)
    assert e.value.status == spax.ERR_WORKSPACE
    bad = spax.PackedMatrix(1000, 512, 0, gm.pm.full, gm.pm.approx)
    y = torch.empty(1000, device="cuda")
    with pytest.raises(spax.SpaxError) as e:
        spax.spax_tiered_gemv(bad, x, gm.fidx, gm.aidx, gm.counts, y, gm.status, gm.ws)
    assert e.value.status == spax.ERR_SHAPE


# ----------------------------------------------------------------------------- dense GEMV

@pytest.mark.parametrize("d_out,d_in", [(128, 1), (1152, 300), (4096, 4096), (22016, 256)])
def test_dense_gemv_parity(d_out, d_in):
    W = _w(d_out, d_in, 400 + d_out % 83)
    gm = GpuMatrix(W, 0)
    x = synth.laplace((d_in,), 6, d_out).cuda()
    y = gm.dense(x)
    check_y(y, oracle.dense_gemv(bf16_bits(W), x.cpu().numpy()))


# ----------------------------------------------------------------------------- calibration

@pytest.mark.parametrize("n_tok,d_in", [(1, 1), (3, 1000), (512, 4096), (64, 14336)])
def test_calibrate_parity(n_tok, d_in):
    X = synth.laplace((n_tok, d_in), 7, n_tok).cuda()
    ws = torch.empty(spax.spax_workspace_bytes(spax.OP_CALIBRATE, 0, d_in), dtype=torch.uint8,
                     device="cuda")
    t = torch.empty(2, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for s1, s2 in [(0, 10000), (3000, 6500), (5000, 7500), (7000, 8500), (9999, 9999)]:
        spax.spax_calibrate_thresholds(X, s1, s2, t, st, ws)
        torch.cuda.synchronize()
        ost, t1, t2 = oracle.calibrate(X.cpu().numpy(), s1, s2)
        assert st.item() == 0 and ost == 0
        assert t.cpu().tolist() == [t1, t2]


def test_calibrate_nonfinite_sets_status():
    X = synth.laplace((4, 100), 8, 1).cuda()
    X[2, 3] = float("nan")
    ws = torch.empty(spax.spax_workspace_bytes(spax.OP_CALIBRATE, 0, 100), dtype=torch.uint8,
                     device="cuda")
    t = torch.empty(2, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    spax.spax_calibrate_thresholds(X, 5000, 7500, t, st, ws)
    torch.cuda.synchronize()
    assert st.item() == spax.ERR_NONFINITE
