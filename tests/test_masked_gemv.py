"""spax_masked_gemv (mask and tiered GEMV in one launch) against the two-call path and the oracle,
through the C ABI (needs a B200).

The fused kernel runs the same rule and the same GEMV code, so its tiers, lists and counts must be
bit-identical to spax_build_mask's and its y bit-identical to spax_tiered_gemv's on those lists;
y is also checked against the fp64 oracle within the parity tolerance.
"""
import numpy as np
import pytest
import torch

from conftest import cuda_ok

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

if cuda_ok():
    import oracle
    from tiered_weight_gemv_b200 import spax, synth
    from gpu_helpers import GpuMatrix, bf16_bits, check_y, oracle_params


@pytest.fixture(scope="module", autouse=True)
def _built(oracle_lib):
    return oracle_lib


def _cases(d):
    kf, ka = d // 3, d // 4
    return [spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka),
            spax.mask_params(spax.MASK_TOPK, k_full=0, k_approx=0),
            spax.mask_params(spax.MASK_TOPK, k_full=d, k_approx=0),
            spax.mask_params(spax.MASK_THRESHOLD, t_skip=0.5, t_full=1.2),
            spax.mask_params(spax.MASK_GUIDED, t_skip=0.36, t_full=0.69, s_skip_bp=3000,
                             s_below_full_bp=6500, delta_bp=100)]


def _fused(gm, x, prm, outputs=True):
    d_in, d_out = gm.d_in, gm.d_out
    o = dict(tier=torch.full((d_in,), 7, dtype=torch.uint8, device="cuda"),
             fidx=torch.full((d_in,), -5, dtype=torch.int32, device="cuda"),
             aidx=torch.full((d_in,), -5, dtype=torch.int32, device="cuda"),
             counts=torch.full((4,), -5, dtype=torch.int32, device="cuda"),
             y=torch.full((d_out,), float("nan"), device="cuda"),
             status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    if outputs:
        spax.spax_masked_gemv(gm.pm, x, prm, o["y"], o["status"], gm.ws, tier=o["tier"],
                              full_idx=o["fidx"], approx_idx=o["aidx"], counts=o["counts"])
    else:
        spax.spax_masked_gemv(gm.pm, x, prm, o["y"], o["status"], gm.ws)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(128, 1), (640, 33), (1152, 300), (4096, 4096),
                                        (22016, 4096), (4096, 11008)])
def test_masked_gemv_equals_two_calls(fmt, d_out, d_in):
    W = synth.weight(d_out, d_in, 9, 900 + d_in % 97, device="cuda")
    gm = GpuMatrix(W, fmt)
    pools = oracle.pack(bf16_bits(W), fmt)
    x = synth.laplace((d_in,), 9, 901 + d_out % 89, device="cuda")
    rows = np.unique(np.concatenate([np.arange(0, d_out, 37), np.arange(d_out - 3, d_out)]))
    for prm in _cases(d_in):
        g = gm.token(x, prm)  # two calls: spax_build_mask + spax_tiered_gemv
        f = _fused(gm, x, prm)
        c = g["counts"]
        assert f["status"][0] == 0
        assert np.array_equal(f["counts"], c)
        assert np.array_equal(f["tier"], g["tier"])
        assert np.array_equal(f["fidx"][: c[0]], g["fidx"]) and np.array_equal(f["aidx"][: c[1]], g["aidx"])
        assert np.array_equal(f["y"], g["y"]), "fused y differs from the two-call y"
        y_ref = oracle.tiered_gemv(*pools, fmt, d_out, d_in, x.cpu().numpy(), g["tier"], rows=rows)
        check_y(f["y"][rows], y_ref)
        # without the optional outputs: the same y, nothing else written
        f2 = _fused(gm, x, prm, outputs=False)
        assert np.array_equal(f2["y"], g["y"])
        assert np.all(f2["tier"] == 7) and np.all(f2["counts"] == -5)


def test_masked_gemv_oracle_lists():
    d_out, d_in = 4096, 4096
    W = synth.weight(d_out, d_in, 9, 950, device="cuda")
    gm = GpuMatrix(W, 0)
    x = synth.laplace((d_in,), 9, 951, device="cuda")
    x[::5] = x[3]  # many equal keys at arbitrary boundaries
    prm = spax.mask_params(spax.MASK_TOPK, k_full=1000, k_approx=900)
    f = _fused(gm, x, prm)
    op = oracle_params(prm)
    st, t_o, f_o, a_o, c_o = oracle.tiers(x.cpu().numpy(), op.pop("mode"), **op)
    assert np.array_equal(f["counts"], c_o) and np.array_equal(f["tier"], t_o)
    assert np.array_equal(f["fidx"][: c_o[0]], f_o) and np.array_equal(f["aidx"][: c_o[1]], a_o)


def test_masked_gemv_nonfinite():
    d_out, d_in = 1152, 300
    gm = GpuMatrix(synth.weight(d_out, d_in, 9, 960, device="cuda"), 0)
    x = synth.laplace((d_in,), 9, 961, device="cuda")
    x[17] = float("inf")
    f = _fused(gm, x, spax.mask_params(spax.MASK_TOPK, k_full=10, k_approx=10))
    assert f["status"][0] == spax.ERR_NONFINITE
    assert np.all(f["tier"] == 0) and np.all(f["counts"] == 0) and np.all(f["y"] == 0.0)


def test_masked_gemv_host_errors():
    gm = GpuMatrix(synth.weight(128, 16, 9, 970, device="cuda"), 0)
    x = torch.zeros(16, device="cuda")
    y = torch.zeros(128, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(spax.SpaxError):
        spax.spax_masked_gemv(gm.pm, x, spax.mask_params(spax.MASK_TOPK, k_full=10, k_approx=10),
                              y, st, gm.ws)
    with pytest.raises(spax.SpaxError):
        spax.spax_masked_gemv(gm.pm, x, spax.mask_params(spax.MASK_THRESHOLD, t_skip=2.0,
                                                         t_full=1.0), y, st, gm.ws)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(spax.SpaxError):
        spax.spax_masked_gemv(gm.pm, x, spax.mask_params(spax.MASK_TOPK, k_full=1, k_approx=1),
                              y, st, small)
