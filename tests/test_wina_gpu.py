"""The WINA score option (columns ranked by |x_j| * ||W[:, j]||, TopK-Guided §1 and §C.1) against
the oracle, through the C ABI (needs a B200).

The column norms follow one fixed definition (fp64 squares summed in row order, sqrt, fp32), so
the library's norms must equal the oracle's bit for bit; the score is one IEEE fp32 product, so
the tiers, lists and counts must equal the oracle's rule on its own scores bit for bit; y is the
product on x (not on the score) and is checked against the fp64 oracle within the tolerance.
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


def _norms(W):
    n = torch.full((W.shape[1],), float("nan"), device="cuda")
    spax.spax_column_norms(W, n)
    torch.cuda.synchronize()
    return n


def _run(gm, x, norms, prm):
    d_in, d_out = gm.d_in, gm.d_out
    o = dict(tier=torch.full((d_in,), 7, dtype=torch.uint8, device="cuda"),
             fidx=torch.full((d_in,), -5, dtype=torch.int32, device="cuda"),
             aidx=torch.full((d_in,), -5, dtype=torch.int32, device="cuda"),
             counts=torch.full((4,), -5, dtype=torch.int32, device="cuda"),
             y=torch.full((d_out,), float("nan"), device="cuda"),
             status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    spax.spax_masked_gemv_wina(gm.pm, x, norms, prm, o["y"], o["status"], gm.ws, tier=o["tier"],
                               full_idx=o["fidx"], approx_idx=o["aidx"], counts=o["counts"])
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}


@pytest.mark.parametrize("d_out,d_in", [(128, 1), (640, 33), (1152, 300), (4096, 4096),
                                        (4096, 11008), (22016, 4096)])
def test_column_norms_bitexact(d_out, d_in):
    W = synth.weight(d_out, d_in, 14, 1 + d_in % 13, device="cuda")
    assert np.array_equal(_norms(W).cpu().numpy(), oracle.column_norms(bf16_bits(W)))


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(640, 33), (1152, 300), (4096, 4096), (4096, 11008)])
def test_wina_masked_gemv_matches_oracle(fmt, d_out, d_in):
    # columns of unequal scale, so the norms reorder the ranking
    W = synth.weight(d_out, d_in, 14, 20 + d_in % 11, device="cuda")
    scale = synth.log_uniform((d_in,), 14, 21, 0.25, 4.0, device="cuda")
    W = (W.float() * scale[None, :]).to(torch.bfloat16).contiguous()
    gm = GpuMatrix(W, fmt)
    Wb = bf16_bits(W)
    pools = oracle.pack(Wb, fmt)
    norms = _norms(W)
    n_host = oracle.column_norms(Wb)
    assert np.array_equal(norms.cpu().numpy(), n_host)
    x = synth.laplace((d_in,), 14, 22 + d_out % 7, device="cuda")
    xh = x.cpu().numpy()
    score = oracle.wina_scores(xh, n_host)
    rows = np.unique(np.concatenate([np.arange(0, d_out, 37), np.arange(d_out - 3, d_out)]))
    kf, ka = (3 * d_in + 5) // 10, (3 * d_in + 5) // 10
    ts, tf = np.quantile(score, [0.4, 0.7]).astype(np.float32)
    # a TopK guess of the boundary keys is on the score, like every other key of this rule
    gs, gf = np.quantile(score, [1 - (kf + ka) / d_in, 1 - kf / d_in])
    ys = []
    for prm in [spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka),
                spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka, t_skip=float(gs),
                                 t_full=float(gf)),
                spax.mask_params(spax.MASK_THRESHOLD, t_skip=float(ts), t_full=float(tf))]:
        r = _run(gm, x, norms, prm)
        ys.append(r["y"])
        assert r["status"][0] == 0
        op = oracle_params(prm)
        st, t_o, f_o, a_o, c_o = oracle.tiers(score, op.pop("mode"), **op)
        assert st == 0 and np.array_equal(r["counts"], c_o) and np.array_equal(r["tier"], t_o)
        assert np.array_equal(r["fidx"][: c_o[0]], f_o) and np.array_equal(r["aidx"][: c_o[1]], a_o)
        y_ref = oracle.tiered_gemv(*pools, fmt, d_out, d_in, xh, t_o, rows=rows)
        check_y(r["y"][rows], y_ref)
    assert np.array_equal(ys[0], ys[1]), "the guess changed y"


def test_wina_with_equal_norms_is_the_magnitude_rule():
    # norms all 4.0 (a power of two): the scores keep the order of |x| exactly, so the WINA
    # kernel must return what spax_masked_gemv returns, bit for bit
    d_out, d_in = 4096, 4096
    gm = GpuMatrix(synth.weight(d_out, d_in, 15, 1, device="cuda"), 0)
    x = synth.laplace((d_in,), 15, 2, device="cuda")
    prm = spax.mask_params(spax.MASK_TOPK, k_full=1229, k_approx=1229)
    r = _run(gm, x, torch.full((d_in,), 4.0, device="cuda"), prm)
    y = torch.empty(d_out, device="cuda")
    tier = torch.empty(d_in, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    spax.spax_masked_gemv(gm.pm, x, prm, y, st, gm.ws, tier=tier)
    torch.cuda.synchronize()
    assert st.item() == 0 and r["status"][0] == 0
    assert np.array_equal(r["tier"], tier.cpu().numpy()) and np.array_equal(r["y"], y.cpu().numpy())


def test_wina_nonfinite_and_host_errors():
    d_out, d_in = 1152, 300
    gm = GpuMatrix(synth.weight(d_out, d_in, 16, 1, device="cuda"), 0)
    x = synth.laplace((d_in,), 16, 2, device="cuda")
    norms = torch.ones(d_in, device="cuda")
    norms[40] = float("inf")
    r = _run(gm, x, norms, spax.mask_params(spax.MASK_TOPK, k_full=30, k_approx=30))
    assert r["status"][0] == spax.ERR_NONFINITE
    assert np.all(r["tier"] == 0) and np.all(r["counts"] == 0) and np.all(r["y"] == 0.0)
    y = torch.zeros(d_out, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        spax.spax_masked_gemv_wina(gm.pm, x, torch.ones(d_in - 1, device="cuda"),
                                   spax.mask_params(spax.MASK_TOPK, k_full=1, k_approx=1), y, st,
                                   gm.ws)
