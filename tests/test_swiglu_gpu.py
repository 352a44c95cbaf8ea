"""spax_masked_gemv_swiglu (the down projection fed from the gate/up output, x = silu(g) * u formed
in the kernel) against the oracle and against spax_masked_gemv, through the C ABI (needs a B200).

The kernel decides the tiers on its own fp32 x, so the checks follow that value: x_out must match
the oracle's fp64 silu(g) * u within the fp32 error of the formula (a few ulp), the tiers, lists
and counts must equal the oracle's rule applied to x_out bit for bit, and y must match the fp64
oracle product on x_out within the parity tolerance. spax_masked_gemv given x_out must return the
same y bit for bit (one definition of x everywhere in the kernel).
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

# |x_gpu - x_ref| <= X_REL * |x_ref|: expf within 2 ulp, then an add, a divide and a multiply
# each rounded once (<= 3.5 ulp of fp32 in all), with margin
X_REL = 6e-7


@pytest.fixture(scope="module", autouse=True)
def _built(oracle_lib):
    return oracle_lib


def _run(gm, gu, prm, outputs=True):
    d_in, d_out = gm.d_in, gm.d_out
    o = dict(x=torch.full((d_in,), float("nan"), device="cuda"),
             tier=torch.full((d_in,), 7, dtype=torch.uint8, device="cuda"),
             fidx=torch.full((d_in,), -5, dtype=torch.int32, device="cuda"),
             aidx=torch.full((d_in,), -5, dtype=torch.int32, device="cuda"),
             counts=torch.full((4,), -5, dtype=torch.int32, device="cuda"),
             y=torch.full((d_out,), float("nan"), device="cuda"),
             status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    kw = dict(x_out=o["x"], tier=o["tier"], full_idx=o["fidx"], approx_idx=o["aidx"],
              counts=o["counts"]) if outputs else {}
    spax.spax_masked_gemv_swiglu(gm.pm, gu, prm, o["y"], o["status"], gm.ws, **kw)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in o.items()}


def _check(gm, pools, gu, prm, rows):
    r = _run(gm, gu, prm)
    assert r["status"][0] == 0
    d = gm.d_in
    g, u = gu[:d].cpu().double().numpy(), gu[d:].cpu().double().numpy()
    x_ref = oracle.swiglu(g, u)
    assert np.all(np.abs(r["x"] - x_ref) <= X_REL * np.abs(x_ref) + 1e-37)
    op = oracle_params(prm)
    st, t_o, f_o, a_o, c_o = oracle.tiers(r["x"], op.pop("mode"), **op)
    assert st == 0 and np.array_equal(r["counts"], c_o) and np.array_equal(r["tier"], t_o)
    assert np.array_equal(r["fidx"][: c_o[0]], f_o) and np.array_equal(r["aidx"][: c_o[1]], a_o)
    y_ref = oracle.tiered_gemv(*pools, gm.fmt, gm.d_out, d, r["x"], t_o, rows=rows)
    check_y(r["y"][rows], y_ref)
    # the plain fused kernel on the same x gives the same y, bit for bit
    y2 = torch.full((gm.d_out,), float("nan"), device="cuda")
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    spax.spax_masked_gemv(gm.pm, torch.tensor(r["x"], device="cuda"), prm, y2, st2, gm.ws)
    torch.cuda.synchronize()
    assert st2.item() == 0 and np.array_equal(y2.cpu().numpy(), r["y"])
    # without the optional outputs: the same y
    assert np.array_equal(_run(gm, gu, prm, outputs=False)["y"], r["y"])
    return r


# (8192, 28672): x does not fit in shared memory beside the lists, and a split holds more positions
# than the stash, so the kernel forms silu(g) * u again for the product (the SwiGLU instance); the
# other shapes keep every x in shared memory and run the plain instance with the SwiGLU fetch.
@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(4096, 11008), (640, 33), (1152, 300), (256, 1),
                                        (8192, 28672)])
def test_swiglu_input_matches_oracle(fmt, d_out, d_in):
    W = synth.weight(d_out, d_in, 11, 1000 + d_in % 97, device="cuda")
    gm = GpuMatrix(W, fmt)
    pools = oracle.pack(bf16_bits(W), fmt)
    rows = np.unique(np.concatenate([np.arange(0, d_out, 41), np.arange(d_out - 3, d_out)]))
    gu = (2.0 * synth.laplace((2 * d_in,), 11, 1001 + d_out % 89, device="cuda")).contiguous()
    kf, ka = (3 * d_in + 5) // 10, (3 * d_in + 5) // 10
    # a TopK guess of the boundary keys: quantiles of |silu(g) * u| (computed here in fp64)
    xg = np.abs(oracle.swiglu(gu[:d_in].cpu().double().numpy(), gu[d_in:].cpu().double().numpy()))
    gs, gf = np.quantile(xg, [1 - (kf + ka) / d_in, 1 - kf / d_in])
    ys = []
    for prm in [spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka),
                spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka, t_skip=float(gs),
                                 t_full=float(gf)),
                spax.mask_params(spax.MASK_THRESHOLD, t_skip=0.2, t_full=0.9)]:
        ys.append(_check(gm, pools, gu, prm, rows)["y"])
    assert np.array_equal(ys[0], ys[1]), "the guess changed y"
    # an offset view of a larger buffer: g, u and x_out not 16-byte aligned (scalar path)
    big = torch.zeros(2 * d_in + 1, device="cuda")
    big[1:] = gu
    _check(gm, pools, big[1:], spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka), rows)


def test_chained_gate_up_to_down():
    """The Llama-2-7B MLP as the decoder runs it: tiered gate/up (one matrix, gate rows then up
    rows) on a Laplace mlp input, then the down projection fed from that output directly."""
    hidden, inter = 4096, 11008
    gate_up = GpuMatrix(torch.cat([synth.weight(inter, hidden, 12, 5, device="cuda"),
                                   synth.weight(inter, hidden, 12, 6, device="cuda")]), 0)
    down_W = synth.weight(hidden, inter, 12, 7, device="cuda")
    down = GpuMatrix(down_W, 0)
    pools = oracle.pack(bf16_bits(down_W), 0)
    x = synth.laplace((hidden,), 12, 8, device="cuda")
    gu = torch.empty(2 * inter, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kf = (3 * hidden + 5) // 10
    spax.spax_masked_gemv(gate_up.pm, x, spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=kf),
                          gu, st, gate_up.ws)
    torch.cuda.synchronize()
    assert st.item() == 0
    kd = (3 * inter + 5) // 10
    rows = np.unique(np.concatenate([np.arange(0, hidden, 29), [hidden - 1]]))
    r = _check(down, pools, gu, spax.mask_params(spax.MASK_TOPK, k_full=kd, k_approx=kd), rows)
    assert r["counts"][0] == kd and r["counts"][1] == kd


def test_swiglu_nonfinite():
    d_out, d_in = 1152, 300
    gm = GpuMatrix(synth.weight(d_out, d_in, 13, 1, device="cuda"), 0)
    gu = synth.laplace((2 * d_in,), 13, 2, device="cuda")
    for where, val in [(7, float("inf")), (d_in + 9, float("nan")), (11, float("-inf"))]:
        bad = gu.clone()
        bad[where] = val
        r = _run(gm, bad, spax.mask_params(spax.MASK_TOPK, k_full=30, k_approx=30))
        assert r["status"][0] == spax.ERR_NONFINITE
        assert np.all(r["tier"] == 0) and np.all(r["counts"] == 0) and np.all(r["y"] == 0.0)


def test_swiglu_host_errors():
    gm = GpuMatrix(synth.weight(128, 16, 13, 3, device="cuda"), 0)
    y = torch.zeros(128, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    prm = spax.mask_params(spax.MASK_TOPK, k_full=2, k_approx=2)
    with pytest.raises(ValueError):  # gu must hold 2 * d_in values
        spax.spax_masked_gemv_swiglu(gm.pm, torch.zeros(16, device="cuda"), prm, y, st, gm.ws)
    with pytest.raises(spax.SpaxError):
        spax.spax_masked_gemv_swiglu(gm.pm, torch.zeros(32, device="cuda"),
                                     spax.mask_params(spax.MASK_TOPK, k_full=10, k_approx=10),
                                     y, st, gm.ws)
