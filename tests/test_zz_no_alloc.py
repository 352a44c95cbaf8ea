"""spax_tiered_gemv_fixed_scratch (the tiered GEMV on the library's own per-device scratch array,
no workspace argument, no allocation) against spax_tiered_gemv, through the C ABI.

Each case runs the fixed-scratch call twice in a row on fresh tokens and compares each result with
the workspace entry point within the parity tolerance. Shapes of different split plans alternate,
so the partial-sum words one shape leaves at zero must serve the next. This file is collected last on
purpose: it must pass in a fresh process and after every other GPU test.
"""
import numpy as np
import pytest
import torch

from conftest import cuda_ok

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

if cuda_ok():
    from tiered_weight_gemv_b200 import spax, synth
    from gpu_helpers import GpuMatrix, check_y


def _token(gm, x, params):
    """Mask once, then both GEMV entry points on the same lists; returns (y_ws, y_fixed, status)."""
    gm.status.zero_()
    spax.spax_build_mask(x, params, gm.tier, gm.fidx, gm.aidx, gm.counts, gm.status)
    spax.spax_tiered_gemv(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status, gm.ws)
    y_ws = gm.y.clone()
    gm.y.fill_(float("nan"))  # every output row must be written again
    spax.spax_tiered_gemv_fixed_scratch(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status)
    torch.cuda.synchronize()
    return y_ws.cpu().numpy(), gm.y.cpu().numpy(), int(gm.status.item())


SHAPES = [(4096, 4096), (1152, 640), (22016, 4096), (4096, 11008), (640, 33)]


@pytest.mark.parametrize("fmt", [0, 1])
def test_fixed_scratch_matches_workspace_call(fmt):
    mats = [GpuMatrix(synth.weight(d_out, d_in, 3, 700 + i, device="cuda"), fmt)
            for i, (d_out, d_in) in enumerate(SHAPES)]
    for call in range(2):  # two calls in a row per shape, shapes interleaved
        for i, gm in enumerate(mats):
            x = synth.laplace((gm.d_in,), 5 + call, 800 + i, device="cuda")
            kf = max(1, gm.d_in * 3 // 10)
            params = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=kf)
            y_ws, y_fx, st = _token(gm, x, params)
            assert st == 0
            assert np.all(np.isfinite(y_fx)), f"{gm.d_out}x{gm.d_in}: unwritten rows"
            check_y(y_fx, y_ws, f"{gm.d_out}x{gm.d_in} call {call}")


def test_fixed_scratch_unsplit_plan_uses_no_scratch():
    # d_out = 2^20 rows and one column: one split per row tile (512 tiles, more CTAs than SMs),
    # so no partial sums at all; every row is written straight from its tile, y = x_0 * W[:, 0].
    d_out, d_in = 1 << 20, 1
    assert spax.spax_fixed_scratch_bytes() == 4 << 20
    assert spax.spax_gemv_plan(spax.OP_TIERED_GEMV, d_out, d_in)[0] == 1
    W = synth.weight(d_out, d_in, 3, 790, device="cuda")
    gm = GpuMatrix(W, 0)
    x = torch.full((d_in,), -1.75, dtype=torch.float32, device="cuda")
    for kf, ka in [(1, 0), (0, 1), (0, 0)]:
        y_ws, y_fx, st = _token(gm, x, spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka))
        assert st == 0
        assert np.array_equal(y_fx, y_ws)
        if kf:
            assert np.array_equal(y_fx, (-1.75 * W[:, 0].float()).cpu().numpy())
        if kf + ka == 0:
            assert np.all(y_fx == 0.0)
