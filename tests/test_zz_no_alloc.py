"""spax_tiered_gemv_fixed_scratch (the tiered GEMV on the library's own per-device scratch array,
no workspace argument, no allocation) against spax_tiered_gemv and the oracle, through the C ABI.

Some callers cannot allocate device memory at the point where they run the GEMV, for example code
inside an allocator's own callbacks or a plugin whose host owns every device allocation. The
fixed-scratch entry point serves them. It runs the same kernel with the same split plan as the
workspace entry point, so its y must equal that call's y bit for bit. Each shape is also checked
against the fp64 oracle within the parity tolerance.

Each case makes two calls in a row on fresh tokens. Shapes of different split plans alternate, so
the partial-sum words that one shape leaves at zero must serve the next. The failure path is
covered too. A call whose split-K wait runs out (the test hook leaves one split out) leaves
flagged words behind. After spax_fixed_scratch_reset, the next call must be exact again.

This file is collected last on purpose: it must pass in a fresh process and after every other GPU
test.
"""
import numpy as np
import pytest
import torch

from conftest import cuda_ok

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

if cuda_ok():
    import oracle
    from tiered_weight_gemv_b200 import spax, synth
    from gpu_helpers import GpuMatrix, bf16_bits, check_y


@pytest.fixture(scope="module", autouse=True)
def _built(oracle_lib):
    return oracle_lib


def _token(gm, x, params):
    """Mask once, then both GEMV entry points on the same lists; returns (y_ws, y_fixed, status,
    tier)."""
    gm.status.zero_()
    spax.spax_build_mask(x, params, gm.tier, gm.fidx, gm.aidx, gm.counts, gm.status)
    spax.spax_tiered_gemv(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status, gm.ws)
    y_ws = gm.y.clone()
    gm.y.fill_(float("nan"))  # every output row must be written again
    spax.spax_tiered_gemv_fixed_scratch(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status)
    torch.cuda.synchronize()
    return y_ws.cpu().numpy(), gm.y.cpu().numpy(), int(gm.status.item()), gm.tier.cpu().numpy()


SHAPES = [(4096, 4096), (1152, 640), (22016, 4096), (4096, 11008), (640, 33)]


def _rows(d_out):
    return np.unique(np.concatenate([np.arange(0, d_out, 29), np.arange(max(0, d_out - 5), d_out)]))


@pytest.mark.parametrize("fmt", [0, 1])
def test_fixed_scratch_matches_workspace_call(fmt):
    Ws = [synth.weight(d_out, d_in, 3, 700 + i, device="cuda") for i, (d_out, d_in) in enumerate(SHAPES)]
    mats = [GpuMatrix(W, fmt) for W in Ws]
    pools = [oracle.pack(bf16_bits(W), fmt) for W in Ws]
    for call in range(2):  # two calls in a row per shape, shapes interleaved
        for i, gm in enumerate(mats):
            x = synth.laplace((gm.d_in,), 5 + call, 800 + i, device="cuda")
            kf = max(1, gm.d_in * 3 // 10)
            params = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=kf)
            y_ws, y_fx, st, tier = _token(gm, x, params)
            what = f"{gm.d_out}x{gm.d_in} call {call}"
            assert st == 0
            assert np.all(np.isfinite(y_fx)), f"{what}: unwritten rows"
            assert np.array_equal(y_fx, y_ws), f"{what}: differs from the workspace call"
            rows = _rows(gm.d_out)
            y_ref = oracle.tiered_gemv(*pools[i], fmt, gm.d_out, gm.d_in, x.cpu().numpy(), tier,
                                       rows=rows)
            check_y(y_fx[rows], y_ref, what)


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
        y_ws, y_fx, st, _ = _token(gm, x, spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=ka))
        assert st == 0
        assert np.array_equal(y_fx, y_ws)
        if kf:
            assert np.array_equal(y_fx, (-1.75 * W[:, 0].float()).cpu().numpy())
        if kf + ka == 0:
            assert np.all(y_fx == 0.0)


def test_fixed_scratch_reset_after_a_wait_ran_out():
    # A fixed-scratch GEMV whose split-K wait runs out (the test hook leaves the last split of
    # every tile out) reports ERR_TIMEOUT and leaves flagged words in the array. After
    # spax_fixed_scratch_reset the next call is exact again, twice in a row.
    d_out, d_in = 4096, 4096
    W = synth.weight(d_out, d_in, 3, 795, device="cuda")
    gm = GpuMatrix(W, 0)
    assert spax.spax_gemv_plan(spax.OP_TIERED_GEMV, d_out, d_in)[0] >= 2
    x = synth.laplace((d_in,), 3, 796, device="cuda")
    params = spax.mask_params(spax.MASK_TOPK, k_full=1229, k_approx=1229)
    gm.status.zero_()
    spax.spax_build_mask(x, params, gm.tier, gm.fidx, gm.aidx, gm.counts, gm.status)
    spax.spax_test_tiered_gemv_timeout(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status,
                                       ws=None, wait_limit_ns=20_000_000)
    torch.cuda.synchronize()
    assert int(gm.status.item()) == spax.ERR_TIMEOUT
    spax.spax_fixed_scratch_reset()
    for _ in range(2):
        y_ws, y_fx, st, _ = _token(gm, x, params)
        assert st == 0
        assert np.array_equal(y_fx, y_ws)
