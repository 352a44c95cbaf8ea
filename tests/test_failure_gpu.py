"""Failure detection on the GPU without a fault: a split-K wait that runs out (needs a B200).

The CTAs that split a row tile wait for one another's partial sums, with a bounded wait. The test
hook spax_test_tiered_gemv_timeout launches the list-driven GEMV with the last split of every tile
left out, so the partial sums those waits need never arrive. The kernel must give up within its
limit, set the status word to SPAX_ERR_TIMEOUT and leave the context usable. The workspace then
holds flagged words; once it is zeroed again, the next call must give exactly the result of a
call on a fresh workspace, and the oracle's result within the parity tolerance.
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


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(4096, 4096), (22016, 4096)])
def test_split_wait_runs_out_and_workspace_recovers(fmt, d_out, d_in):
    W = synth.weight(d_out, d_in, 21, 1 + fmt, device="cuda")
    gm = GpuMatrix(W, fmt)
    assert spax.spax_gemv_plan(spax.OP_TIERED_GEMV, d_out, d_in, fmt)[0] >= 2
    x = synth.laplace((d_in,), 21, 3, device="cuda")
    prm = spax.mask_params(spax.MASK_TOPK, k_full=d_in * 3 // 10, k_approx=d_in * 3 // 10)
    ref = gm.token(x, prm)  # a call on a fresh workspace
    assert ref["status"] == 0

    gm.status.zero_()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    spax.spax_test_tiered_gemv_timeout(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status,
                                       ws=gm.ws, wait_limit_ns=20_000_000)
    t1.record()
    torch.cuda.synchronize()  # the context is still usable: this returns
    assert int(gm.status.item()) == spax.ERR_TIMEOUT
    assert 15.0 <= t0.elapsed_time(t1) < 2000.0  # the waits ran to their 20 ms limit and stopped
    # Every word that arrived was read and cleared by the CTA that sums its rows. Words stay
    # flagged only where the missing split owned a non-empty slice of a tile's rows: it was the
    # one to read the other splits' words for those rows.
    S, R = spax.spax_gemv_plan(spax.OP_TIERED_GEMV, d_out, d_in, fmt)
    dirty = False
    for r0 in range(0, d_out, R):
        n4 = min(R, d_out - r0) // 4
        c4 = -(-n4 // S)
        dirty |= (S - 1) * c4 < n4
    assert (torch.count_nonzero(gm.ws).item() > 0) == dirty

    gm.ws.zero_()  # the documented recovery: zero the workspace again
    for _ in range(2):
        again = gm.token(x, prm)
        assert again["status"] == 0
        assert np.array_equal(again["y"], ref["y"])
    pools = oracle.pack(bf16_bits(W), fmt)
    rows = np.unique(np.concatenate([np.arange(0, d_out, 41), np.arange(d_out - 4, d_out)]))
    y_ref = oracle.tiered_gemv(*pools, fmt, d_out, d_in, x.cpu().numpy(), again["tier"], rows=rows)
    check_y(again["y"][rows], y_ref)


def test_timeout_hook_rejects_bad_arguments():
    gm = GpuMatrix(synth.weight(4096, 4096, 21, 5, device="cuda"), 0)
    x = torch.zeros(4096, device="cuda")
    with pytest.raises(spax.SpaxError):  # a wait limit outside [1 ms, 2 s]
        spax.spax_test_tiered_gemv_timeout(gm.pm, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status,
                                           ws=gm.ws, wait_limit_ns=10)
    one = GpuMatrix(synth.weight(1 << 20, 1, 21, 6, device="cuda"), 0)  # one split per tile
    x1 = torch.ones(1, device="cuda")
    with pytest.raises(spax.SpaxError):
        spax.spax_test_tiered_gemv_timeout(one.pm, x1, one.fidx, one.aidx, one.counts, one.y,
                                           one.status, ws=one.ws)
