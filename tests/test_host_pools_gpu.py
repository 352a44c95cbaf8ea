"""Weights offloaded to host memory (the SpAx setting): the packed pools in page-locked host memory,
read by the same kernels over the host link, through the C ABI (needs a B200).

Nothing in the arithmetic depends on where the pools live, so every result must equal the
device-pool result bit for bit: y of the masked GEMV (and its mask outputs), of the two-call
path and of the dense GEMV. The host-pool results are also checked against the oracle on the
same seeded inputs: tiers, lists and counts bit-exact, y within the parity tolerance (the tiered
product from the oracle's own packed pools; the dense product from the bf16 matrix).
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


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("d_out,d_in", [(640, 33), (4096, 4096), (4096, 11008)])
def test_host_pools_give_device_results(fmt, d_out, d_in):
    W = synth.weight(d_out, d_in, 17, 1 + d_in % 5, device="cuda")
    gm = GpuMatrix(W, fmt)
    host = spax.packed_to_host(gm.pm)
    assert host.full.is_pinned() and not host.full.is_cuda
    x = synth.laplace((d_in,), 17, 2, device="cuda")
    kf = (3 * d_in + 5) // 10
    prm = spax.mask_params(spax.MASK_TOPK, k_full=kf, k_approx=kf)
    outs = []
    for pm in (gm.pm, host):
        y = torch.full((d_out,), float("nan"), device="cuda")
        tier = torch.empty(d_in, dtype=torch.uint8, device="cuda")
        fidx = torch.full((d_in,), -5, dtype=torch.int32, device="cuda")
        aidx = torch.full((d_in,), -5, dtype=torch.int32, device="cuda")
        counts = torch.full((4,), -5, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        spax.spax_masked_gemv(pm, x, prm, y, st, gm.ws, tier=tier, full_idx=fidx,
                              approx_idx=aidx, counts=counts)
        torch.cuda.synchronize()
        assert st.item() == 0
        c = counts.cpu().numpy()
        outs.append((y.cpu().numpy(), tier.cpu().numpy(), fidx[: c[0]].cpu().numpy(),
                     aidx[: c[1]].cpu().numpy(), c))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    # the host-pool run against the oracle: the rule bit-exact, y within tolerance
    y_h, tier_h, fidx_h, aidx_h, c_h = outs[1]
    xn = x.cpu().numpy()
    op = oracle_params(prm)
    st_o, tier_o, fi_o, ai_o, c_o = oracle.tiers(xn, op.pop("mode"), **op)
    assert st_o == 0 and np.array_equal(tier_h, tier_o) and np.array_equal(c_h, c_o)
    assert np.array_equal(fidx_h, fi_o) and np.array_equal(aidx_h, ai_o)
    pools = oracle.pack(bf16_bits(W), fmt)
    y_ref = oracle.tiered_gemv(*pools, fmt, d_out, d_in, xn, tier_o)
    check_y(y_h, y_ref, "masked GEMV, host pools")
    # two-call path on the same lists
    gm.token(x, prm)
    torch.cuda.synchronize()
    y_dev = gm.y.clone()
    gm.y.fill_(float("nan"))
    spax.spax_tiered_gemv(host, x, gm.fidx, gm.aidx, gm.counts, gm.y, gm.status, gm.ws)
    torch.cuda.synchronize()
    assert gm.status.item() == 0 and torch.equal(gm.y, y_dev)
    check_y(gm.y.cpu().numpy(), y_ref, "two-call path, host pools")
    if fmt == 0:  # dense over the same bf16 pool
        ys = []
        for full in (gm.pm.full, host.full):
            y = torch.full((d_out,), float("nan"), device="cuda")
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            spax.spax_dense_gemv(full, x, y, d_out, d_in, st, gm.dense_ws)
            torch.cuda.synchronize()
            assert st.item() == 0
            ys.append(y.cpu().numpy())
        assert np.array_equal(ys[0], ys[1])
        check_y(ys[1], oracle.dense_gemv(bf16_bits(W), xn), "dense GEMV, host pool")
