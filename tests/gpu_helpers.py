"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the oracle on
the same seeded inputs, and compare (tiers and lists bit-exact; y within the stated tolerance).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from tiered_weight_gemv_b200 import spax

# Output tolerance against the fp64 oracle on identical dequantised values.
REL_L2_TOL = 2e-3
MAX_ABS_FRAC_TOL = 1e-2


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "y"):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    assert y_gpu.shape == y_ref.shape
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite output"
    nref = np.linalg.norm(y_ref)
    if nref == 0.0:
        assert np.all(y_gpu == 0.0), f"{what}: expected exact zeros"
        return 0.0
    rel = np.linalg.norm(y_gpu - y_ref) / nref
    mabs = np.max(np.abs(y_gpu - y_ref))
    assert rel <= REL_L2_TOL, f"{what}: rel L2 {rel:.3e}"
    assert mabs <= MAX_ABS_FRAC_TOL * np.max(np.abs(y_ref)), f"{what}: max abs {mabs:.3e}"
    return rel


class GpuMatrix:
    """A packed matrix on the GPU plus everything one token's mask + GEMV needs."""

    def __init__(self, W: torch.Tensor, fmt: int):
        self.W = W
        self.d_out, self.d_in = W.shape
        self.fmt = fmt
        self.pm = spax.alloc_packed(self.d_out, self.d_in, fmt)
        spax.spax_pack_weights(W, fmt, self.pm)
        self.ws = spax.alloc_workspace(spax.OP_TIERED_GEMV, self.d_out, self.d_in)
        self.dense_ws = spax.alloc_workspace(spax.OP_DENSE_GEMV, self.d_out, self.d_in)
        dev = W.device
        self.tier = torch.empty(self.d_in, dtype=torch.uint8, device=dev)
        self.fidx = torch.empty(self.d_in, dtype=torch.int32, device=dev)
        self.aidx = torch.empty(self.d_in, dtype=torch.int32, device=dev)
        self.counts = torch.empty(4, dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.y = torch.empty(self.d_out, dtype=torch.float32, device=dev)

    def token(self, x: torch.Tensor, params):
        self.status.zero_()  # the kernels only ever set it
        spax.spax_build_mask(x, params, self.tier, self.fidx, self.aidx, self.counts, self.status)
        spax.spax_tiered_gemv(self.pm, x, self.fidx, self.aidx, self.counts, self.y, self.status,
                              self.ws)
        torch.cuda.synchronize()
        c = self.counts.cpu().numpy().copy()
        return dict(tier=self.tier.cpu().numpy().copy(), fidx=self.fidx[: c[0]].cpu().numpy().copy(),
                    aidx=self.aidx[: c[1]].cpu().numpy().copy(), counts=c,
                    y=self.y.cpu().numpy().copy(), status=int(self.status.item()))

    def dense(self, x: torch.Tensor):
        spax.spax_dense_gemv(self.pm.full, x, self.y, self.d_out, self.d_in, self.status,
                             self.dense_ws)
        torch.cuda.synchronize()
        return self.y.cpu().numpy().copy()


def oracle_params(params) -> dict:
    mode = {spax.MASK_THRESHOLD: oracle.MODE_THRESHOLD, spax.MASK_TOPK: oracle.MODE_TOPK,
            spax.MASK_GUIDED: oracle.MODE_GUIDED,
            spax.MASK_TOPK_SCALED: oracle.MODE_TOPK}[params.mode]  # the same columns as TOPK
    return dict(mode=mode, t_skip=params.t_skip, t_full=params.t_full, k_full=params.k_full,
                k_approx=params.k_approx, s_skip_bp=params.s_skip_bp,
                s_below_full_bp=params.s_below_full_bp, delta_bp=params.delta_bp)


def check_masked_equals_two_call(gm: GpuMatrix, x: torch.Tensor, params, g: dict):
    """spax_masked_gemv (mask + GEMV in one launch) on the same token: its tiers, lists, counts
    and y must equal the two-call results g bit for bit (same rule, same product order)."""
    d_in = gm.d_in
    tier = torch.full((d_in,), 7, dtype=torch.uint8, device=x.device)
    fidx = torch.full((d_in,), -5, dtype=torch.int32, device=x.device)
    aidx = torch.full((d_in,), -5, dtype=torch.int32, device=x.device)
    counts = torch.full((4,), -5, dtype=torch.int32, device=x.device)
    y = torch.full((gm.d_out,), float("nan"), device=x.device)
    st = torch.zeros(1, dtype=torch.int32, device=x.device)
    spax.spax_masked_gemv(gm.pm, x, params, y, st, gm.ws, tier=tier, full_idx=fidx,
                          approx_idx=aidx, counts=counts)
    torch.cuda.synchronize()
    c = counts.cpu().numpy()
    assert st.item() == 0 and np.array_equal(c, g["counts"])
    assert np.array_equal(tier.cpu().numpy(), g["tier"])
    assert np.array_equal(fidx[: c[0]].cpu().numpy(), g["fidx"])
    assert np.array_equal(aidx[: c[1]].cpu().numpy(), g["aidx"])
    assert np.array_equal(y.cpu().numpy(), g["y"]), "masked GEMV y differs from the two-call y"


def check_token(gm: GpuMatrix, pools, x: torch.Tensor, params, rows=None, masked=True):
    """Run one token on both sides and compare; pools = the oracle's own (full, approx) pools.
    masked: also run the one-launch masked GEMV and require the two-call results bit for bit."""
    g = gm.token(x, params)
    xn = x.cpu().numpy()
    op = oracle_params(params)
    st, tier, fi, ai, counts = oracle.tiers(xn, op.pop("mode"), **op)
    assert st == 0 and g["status"] == 0
    assert np.array_equal(g["tier"], tier), "tier codes differ"
    assert np.array_equal(g["counts"], counts), f"counts {g['counts']} vs {counts}"
    assert np.array_equal(g["fidx"], fi) and np.array_equal(g["aidx"], ai), "lists differ"
    full_o, approx_o = pools
    y_ref = oracle.tiered_gemv(full_o, approx_o, gm.fmt, gm.d_out, gm.d_in, xn, tier, rows=rows)
    y = g["y"] if rows is None else g["y"][rows]
    rel = check_y(y, y_ref)
    if masked and gm.d_in <= spax.MASK_MAX_DIN:
        check_masked_equals_two_call(gm, x, params, g)
    return rel, g
