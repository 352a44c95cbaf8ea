"""Python binding of libspax.so: argument marshalling only, every step runs in the CUDA library.

The functions carry the names of the C entry points in ``include/spax.h`` and take torch tensors
(device memory and the current CUDA stream come from PyTorch). They raise ``SpaxError`` on a
non-OK status. Importing this module fails loudly when ``libspax.so`` is missing: there is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspax.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libspax.so not found at {_LIB_PATH}; build it with "
        "`python -m tiered_weight_gemv_b200.build` (nvcc, sm_100a)")
_lib = ctypes.CDLL(_LIB_PATH)

OK = 0
ERR_ARG, ERR_SHAPE, ERR_WORKSPACE, ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT, ERR_INDEX = 1, 2, 3, 4, 5, 6, 7
FULL_BF16, FULL_INT4_G128 = 0, 1
MASK_THRESHOLD, MASK_TOPK, MASK_GUIDED, MASK_TOPK_SCALED = 0, 1, 2, 3
OP_TIERED_GEMV, OP_DENSE_GEMV, OP_CALIBRATE = 0, 1, 2
MASK_MAX_DIN = 32768


class SpaxError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {status_string(status)} (status {status})")
        self.status = status


class spax_mask_params(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("t_skip", ctypes.c_float), ("t_full", ctypes.c_float),
                ("k_full", ctypes.c_int32), ("k_approx", ctypes.c_int32),
                ("s_skip_bp", ctypes.c_int32), ("s_below_full_bp", ctypes.c_int32),
                ("delta_bp", ctypes.c_int32)]


class spax_packed(ctypes.Structure):
    _fields_ = [("d_out", ctypes.c_int32), ("d_in", ctypes.c_int32), ("full_fmt", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("d_full", ctypes.c_void_p),
                ("d_approx", ctypes.c_void_p)]


_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "spax_abi_version": ([], _I),
    "spax_status_string": ([_I], ctypes.c_char_p),
    "spax_pack_bytes": ([_I, _I, _I, _P, _P], _Z),
    "spax_pack_weights": ([_P, _I, _I, _I, _P, _P, _P], _I),
    "spax_calibrate_thresholds": ([_P, _I, _I, _I, _I, _P, _P, _P, _Z, _P], _I),
    "spax_build_mask": ([_P, _I, ctypes.POINTER(spax_mask_params), _P, _P, _P, _P, _P, _P], _I),
    "spax_tiered_gemv": ([ctypes.POINTER(spax_packed), _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "spax_dense_gemv": ([_P, _P, _P, _I, _I, _P, _P, _Z, _P], _I),
    "spax_masked_gemv": ([ctypes.POINTER(spax_packed), _P, ctypes.POINTER(spax_mask_params), _P,
                          _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "spax_masked_gemv_wina": ([ctypes.POINTER(spax_packed), _P, _P,
                               ctypes.POINTER(spax_mask_params), _P, _P, _P, _P, _P, _P, _P, _Z,
                               _P], _I),
    "spax_column_norms": ([_P, _I, _I, _P, _P], _I),
    "spax_masked_gemv_swiglu": ([ctypes.POINTER(spax_packed), _P, ctypes.POINTER(spax_mask_params),
                                 _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P], _I),
    "spax_tiered_gemv_fixed_scratch": ([ctypes.POINTER(spax_packed), _P, _P, _P, _P, _P, _P, _P],
                                       _I),
    "spax_fixed_scratch_bytes": ([], _Z),
    "spax_fixed_scratch_reset": ([_P], _I),
    "spax_output_change": ([_P, _P, _I, _P, _P], _I),
    "spax_probe_sensitivity": ([ctypes.POINTER(spax_packed), _P, _I, _I, _P, _P, _P, _P, _Z, _P],
                               _I),
    "spax_test_tiered_gemv_timeout": ([ctypes.POINTER(spax_packed), _P, _P, _P, _P, _P, _P, _P, _Z,
                                      ctypes.c_uint64, _P], _I),
    "spax_workspace_bytes": ([_I, _I, _I], _Z),
    "spax_gemv_plan": ([_I, _I, _I, _I, _P, _P], _I),
    "spax_gemv_plan_sms": ([_I, _I, _I, _I, _I, _P, _P, _P], _I),
    "spax_block_budgets": ([_P, _I, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                            ctypes.c_double, _P], _I),
    "spax_weight_bytes": ([_I, _I, ctypes.c_int64, ctypes.c_int64], ctypes.c_uint64),
    "spax_greedy_allocation": ([_P, _I, ctypes.c_double, ctypes.c_double, ctypes.c_double, _P, _P,
                                _I, _P, _P, _P], _I),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


def status_string(status: int) -> str:
    return _lib.spax_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != OK:
        raise SpaxError(fn, status)


def _dev(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dev_or_pinned(t, name="tensor"):
    """A weight pool: device memory, or page-locked host memory (mapped into the device)."""
    if isinstance(t, torch.Tensor) and not t.is_cuda and t.is_pinned() and t.is_contiguous():
        return ctypes.c_void_p(t.data_ptr())
    return _dev(t, None, name)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------------------ host-only calls

def spax_abi_version() -> int:
    return int(_lib.spax_abi_version())


def spax_pack_bytes(d_out: int, d_in: int, full_fmt: int):
    fb, ab = ctypes.c_size_t(0), ctypes.c_size_t(0)
    tot = _lib.spax_pack_bytes(d_out, d_in, full_fmt, ctypes.byref(fb), ctypes.byref(ab))
    if tot == 0:
        raise SpaxError("spax_pack_bytes", ERR_SHAPE)
    return int(fb.value), int(ab.value)


def spax_workspace_bytes(op: int, d_out: int, d_in: int) -> int:
    return int(_lib.spax_workspace_bytes(op, d_out, d_in))


def spax_gemv_plan(op: int, d_out: int, d_in: int, full_fmt: int = FULL_BF16):
    s, r = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("spax_gemv_plan", _lib.spax_gemv_plan(op, d_out, d_in, full_fmt, ctypes.byref(s),
                                                 ctypes.byref(r)))
    return int(s.value), int(r.value)


def spax_gemv_plan_sms(op: int, d_out: int, d_in: int, full_fmt: int, sm_count: int):
    """Host-only: (splits, row_tile, workspace bytes) of op's plan on a GPU with sm_count SMs."""
    sp, r, w = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_size_t(0)
    _check("spax_gemv_plan_sms", _lib.spax_gemv_plan_sms(op, d_out, d_in, full_fmt, sm_count,
                                                         ctypes.byref(sp), ctypes.byref(r),
                                                         ctypes.byref(w)))
    return int(sp.value), int(r.value), int(w.value)


def spax_block_budgets(sens, s: float, lam: float, lo: float = 0.05, hi: float = 0.95):
    sens = np.ascontiguousarray(sens, dtype=np.float64)
    out = np.zeros_like(sens)
    _check("spax_block_budgets", _lib.spax_block_budgets(
        sens.ctypes.data_as(_P), sens.size, s, lam, lo, hi, out.ctypes.data_as(_P)))
    return out


BLOCK_ERROR_FN = ctypes.CFUNCTYPE(ctypes.c_double, ctypes.POINTER(ctypes.c_double), ctypes.c_int,
                                  ctypes.c_void_p)


def spax_greedy_allocation(params, alpha: float, p_target: float, err, p_max: float = 1.0,
                           max_steps: int = 100000):
    """Per-matrix sparsities of one block (the library's greedy allocation). err(p) -> block
    error for a numpy array of per-matrix sparsities. Returns (p, order)."""
    f = np.ascontiguousarray(params, dtype=np.float64)
    n = f.size
    cb = BLOCK_ERROR_FN(lambda pp, nn, ctx: float(err(np.ctypeslib.as_array(pp, (nn,)).copy())))
    p = np.zeros(n, np.float64)
    order = np.zeros(max(1, max_steps), np.int32)
    steps = ctypes.c_int32(0)
    _check("spax_greedy_allocation", _lib.spax_greedy_allocation(
        f.ctypes.data_as(_P), n, alpha, p_target, p_max, ctypes.cast(cb, _P), None, max_steps,
        p.ctypes.data_as(_P), order.ctypes.data_as(_P), ctypes.byref(steps)))
    return p, order[: steps.value].copy()


def spax_weight_bytes(d_out: int, full_fmt: int, n_full: int, n_approx: int) -> int:
    return int(_lib.spax_weight_bytes(d_out, full_fmt, int(n_full), int(n_approx)))


# ------------------------------------------------------------------------------ device calls

@dataclass
class PackedMatrix:
    """Both pools of a packed d_out x d_in matrix (device uint8 tensors) and its C descriptor."""
    d_out: int
    d_in: int
    full_fmt: int
    full: torch.Tensor
    approx: torch.Tensor

    def desc(self) -> spax_packed:
        return spax_packed(self.d_out, self.d_in, self.full_fmt, 0, self.full.data_ptr(),
                           self.approx.data_ptr())


def alloc_packed(d_out: int, d_in: int, full_fmt: int, device="cuda") -> PackedMatrix:
    fb, ab = spax_pack_bytes(d_out, d_in, full_fmt)
    return PackedMatrix(d_out, d_in, full_fmt,
                        torch.empty(fb, dtype=torch.uint8, device=device),
                        torch.empty(ab, dtype=torch.uint8, device=device))


def packed_to_host(pm: PackedMatrix) -> PackedMatrix:
    """A copy of a packed matrix in page-locked host memory. Unified addressing maps such memory
    into the device address space, so the GEMV kernels read the pools straight over the host
    link (the offloaded-weights setting); the descriptor's pointers are the host pointers."""
    full = torch.empty(pm.full.numel(), dtype=torch.uint8, pin_memory=True)
    approx = torch.empty(pm.approx.numel(), dtype=torch.uint8, pin_memory=True)
    full.copy_(pm.full)
    approx.copy_(pm.approx)
    return PackedMatrix(pm.d_out, pm.d_in, pm.full_fmt, full, approx)


def spax_pack_weights(W: torch.Tensor, full_fmt: int, dst: PackedMatrix, stream=None) -> None:
    d_out, d_in = W.shape
    if (dst.d_out, dst.d_in, dst.full_fmt) != (d_out, d_in, full_fmt):
        raise ValueError("destination descriptor does not match W")
    fb, ab = spax_pack_bytes(d_out, d_in, full_fmt)
    if dst.full.numel() < fb or dst.approx.numel() < ab:
        raise ValueError("destination pools too small")
    _check("spax_pack_weights", _lib.spax_pack_weights(
        _dev(W, torch.bfloat16, "W"), d_out, d_in, full_fmt, _dev(dst.full, torch.uint8, "full"),
        _dev(dst.approx, torch.uint8, "approx"), _stream(stream)))


def spax_calibrate_thresholds(calib_x: torch.Tensor, s_skip_bp: int, s_below_full_bp: int,
                              t_out: torch.Tensor, status: torch.Tensor, ws: torch.Tensor,
                              stream=None) -> None:
    n_tok, d_in = calib_x.shape
    _check("spax_calibrate_thresholds", _lib.spax_calibrate_thresholds(
        _dev(calib_x, torch.float32, "calib_x"), n_tok, d_in, s_skip_bp, s_below_full_bp,
        _dev(t_out, torch.float32, "t_out"), _dev(status, torch.int32, "status"),
        _dev(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)))


def mask_params(mode: int, *, t_skip=0.0, t_full=0.0, k_full=0, k_approx=0, s_skip_bp=0,
                s_below_full_bp=0, delta_bp=0) -> spax_mask_params:
    """The rule's parameters (spax.h, spax_mask_params). In MASK_TOPK mode t_full / t_skip may
    carry a guess of the |x| at rank k_full / k_full + k_approx (calibrated quantiles); it only
    speeds the selection up when it holds, and 0 means no guess. MASK_TOPK_SCALED is the same
    rule with the guesses given as multiples of the token's mean |x|."""
    return spax_mask_params(mode, t_skip, t_full, k_full, k_approx, s_skip_bp, s_below_full_bp,
                            delta_bp)


def spax_build_mask(x: torch.Tensor, params: spax_mask_params, tier: torch.Tensor,
                    full_idx: torch.Tensor, approx_idx: torch.Tensor, counts: torch.Tensor,
                    status: torch.Tensor, stream=None) -> None:
    d_in = x.numel()
    for t, n in ((tier, d_in), (full_idx, d_in), (approx_idx, d_in), (counts, 4)):
        if t.numel() < n:
            raise ValueError("mask output too small")
    _check("spax_build_mask", _lib.spax_build_mask(
        _dev(x, torch.float32, "x"), d_in, ctypes.byref(params), _dev(tier, torch.uint8, "tier"),
        _dev(full_idx, torch.int32, "full_idx"), _dev(approx_idx, torch.int32, "approx_idx"),
        _dev(counts, torch.int32, "counts"), _dev(status, torch.int32, "status"),
        _stream(stream)))


def spax_tiered_gemv(W: PackedMatrix, x: torch.Tensor, full_idx: torch.Tensor,
                     approx_idx: torch.Tensor, counts: torch.Tensor, y: torch.Tensor,
                     status: torch.Tensor, ws: torch.Tensor, stream=None, desc=None) -> None:
    if x.numel() != W.d_in or y.numel() != W.d_out:
        raise ValueError("x / y sizes do not match W")
    d = W.desc() if desc is None else desc
    _check("spax_tiered_gemv", _lib.spax_tiered_gemv(
        ctypes.byref(d), _dev(x, torch.float32, "x"), _dev(full_idx, torch.int32, "full_idx"),
        _dev(approx_idx, torch.int32, "approx_idx"), _dev(counts, torch.int32, "counts"),
        _dev(y, torch.float32, "y"), _dev(status, torch.int32, "status"), _dev(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))


def spax_masked_gemv(W: PackedMatrix, x: torch.Tensor, params: spax_mask_params, y: torch.Tensor,
                     status: torch.Tensor, ws: torch.Tensor, tier=None, full_idx=None,
                     approx_idx=None, counts=None, stream=None, desc=None) -> None:
    """The mask and the tiered GEMV in one launch; tier / lists / counts are optional outputs."""
    if x.numel() != W.d_in or y.numel() != W.d_out:
        raise ValueError("x / y sizes do not match W")
    for t, n in ((tier, W.d_in), (full_idx, W.d_in), (approx_idx, W.d_in), (counts, 4)):
        if t is not None and t.numel() < n:
            raise ValueError("mask output too small")
    d = W.desc() if desc is None else desc
    _check("spax_masked_gemv", _lib.spax_masked_gemv(
        ctypes.byref(d), _dev(x, torch.float32, "x"), ctypes.byref(params),
        _dev(y, torch.float32, "y"), _dev(tier, torch.uint8, "tier"),
        _dev(full_idx, torch.int32, "full_idx"), _dev(approx_idx, torch.int32, "approx_idx"),
        _dev(counts, torch.int32, "counts"), _dev(status, torch.int32, "status"),
        _dev(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)))


def spax_column_norms(W: torch.Tensor, norms: torch.Tensor, stream=None) -> None:
    """Per-column Euclidean norms of the row-major bf16 W (for the WINA score)."""
    d_out, d_in = W.shape
    if norms.numel() < d_in:
        raise ValueError("norms too small")
    _check("spax_column_norms", _lib.spax_column_norms(
        _dev(W, torch.bfloat16, "W"), d_out, d_in, _dev(norms, torch.float32, "norms"),
        _stream(stream)))


def spax_masked_gemv_wina(W: PackedMatrix, x: torch.Tensor, norms: torch.Tensor,
                          params: spax_mask_params, y: torch.Tensor, status: torch.Tensor,
                          ws: torch.Tensor, tier=None, full_idx=None, approx_idx=None, counts=None,
                          stream=None, desc=None) -> None:
    """spax_masked_gemv ranking columns by the WINA score |x_j| * norms[j]."""
    if x.numel() != W.d_in or norms.numel() != W.d_in or y.numel() != W.d_out:
        raise ValueError("x / norms / y sizes do not match W")
    for t, n in ((tier, W.d_in), (full_idx, W.d_in), (approx_idx, W.d_in), (counts, 4)):
        if t is not None and t.numel() < n:
            raise ValueError("mask output too small")
    d = W.desc() if desc is None else desc
    _check("spax_masked_gemv_wina", _lib.spax_masked_gemv_wina(
        ctypes.byref(d), _dev(x, torch.float32, "x"), _dev(norms, torch.float32, "norms"),
        ctypes.byref(params), _dev(y, torch.float32, "y"), _dev(tier, torch.uint8, "tier"),
        _dev(full_idx, torch.int32, "full_idx"), _dev(approx_idx, torch.int32, "approx_idx"),
        _dev(counts, torch.int32, "counts"), _dev(status, torch.int32, "status"),
        _dev(ws, None, "ws"), ws.numel() * ws.element_size(), _stream(stream)))


def spax_masked_gemv_swiglu(W: PackedMatrix, gu: torch.Tensor, params: spax_mask_params,
                            y: torch.Tensor, status: torch.Tensor, ws: torch.Tensor, x_out=None,
                            tier=None, full_idx=None, approx_idx=None, counts=None, stream=None,
                            desc=None) -> None:
    """spax_masked_gemv on x = silu(g) * u formed in the kernel from gu = [g; u] (2 * d_in)."""
    if gu.numel() != 2 * W.d_in or y.numel() != W.d_out:
        raise ValueError("gu / y sizes do not match W")
    for t, n in ((x_out, W.d_in), (tier, W.d_in), (full_idx, W.d_in), (approx_idx, W.d_in),
                 (counts, 4)):
        if t is not None and t.numel() < n:
            raise ValueError("output too small")
    d = W.desc() if desc is None else desc
    _check("spax_masked_gemv_swiglu", _lib.spax_masked_gemv_swiglu(
        ctypes.byref(d), _dev(gu, torch.float32, "gu"), ctypes.byref(params),
        _dev(y, torch.float32, "y"), _dev(x_out, torch.float32, "x_out"),
        _dev(tier, torch.uint8, "tier"), _dev(full_idx, torch.int32, "full_idx"),
        _dev(approx_idx, torch.int32, "approx_idx"), _dev(counts, torch.int32, "counts"),
        _dev(status, torch.int32, "status"), _dev(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))


def spax_tiered_gemv_fixed_scratch(W: PackedMatrix, x: torch.Tensor, full_idx: torch.Tensor,
                                   approx_idx: torch.Tensor, counts: torch.Tensor, y: torch.Tensor,
                                   status: torch.Tensor, stream=None, desc=None) -> None:
    """spax_tiered_gemv without a workspace argument: the library's own per-device scratch array
    is used, so nothing is allocated. Calls on one device must not overlap."""
    if x.numel() != W.d_in or y.numel() != W.d_out:
        raise ValueError("x / y sizes do not match W")
    d = W.desc() if desc is None else desc
    _check("spax_tiered_gemv_fixed_scratch", _lib.spax_tiered_gemv_fixed_scratch(
        ctypes.byref(d), _dev(x, torch.float32, "x"), _dev(full_idx, torch.int32, "full_idx"),
        _dev(approx_idx, torch.int32, "approx_idx"), _dev(counts, torch.int32, "counts"),
        _dev(y, torch.float32, "y"), _dev(status, torch.int32, "status"), _stream(stream)))


def spax_fixed_scratch_bytes() -> int:
    return int(_lib.spax_fixed_scratch_bytes())


def spax_fixed_scratch_reset(stream=None) -> None:
    """Zero the current device's fixed scratch array (after a fixed-scratch call reported a
    device error such as ERR_TIMEOUT)."""
    _check("spax_fixed_scratch_reset", _lib.spax_fixed_scratch_reset(_stream(stream)))


def spax_test_tiered_gemv_timeout(W: PackedMatrix, x: torch.Tensor, full_idx: torch.Tensor,
                                  approx_idx: torch.Tensor, counts: torch.Tensor, y: torch.Tensor,
                                  status: torch.Tensor, ws=None, wait_limit_ns: int = 20_000_000,
                                  stream=None) -> None:
    """Failure-detection test hook: the list-driven GEMV with the last split of every row tile
    left out, so its waits run out after wait_limit_ns and status becomes ERR_TIMEOUT. ws None
    selects the fixed scratch array."""
    d = W.desc()
    _check("spax_test_tiered_gemv_timeout", _lib.spax_test_tiered_gemv_timeout(
        ctypes.byref(d), _dev(x, torch.float32, "x"), _dev(full_idx, torch.int32, "full_idx"),
        _dev(approx_idx, torch.int32, "approx_idx"), _dev(counts, torch.int32, "counts"),
        _dev(y, torch.float32, "y"), _dev(status, torch.int32, "status"),
        None if ws is None else _dev(ws, None, "ws"),
        0 if ws is None else ws.numel() * ws.element_size(), int(wait_limit_ns),
        _stream(stream)))


def spax_output_change(y: torch.Tensor, y_ref: torch.Tensor, acc: torch.Tensor,
                       stream=None) -> None:
    """acc[0] += sum (y - y_ref)^2, acc[1] += sum y_ref^2 (fp64 device accumulators)."""
    if y.numel() != y_ref.numel() or acc.numel() < 2:
        raise ValueError("sizes do not match")
    _check("spax_output_change", _lib.spax_output_change(
        _dev(y, torch.float32, "y"), _dev(y_ref, torch.float32, "y_ref"), y.numel(),
        _dev(acc, torch.float64, "acc"), _stream(stream)))


def spax_probe_sensitivity(W: PackedMatrix, X: torch.Tensor, s_probe_bp: int, y2: torch.Tensor,
                           acc: torch.Tensor, status: torch.Tensor, ws: torch.Tensor, stream=None,
                           desc=None) -> None:
    """Output change of one matrix at probe sparsity s_probe_bp / 1e4 over the calibration
    tokens X [n_tok, d_in], accumulated into acc (two fp64 on the device)."""
    n_tok, d_in = X.shape
    if d_in != W.d_in or y2.numel() < 2 * W.d_out or acc.numel() < 2:
        raise ValueError("sizes do not match W")
    d = W.desc() if desc is None else desc
    _check("spax_probe_sensitivity", _lib.spax_probe_sensitivity(
        ctypes.byref(d), _dev(X, torch.float32, "X"), n_tok, s_probe_bp,
        _dev(y2, torch.float32, "y2"), _dev(acc, torch.float64, "acc"),
        _dev(status, torch.int32, "status"), _dev(ws, None, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)))


def spax_dense_gemv(Wt: torch.Tensor, x: torch.Tensor, y: torch.Tensor, d_out: int, d_in: int,
                    status: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    if x.numel() != d_in or y.numel() != d_out or Wt.numel() * Wt.element_size() < 2 * d_in * d_out:
        raise ValueError("sizes do not match")
    _check("spax_dense_gemv", _lib.spax_dense_gemv(
        _dev_or_pinned(Wt, "Wt"), _dev(x, torch.float32, "x"), _dev(y, torch.float32, "y"), d_out,
        d_in, _dev(status, torch.int32, "status"), _dev(ws, None, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)))


def alloc_workspace(op: int, d_out: int, d_in: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace (the GEMV's flagged partial sums must start at zero)."""
    n = spax_workspace_bytes(op, d_out, d_in)
    if n == 0:
        raise SpaxError("spax_workspace_bytes", ERR_SHAPE)
    return torch.zeros(n, dtype=torch.uint8, device=device)
