"""CPU oracle of the three-tier decode GEMV (plain C, fp64 accumulation) behind ctypes.

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package. The product path (``tiered_weight_gemv_b200``)
never imports it, and it never imports the product: the two share no code, header, table or
helper. Inputs come from the seeded generators in ``tiered_weight_gemv_b200.synth``, which hold
none of the method's arithmetic.

Every function cites the passage it follows (see ``spax_oracle.c`` for the rules written out):
  * SpAx: Activation Sparsity with Weight Approximation for Faster LLM Decoding on Offloaded
    Weights — Abstract (three tiers by activation magnitude).
  * eigenradar commentary on SpAx — "The route outside GPU memory" (original / two-bit / unread
    tier per column; bytes moved per token).
  * TopK-Guided: Adaptive, Budget-Aware Activation Sparsity for Efficient LLM Inference —
    Abstract, §1 (threshold and TopK rules), §2.1 (guided ±δ clip), §2.2 (block budgets).

Every oracle function is pinned by the ``-m "not gpu"`` tests against brute force, closed forms,
invariants or library routines; none is "parity unpinned" except the readings listed in the
design notes (the guided three-tier split and the budget formula, pinned only by invariants).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spax_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libspax_oracle.so")
_LIB_OMP_PATH = os.path.join(_HERE, "libspax_oracle_omp.so")  # same source, OpenMP over rows

FULL_BF16 = 0
FULL_INT4 = 1
MODE_THRESHOLD = 0
MODE_TOPK = 1
MODE_GUIDED = 2
OK = 0
ERR_NONFINITE = 5


def build(force: bool = False, omp: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32 steps: no fast-math, no FMA contraction). omp=True
    builds the multi-core variant of the same source (products split over row chunks)."""
    path = _LIB_OMP_PATH if omp else _LIB_PATH
    if force or not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(_SRC):
        tmp = path + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
             "-Wall", "-Wno-unknown-pragmas"] + (["-fopenmp"] if omp else []) +
            ["-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, path)
    return path


_lib = None
_lib_omp = None
_use_omp = False


def use_openmp(on: bool = True) -> int:
    """Route the products through the OpenMP build (on) or the plain one (off); returns the
    number of threads the products then use."""
    global _use_omp
    _use_omp = bool(on)
    return int(_L().oracle_threads())


def _L():
    global _lib, _lib_omp
    if _use_omp:
        if _lib_omp is None:
            _lib_omp = _load(build(omp=True))
        return _lib_omp
    if _lib is None:
        _lib = _load(build())
    return _lib


def _load(path):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    lib.oracle_tiers.argtypes = [P, i32, i32, f32, f32, i32, i32, i32, i32, i32, P, P, P, P]
    lib.oracle_tiers.restype = i32
    lib.oracle_quant2_group.argtypes = [P, i32, P, P, P]
    lib.oracle_quant4_group.argtypes = [P, i32, P, P]
    lib.oracle_pack.argtypes = [P, i32, i32, i32, P, P]
    lib.oracle_pack.restype = i32
    lib.oracle_pack_column.argtypes = [P, i32, i32, i32, i32, P, P]
    lib.oracle_pack_column.restype = i32
    lib.oracle_full_col_bytes.argtypes = [i32, i32]
    lib.oracle_full_col_bytes.restype = i64
    lib.oracle_approx_col_bytes.argtypes = [i32]
    lib.oracle_approx_col_bytes.restype = i64
    lib.oracle_full_value.argtypes = [P, i32, i32]
    lib.oracle_full_value.restype = f64
    lib.oracle_approx_value.argtypes = [P, i32]
    lib.oracle_approx_value.restype = f64
    lib.oracle_tiered_gemv.argtypes = [P, P, i32, i32, i32, P, P, P, i32, P]
    lib.oracle_tiered_gemv.restype = i32
    lib.oracle_dense_gemv.argtypes = [P, i32, i32, P, P, i32, P]
    lib.oracle_dense_gemv.restype = i32
    lib.oracle_calibrate.argtypes = [P, i64, i32, i32, P]
    lib.oracle_calibrate.restype = i32
    lib.oracle_block_budgets.argtypes = [P, i32, f64, f64, f64, f64, P]
    lib.oracle_block_budgets.restype = i32
    lib.oracle_weight_bytes.argtypes = [i32, i32, i64, i64]
    lib.oracle_weight_bytes.restype = ctypes.c_uint64
    lib.oracle_f32_to_bf16.argtypes = [f32]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f32.restype = f32
    lib.oracle_column_norms.argtypes = [P, i32, i32, P]
    lib.oracle_column_norms.restype = i32
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = i32
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


# ----------------------------------------------------------------------------- bf16 helpers

def f32_to_bf16_bits(v: float) -> int:
    """fp32 -> bf16 bits, round to nearest even (written from the definition in C)."""
    return int(_L().oracle_f32_to_bf16(float(v)))


def bf16_bits_to_f32(h: int) -> float:
    return float(_L().oracle_bf16_to_f32(int(h)))


# ----------------------------------------------------------------------------- tier rule

def tiers(x, mode, *, t_skip=0.0, t_full=0.0, k_full=0, k_approx=0, s_skip_bp=0,
          s_below_full_bp=0, delta_bp=0):
    """Tier of every column plus ascending compacted lists (SpAx Abstract; TopK-Guided §1, §2.1).

    Returns (status, tier uint8[d], full_idx int32[n_full], approx_idx int32[n_approx],
    counts int32[4] = {n_full, n_approx, n1, n2}).
    """
    x = _c(x, np.float32)
    d = x.size
    tier = np.zeros(d, np.uint8)
    fi = np.zeros(max(d, 1), np.int32)
    ai = np.zeros(max(d, 1), np.int32)
    counts = np.zeros(4, np.int32)
    st = _L().oracle_tiers(_p(x), d, mode, t_skip, t_full, k_full, k_approx, s_skip_bp,
                           s_below_full_bp, delta_bp, _p(tier), _p(fi), _p(ai), _p(counts))
    return st, tier, fi[: counts[0]].copy(), ai[: counts[1]].copy(), counts


# ----------------------------------------------------------------------------- quantisers

def quant2_group(w_bits):
    """2-bit asymmetric quantiser of one group of bf16 values (given as uint16 bits)."""
    w = _c(w_bits, np.uint16)
    q = np.zeros(w.size, np.uint8)
    sb = np.zeros(1, np.uint16)
    mb = np.zeros(1, np.uint16)
    _L().oracle_quant2_group(_p(w), w.size, _p(q), _p(sb), _p(mb))
    return q, int(sb[0]), int(mb[0])


def quant4_group(w_bits):
    """int4 symmetric quantiser of one group of bf16 values (given as uint16 bits)."""
    w = _c(w_bits, np.uint16)
    q = np.zeros(w.size, np.int8)
    sb = np.zeros(1, np.uint16)
    _L().oracle_quant4_group(_p(w), w.size, _p(q), _p(sb))
    return q, int(sb[0])


# ----------------------------------------------------------------------------- packing

def full_col_bytes(d_out: int, fmt: int) -> int:
    return int(_L().oracle_full_col_bytes(d_out, fmt))


def approx_col_bytes(d_out: int) -> int:
    return int(_L().oracle_approx_col_bytes(d_out))


def pack(W_bits, fmt: int):
    """Pack a row-major bf16 matrix (uint16 bits [d_out, d_in]) into (full, approx) byte pools."""
    W = _c(W_bits, np.uint16)
    d_out, d_in = W.shape
    full = np.zeros(full_col_bytes(d_out, fmt) * d_in, np.uint8)
    approx = np.zeros(approx_col_bytes(d_out) * d_in, np.uint8)
    st = _L().oracle_pack(_p(W), d_out, d_in, fmt, _p(full), _p(approx))
    if st != OK:
        raise ValueError(f"oracle_pack status {st}")
    return full, approx


def pack_column(W_bits, fmt: int, j: int):
    """Pack one column j; returns its (full column bytes, approx column bytes)."""
    W = _c(W_bits, np.uint16)
    d_out, d_in = W.shape
    fc = np.zeros(full_col_bytes(d_out, fmt), np.uint8)
    ac = np.zeros(approx_col_bytes(d_out), np.uint8)
    st = _L().oracle_pack_column(_p(W), d_out, d_in, fmt, j, _p(fc), _p(ac))
    if st != OK:
        raise ValueError(f"oracle_pack_column status {st}")
    return fc, ac


def full_value(full_col, fmt: int, r: int) -> float:
    fc = _c(full_col, np.uint8)
    return float(_L().oracle_full_value(_p(fc), fmt, r))


def approx_value(approx_col, r: int) -> float:
    ac = _c(approx_col, np.uint8)
    return float(_L().oracle_approx_value(_p(ac), r))


# ----------------------------------------------------------------------------- products

def tiered_gemv(full, approx, fmt, d_out, d_in, x, tier, rows=None):
    """fp64 tiered product from the oracle's packed pools (SpAx Abstract; eigenradar)."""
    full = _c(full, np.uint8)
    approx = _c(approx, np.uint8)
    x = _c(x, np.float32)
    tier = _c(tier, np.uint8)
    if rows is None:
        y = np.zeros(d_out, np.float64)
        st = _L().oracle_tiered_gemv(_p(full), _p(approx), fmt, d_out, d_in, _p(x), _p(tier),
                                     None, 0, _p(y))
    else:
        rows = _c(rows, np.int32)
        y = np.zeros(rows.size, np.float64)
        st = _L().oracle_tiered_gemv(_p(full), _p(approx), fmt, d_out, d_in, _p(x), _p(tier),
                                     _p(rows), rows.size, _p(y))
    if st != OK:
        raise ValueError(f"oracle_tiered_gemv status {st}")
    return y


def dense_gemv(W_bits, x, rows=None):
    """fp64 dense product y = W x from the row-major bf16 matrix (uint16 bits)."""
    W = _c(W_bits, np.uint16)
    x = _c(x, np.float32)
    d_out, d_in = W.shape
    if rows is None:
        y = np.zeros(d_out, np.float64)
        _L().oracle_dense_gemv(_p(W), d_out, d_in, _p(x), None, 0, _p(y))
    else:
        rows = _c(rows, np.int32)
        y = np.zeros(rows.size, np.float64)
        _L().oracle_dense_gemv(_p(W), d_out, d_in, _p(x), _p(rows), rows.size, _p(y))
    return y


def probe_sensitivity(full, approx, fmt, d_out, d_in, X, s_probe_bp: int):
    """Output change of one matrix at the probe sparsity s = s_probe_bp / 1e4 over calibration
    tokens (TopK-Guided §2.2: block sensitivity measured at a probe sparsity). For each row x of X:
    y_ref = the tiered product with every column full, y = the product with the TopK rule
    k_full = d_in - floor(s d_in + 1/2), k_approx = 0. Returns (sum (y - y_ref)^2, sum y_ref^2)
    in fp64, both summed over tokens and rows."""
    X = np.atleast_2d(_c(X, np.float32))
    skip = (int(s_probe_bp) * d_in + 5000) // 10000
    all_full = np.full(d_in, 2, np.uint8)
    a0 = a1 = 0.0
    for x in X:
        st, tier, _, _, _ = tiers(x, MODE_TOPK, k_full=d_in - skip, k_approx=0)
        if st != OK:
            raise ValueError("non-finite calibration token")
        y = tiered_gemv(full, approx, fmt, d_out, d_in, x, tier)
        y_ref = tiered_gemv(full, approx, fmt, d_out, d_in, x, all_full)
        a0 += float(np.sum((y - y_ref) ** 2))
        a1 += float(np.sum(y_ref ** 2))
    return a0, a1


def block_sensitivity(accs):
    """A block's sensitivity from its matrices' (change, reference) sums: sqrt(sum a0 / sum a1)."""
    a0 = sum(a[0] for a in accs)
    a1 = sum(a[1] for a in accs)
    return float(np.sqrt(a0 / a1)) if a1 > 0 else 0.0


# ----------------------------------------------------------------------------- calibration etc.

def calibrate(X, s_skip_bp: int, s_below_full_bp: int):
    """Quantile thresholds of pooled |x| (TopK-Guided §2.1 calibrated threshold)."""
    X = _c(X, np.float32).ravel()
    t = np.zeros(2, np.float32)
    st = _L().oracle_calibrate(_p(X), X.size, s_skip_bp, s_below_full_bp, _p(t))
    return st, float(t[0]), float(t[1])


def block_budgets(sens, s, lam, lo=0.05, hi=0.95):
    """Sensitivity-aware block budgets (TopK-Guided §2.2), exact piecewise-linear solve."""
    sens = _c(sens, np.float64)
    out = np.zeros(sens.size, np.float64)
    st = _L().oracle_block_budgets(_p(sens), sens.size, s, lam, lo, hi, _p(out))
    if st != OK:
        raise ValueError(f"oracle_block_budgets status {st}")
    return out


def column_norms(W_bits):
    """fp32 norm of every column of the row-major bf16 W (uint16 bits), for the WINA score
    (TopK-Guided §C.1): fp64 sum of squares in row order, correctly rounded sqrt, then fp32."""
    W = _c(W_bits, np.uint16)
    d_out, d_in = W.shape
    out = np.zeros(d_in, np.float32)
    st = _L().oracle_column_norms(_p(W), d_out, d_in, _p(out))
    if st != OK:
        raise ValueError(f"oracle_column_norms status {st}")
    return out


def wina_scores(x, norms):
    """WINA score s_j = |x_j| * norm_j, one IEEE fp32 product (TopK-Guided §1, §C.1); the tier rule
    then ranks s in place of |x|."""
    x = _c(x, np.float32)
    norms = _c(norms, np.float32)
    return (np.abs(x) * norms).astype(np.float32)


def swiglu(g, u):
    """Gated-MLP activation feeding the down projection, x_j = silu(g_j) * u_j with
    silu(g) = g / (1 + e^-g), in fp64 (the Llama-2-7B block's MLP: down reads SiLU(gate x) times
    (up x)). Written from the definition; the library forms the same x in fp32."""
    g = np.asarray(g, np.float64)
    u = np.asarray(u, np.float64)
    return g / (1.0 + np.exp(-g)) * u


def greedy_allocation(params, alpha, p_target, err, p_max=1.0, step_base="mean", max_steps=100000):
    """Block-wise greedy per-matrix sparsity (TopK-Guided, Appendix D and Table 4), written out
    step by step: every matrix m has step alpha * base / f_m (base = the mean parameter count, or
    the total for step_base="sum": the pages do not say which, and Table 4 fits both); each round
    tries the next increment of every matrix that stays within p_max, keeps the one with the least
    block error err(p) (first index on a tie) and stops once the compute-weighted sparsity
    sum f_m p_m / sum f_m reaches p_target. Returns (p, order, reached)."""
    f = [float(v) for v in params]
    n = len(f)
    total = sum(f)
    base = total / n if step_base == "mean" else total
    steps = [alpha * base / fm for fm in f]
    p = [0.0] * n
    order = []
    while sum(fm * pm for fm, pm in zip(f, p)) / total < p_target - 1e-12:
        if len(order) >= max_steps:
            return np.array(p), order, False
        best, best_err = -1, 0.0
        for m in range(n):
            if p[m] + steps[m] > p_max + 1e-12:
                continue
            cand = list(p)
            cand[m] += steps[m]
            e = float(err(np.array(cand)))
            if best < 0 or e < best_err:
                best, best_err = m, e
        if best < 0:
            return np.array(p), order, False
        p[best] += steps[best]
        order.append(best)
    return np.array(p), order, True


def weight_bytes(d_out: int, fmt: int, n_full: int, n_approx: int) -> int:
    """Bytes the tiered product reads for one token (eigenradar: bytes moved per token)."""
    return int(_L().oracle_weight_bytes(d_out, fmt, n_full, n_approx))
