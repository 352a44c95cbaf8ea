"""The C-ABI library without a GPU: it loads, exports exactly what include/spax.h declares, the
Python binding covers every entry point, and the host-only calls (byte accounts, block budgets,
argument validation) agree with the oracle. No call here launches a kernel.
"""
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from tiered_weight_gemv_b200 import spax

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spax.h")
LIB = os.path.join(ROOT, "tiered_weight_gemv_b200", "libspax.so")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)  # comments
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"#[^\n]*", " ", text)  # preprocessor lines (macros are not symbols)
    text = re.sub(r"typedef[^;]*;", " ", text, flags=re.S)
    return sorted(set(re.findall(r"\b(spax_[a-z0-9_]+)\s*\(", text)))


def exported_symbols():
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    return sorted({ln.split()[-1] for ln in out.splitlines() if ln.split()[-2:-1] == ["T"]})


def test_header_declares_the_entry_points():
    fns = header_functions()
    for name in ["spax_pack_weights", "spax_calibrate_thresholds", "spax_build_mask",
                 "spax_tiered_gemv", "spax_dense_gemv", "spax_workspace_bytes"]:
        assert name in fns


def test_library_exports_exactly_the_header():
    assert exported_symbols() == header_functions()


def test_binding_covers_every_entry_point():
    assert sorted(spax.EXPORTED) == header_functions()
    for name in header_functions():
        assert callable(getattr(spax._lib, name))


def test_abi_version_matches_header():
    m = re.search(r"#define\s+SPAX_ABI_VERSION\s+(\d+)", open(HEADER).read())
    assert m and spax._lib.spax_abi_version() == int(m.group(1))


def test_status_strings_are_distinct():
    codes = [spax.OK, spax.ERR_ARG, spax.ERR_SHAPE, spax.ERR_WORKSPACE, spax.ERR_CUDA,
             spax.ERR_NONFINITE, spax.ERR_TIMEOUT, spax.ERR_INDEX]
    strings = [spax.status_string(c) for c in codes]
    assert len(set(strings)) == len(codes) and all(strings)
    assert spax.status_string(999)  # unknown codes still give a string


@pytest.mark.parametrize("fmt", [spax.FULL_BF16, spax.FULL_INT4_G128])
@pytest.mark.parametrize("d_out,d_in", [(128, 1), (640, 33), (4096, 4096), (22016, 4096),
                                        (8192, 28672)])
def test_pack_bytes_match_the_oracle_layout(fmt, d_out, d_in):
    fb, ab = spax.spax_pack_bytes(d_out, d_in, fmt)
    assert fb == d_in * oracle.full_col_bytes(d_out, fmt)
    assert ab == d_in * oracle.approx_col_bytes(d_out)


def test_pack_bytes_reject_bad_shapes():
    for d_out, d_in, fmt in [(100, 4, 0), (0, 4, 0), (128, 0, 0), (128, 4, 7)]:
        with pytest.raises(spax.SpaxError):
            spax.spax_pack_bytes(d_out, d_in, fmt)


def test_weight_bytes_match_the_oracle_account():
    rng = np.random.default_rng(3)
    for _ in range(200):
        d_out = 128 * int(rng.integers(1, 300))
        fmt = int(rng.integers(0, 2))
        nf, na = (int(v) for v in rng.integers(0, 40000, 2))
        assert spax.spax_weight_bytes(d_out, fmt, nf, na) == oracle.weight_bytes(d_out, fmt, nf, na)


def test_weight_bytes_closed_form():
    # bf16 full columns 2 B per row; 2-bit columns 1/4 B per row plus a 4-byte (scale, min)
    # record per 128 rows; int4 full columns 1/2 B per row plus a 2-byte scale per 128 rows
    d_out = 4096
    assert spax.spax_weight_bytes(d_out, spax.FULL_BF16, 1, 0) == 2 * d_out
    assert spax.spax_weight_bytes(d_out, spax.FULL_BF16, 0, 1) == d_out // 4 + 4 * d_out // 128
    assert spax.spax_weight_bytes(d_out, spax.FULL_INT4_G128, 1, 0) == d_out // 2 + 2 * d_out // 128
    assert spax.spax_weight_bytes(d_out, spax.FULL_BF16, 0, 0) == 0


def test_block_budgets_match_the_oracle():
    rng = np.random.default_rng(7)
    b = np.arange(32)
    cases = [(1 + 3 * np.exp(-b / 4), s, 0.5) for s in (0.3, 0.5, 0.7)]
    cases += [(rng.uniform(0.1, 10, int(rng.integers(1, 64))), float(rng.uniform(0.05, 0.95)),
               float(rng.uniform(0, 3))) for _ in range(40)]
    for sens, s, lam in cases:
        got = spax.spax_block_budgets(sens, s, lam)
        ref = np.asarray(oracle.block_budgets(sens, s, lam), np.float64)
        assert np.max(np.abs(got - ref)) <= 1e-12, (s, lam)
        assert abs(got.mean() - s) <= 1e-9
        assert got.min() >= 0.05 - 1e-15 and got.max() <= 0.95 + 1e-15


def test_block_budgets_reject_bad_arguments():
    sens = np.ones(4)
    for s, lam, lo, hi in [(0.5, -1.0, 0.05, 0.95), (0.01, 0.5, 0.05, 0.95),
                           (0.5, 0.5, 0.6, 0.95), (0.5, 0.5, 0.05, 1.5)]:
        with pytest.raises(spax.SpaxError):
            spax.spax_block_budgets(sens, s, lam, lo, hi)
    with pytest.raises(spax.SpaxError):
        spax.spax_block_budgets(np.array([1.0, -1.0]), 0.5, 0.5)


def test_device_calls_validate_arguments_before_any_launch():
    # these fail the host-side checks, so they return before touching CUDA (no GPU here)
    L = spax._lib
    prm = spax.mask_params(spax.MASK_TOPK, k_full=1, k_approx=1)
    assert L.spax_build_mask(None, 16, prm, None, None, None, None, None, None) == spax.ERR_ARG
    dummy = 256  # a non-null, 256-byte aligned address that is never dereferenced
    bad_k = spax.mask_params(spax.MASK_TOPK, k_full=10, k_approx=10)
    assert L.spax_build_mask(dummy, 16, bad_k, dummy, dummy, dummy, dummy, dummy, None) == spax.ERR_ARG
    assert L.spax_build_mask(dummy, spax.MASK_MAX_DIN + 1, prm, dummy, dummy, dummy, dummy, dummy,
                             None) == spax.ERR_SHAPE
    bad_t = spax.mask_params(spax.MASK_THRESHOLD, t_skip=1.0, t_full=0.5)
    assert L.spax_build_mask(dummy, 16, bad_t, dummy, dummy, dummy, dummy, dummy, None) == spax.ERR_ARG
    bad_scaled = spax.mask_params(spax.MASK_TOPK_SCALED, k_full=10, k_approx=10, t_full=1.2)
    assert L.spax_build_mask(dummy, 16, bad_scaled, dummy, dummy, dummy, dummy, dummy,
                             None) == spax.ERR_ARG
    unknown = spax.mask_params(4, k_full=1, k_approx=1)  # no such rule
    assert L.spax_build_mask(dummy, 16, unknown, dummy, dummy, dummy, dummy, dummy, None) == spax.ERR_ARG
    # the fp64 accumulator of the sensitivity calls must be 8-byte aligned
    assert L.spax_output_change(dummy, dummy, 16, dummy + 4, None) == spax.ERR_ARG
    assert L.spax_output_change(dummy, dummy, 0, dummy, None) == spax.ERR_SHAPE
    assert L.spax_tiered_gemv(None, dummy, dummy, dummy, dummy, dummy, dummy, dummy, 1 << 20,
                              None) == spax.ERR_ARG
    desc = spax.spax_packed(100, 16, spax.FULL_BF16, 0, dummy, dummy)  # d_out % 128 != 0
    import ctypes
    assert L.spax_tiered_gemv(ctypes.byref(desc), dummy, dummy, dummy, dummy, dummy, dummy, dummy,
                              1 << 20, None) == spax.ERR_SHAPE
    assert L.spax_tiered_gemv_fixed_scratch(ctypes.byref(desc), dummy, dummy, dummy, dummy, dummy,
                                            dummy, None) == spax.ERR_SHAPE
    assert L.spax_dense_gemv(dummy, dummy, dummy, 100, 16, dummy, dummy, 1 << 20, None) == spax.ERR_SHAPE
    assert L.spax_pack_weights(None, 128, 16, spax.FULL_BF16, dummy, dummy, None) == spax.ERR_ARG
    assert L.spax_calibrate_thresholds(dummy, 4, 16, 12000, 3000, dummy, dummy, dummy, 1 << 20,
                                       None) == spax.ERR_ARG  # a target above 100%
    assert L.spax_calibrate_thresholds(dummy, 4, 16, 3000, 6000, dummy, dummy, None, 1 << 20,
                                       None) == spax.ERR_WORKSPACE


def test_plan_for_an_sm_count_and_the_fixed_scratch_bound():
    """spax_gemv_plan_sms (no CUDA call) gives the plans the calls make. On 148 SMs no tiered plan
    needs more than the fixed scratch array (4 MiB): a plan with splits stays within
    148 x 2048 x 8 bytes. On a hypothetical 1184-SM part the same rule asks for more for some
    shapes, which is exactly the condition under which spax_tiered_gemv_fixed_scratch returns
    SPAX_ERR_WORKSPACE."""
    fixed = spax.spax_fixed_scratch_bytes()
    assert fixed == 4 << 20
    worst = 0
    for d_out in list(range(128, 40000, 128)) + [57344, 1 << 20]:
        S, R, ws = spax.spax_gemv_plan_sms(spax.OP_TIERED_GEMV, d_out, 4096, spax.FULL_BF16, 148)
        T = -(-d_out // R)
        assert R in (512, 1024, 2048) and S >= 1
        if S > 1:
            assert T * S <= 148  # one wave
            assert ws >= S * d_out * 8 and ws <= 148 * 2048 * 8 + 255
        worst = max(worst, ws)
    assert worst <= fixed
    S, R, ws = spax.spax_gemv_plan_sms(spax.OP_TIERED_GEMV, 8192, 8192, spax.FULL_BF16, 1184)
    assert S * (-(-8192 // R)) <= 1184 and ws > fixed  # the case the fixed-scratch call rejects
    # the block's plans on B200 (the tiered rule and the dense rule differ)
    assert spax.spax_gemv_plan_sms(spax.OP_TIERED_GEMV, 12288, 4096, 0, 148)[:2] == (6, 512)
    assert spax.spax_gemv_plan_sms(spax.OP_TIERED_GEMV, 22016, 4096, 0, 148)[:2] == (3, 512)
    assert spax.spax_gemv_plan_sms(spax.OP_DENSE_GEMV, 22016, 4096, 0, 148)[:2] == (13, 2048)
    with pytest.raises(spax.SpaxError):
        spax.spax_gemv_plan_sms(spax.OP_TIERED_GEMV, 100, 4096, 0, 148)  # d_out % 128 != 0
    with pytest.raises(spax.SpaxError):
        spax.spax_gemv_plan_sms(spax.OP_TIERED_GEMV, 4096, 4096, 0, 0)
