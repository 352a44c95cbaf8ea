"""The host restatement of the guessed TopK search in test_topk_guess_gpu.py (which branch each
GPU case takes) uses the kernel's window size and gather capacity; both must be the constants
select.cuh compiles with, or the GPU test's branch assertions would check the wrong thing."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _constexpr(src, name):
    m = re.search(r"constexpr\s+int\s+" + name + r"\s*=\s*(\d+)\s*;", src)
    assert m, name
    return int(m.group(1))


def test_host_restatement_uses_the_kernel_constants():
    pytest.importorskip("numpy")
    src = open(os.path.join(ROOT, "tiered_weight_gemv_b200", "csrc", "select.cuh")).read()
    text = open(os.path.join(ROOT, "tests", "test_topk_guess_gpu.py")).read()
    bins = int(re.search(r"^BINS = (\d+)", text, re.M).group(1))
    cand = int(re.search(r"^CAND = (\d+)", text, re.M).group(1))
    assert bins == _constexpr(src, "kGuessBins")
    assert cand == _constexpr(src, "kSelCand")
