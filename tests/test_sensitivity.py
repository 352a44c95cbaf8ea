"""The measured block sensitivity of TopK-Guided §2.2: each block's output change when its inputs
are sparsified to a probe sparsity, the input of the sensitivity-aware block budgets.

CPU pins of the oracle (probe_sensitivity / block_sensitivity):
  * 7 times the identity (exact in bf16 and in int4, whose group scale is then exactly 1): the
    output is 7x, so the change is 49 times the squared norm of the skipped entries of x, computed
    here from an independent ranking;
  * no sparsity: the change is exactly 0; full sparsity: the change equals the output;
  * orthogonal columns: the change can only grow with the probe sparsity (nested skipped sets add
    nonnegative terms);
  * scaling x by a power of two leaves the sensitivity unchanged.
GPU: spax_probe_sensitivity against the oracle on a small stack, and exactly 0 at no sparsity.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import cuda_ok
from tiered_weight_gemv_b200 import synth


@pytest.fixture(scope="module", autouse=True)
def _built(oracle_lib):
    return oracle_lib


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 values that are exact in bf16 -> their bf16 bit patterns."""
    b = np.asarray(a, np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0)
    return (b >> 16).astype(np.uint16)


def _topk_skipped(x, skip):
    """Indices of the `skip` smallest |x|, ranked independently: |x| descending, ties by index."""
    order = sorted(range(x.size), key=lambda j: (-abs(float(x[j])), j))
    return order[x.size - skip:] if skip else []


@pytest.mark.parametrize("fmt", [0, 1])
def test_scaled_identity_closed_form(fmt):
    d = 256
    W = _bf16_bits(7.0 * np.eye(d, dtype=np.float32))
    full, approx = oracle.pack(W, fmt)
    X = synth.laplace((3, d), 41, 1).numpy()
    for s_bp in (0, 1250, 5000, 9000, 10000):
        a0, a1 = oracle.probe_sensitivity(full, approx, fmt, d, d, X, s_bp)
        skip = (s_bp * d + 5000) // 10000
        want0 = 49.0 * sum(float(np.sum(x.astype(np.float64)[_topk_skipped(x, skip)] ** 2)) for x in X)
        want1 = 49.0 * float(np.sum(X.astype(np.float64) ** 2))
        assert a1 == pytest.approx(want1, rel=1e-12)
        assert a0 == pytest.approx(want0, rel=1e-12, abs=0.0)
        if s_bp == 0:
            assert a0 == 0.0
        if s_bp == 10000:
            assert a0 == pytest.approx(a1, rel=1e-12)


def test_orthogonal_columns_change_grows_with_sparsity():
    # a signed permutation matrix: orthogonal columns, exact in bf16 and in both packings
    rng = np.random.default_rng(3)
    d = 384
    P = np.zeros((d, d), np.float32)
    P[rng.permutation(d), np.arange(d)] = rng.choice([-1.0, 1.0], d)
    full, approx = oracle.pack(_bf16_bits(P), 0)
    X = synth.laplace((4, d), 41, 2).numpy()
    prev = -1.0
    for s_bp in range(0, 10001, 1000):
        a0, a1 = oracle.probe_sensitivity(full, approx, 0, d, d, X, s_bp)
        assert a0 >= prev
        prev = a0


def test_power_of_two_scaling_leaves_sensitivity_unchanged():
    W = synth.weight(256, 128, 41, 3)
    full, approx = oracle.pack(W.view(torch.int16).numpy().view(np.uint16), 0)
    X = synth.laplace((3, 128), 41, 4).numpy()
    for s_bp in (2000, 6000):
        s1 = oracle.block_sensitivity([oracle.probe_sensitivity(full, approx, 0, 256, 128, X, s_bp)])
        s2 = oracle.block_sensitivity([oracle.probe_sensitivity(full, approx, 0, 256, 128, 4 * X, s_bp)])
        assert s1 > 0 and s1 == pytest.approx(s2, rel=1e-12)


@pytest.mark.gpu
@pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")
@pytest.mark.parametrize("fmt", [0, 1])
def test_probe_sensitivity_matches_oracle(fmt):
    from gpu_helpers import GpuMatrix, bf16_bits
    from tiered_weight_gemv_b200 import spax
    shapes = [(256, 384), (384, 256)]  # two matrices per block, three blocks
    n_tok = 8
    sig_gpu, sig_ref = {}, {}
    for s_bp in (0, 3000, 6000):
        for b in range(3):
            accs_g, accs_o = [], []
            for m, (d_out, d_in) in enumerate(shapes):
                W = synth.weight(d_out, d_in, 42, 10 * b + m, device="cuda")
                gm = GpuMatrix(W, fmt)
                X = synth.laplace((n_tok, d_in), 42, 100 + 10 * b + m, device="cuda")
                y2 = torch.empty(2 * d_out, device="cuda")
                acc = torch.zeros(2, dtype=torch.float64, device="cuda")
                st = torch.zeros(1, dtype=torch.int32, device="cuda")
                spax.spax_probe_sensitivity(gm.pm, X, s_bp, y2, acc, st, gm.ws)
                torch.cuda.synchronize()
                assert st.item() == 0
                a = acc.cpu().numpy()
                o = oracle.probe_sensitivity(*oracle.pack(bf16_bits(W), fmt), fmt, d_out, d_in,
                                             X.cpu().numpy(), s_bp)
                if s_bp == 0:
                    assert a[0] == 0.0  # the same columns in the same order: no change at all
                else:
                    assert a[0] == pytest.approx(o[0], rel=1e-4)
                assert a[1] == pytest.approx(o[1], rel=1e-5)
                accs_g.append(tuple(a))
                accs_o.append(o)
            sig_gpu[(s_bp, b)] = oracle.block_sensitivity(accs_g)
            sig_ref[(s_bp, b)] = oracle.block_sensitivity(accs_o)
    for k in sig_gpu:
        assert sig_gpu[k] == pytest.approx(sig_ref[k], rel=1e-4, abs=0.0)
    # the budgets that follow (TopK-Guided §2.2): more sensitive blocks get less sparsity
    sens = np.array([sig_gpu[(6000, b)] for b in range(3)])
    s_b = spax.spax_block_budgets(sens, 0.5, 0.5)
    assert abs(s_b.mean() - 0.5) < 1e-9
    assert np.all(np.diff(s_b[np.argsort(sens)]) <= 1e-12)
