"""GPU parity of the sign-pattern selector (axr_select_signs) against the oracle: the MSE of every candidate and the
pick (its oracle MSE must be within 1e-6 relative of the oracle minimum: candidates come in exactly tied classes
{+-s*h_r}, so indices are not compared)."""

import functools

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantized_b200 import ops
from kv_cache_quantized_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

MSE_RTOL = 1e-3
PICK_RTOL = 1e-6


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(q, k, v, cands, bits, causal=True):
    mse, best = ops.select_signs(cuda(q), cuda(k), cuda(v), cuda(cands), bits, causal=causal)
    gm, gb = mse.cpu().numpy(), int(best.cpu().numpy()[0])
    om, ob = oracle.select_signs(q, k, v, cands, bits, causal=causal)
    assert np.all(np.abs(gm - om) <= MSE_RTOL * om), np.max(np.abs(gm - om) / om)
    assert gb == int(np.argmin(gm))
    assert om[gb] <= om[ob] * (1 + PICK_RTOL), (gb, ob, om[gb], om[ob])
    return gm, om


@pytest.mark.parametrize("bits", [2, 4])
def test_exhaustive_d8(bits):
    """All 2^8 sign vectors at d=8 (the exhaustive search), two query tiles, layer-scaled keys."""
    d = 8
    q = W.normal((2, 2, 4, 100, d), 40 + bits, np.float32)
    k = W.layer_scaled_keys((2, 2, 2, 100, d), 41 + bits)
    v = W.normal((2, 2, 2, 100, d), 42 + bits, np.float16)
    gm, om = _run(q, k, v, W.all_sign_vectors(d), bits)
    # Multiplying the signs by a Walsh row only permutes the transformed coordinates, so the GPU's objective is
    # constant on the 32 classes {s * h_r} (up to fp32 summation order).  Negating s mirrors every index except
    # where a transformed coordinate is exactly zero (an exact tie on the middle threshold, which goes up on both
    # sides); fp16 keys at d=8 do produce such exact zeros, so +-s pairs are not asserted equal here.
    reps = {}
    H = _walsh(d)
    for i, s in enumerate(W.all_sign_vectors(d)):
        key = min(tuple(int(x) for x in s * H[r]) for r in range(d))
        reps.setdefault(key, []).append(gm[i])
    assert len(reps) == 32
    for vals in reps.values():
        assert np.max(vals) - np.min(vals) <= 1e-4 * np.min(vals)


def _walsh(d):
    import scipy.linalg
    return scipy.linalg.hadamard(d)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_qwen3b_shaped_reduced(bits):
    """The calibration shape (Hq=16, Hkv=2, d=128, 512 tokens, layer-wise norm heterogeneity), reduced to 2 layers,
    1 sequence and 8 candidates so the oracle finishes in seconds."""
    c = W.QWEN3B_SELECT
    inp = W.calibration_inputs(c, layers=2, seqs=1, n_cand=8)
    _run(inp["q"], inp["k"], inp["v"], inp["candidates"], bits)


def test_non_causal_d64():
    q = W.normal((1, 2, 8, 70, 64), 60, np.float32)
    k = W.layer_scaled_keys((1, 2, 2, 70, 64), 61)
    v = W.normal((1, 2, 2, 70, 64), 62, np.float16)
    _run(q, k, v, W.candidate_signs(5, 64, 63), 3, causal=False)


def test_chunking_over_candidates():
    """More candidates than one chunk (8): chunks accumulate into the right slots."""
    q = W.normal((1, 1, 4, 64, 64), 70, np.float32)
    k = W.layer_scaled_keys((1, 1, 2, 64, 64), 71)
    v = W.normal((1, 1, 2, 64, 64), 72, np.float16)
    _run(q, k, v, W.candidate_signs(19, 64, 73), 4)


def _run_per_layer(q, k, v, cands, bits, causal=True, exclude_boundary=False):
    """Per-layer selection on the GPU against the oracle.  With exclude_boundary (small d), candidates under which a
    key coordinate sits within the index criterion's 1e-6 of a threshold (parity.boundary_candidates, per layer)
    are left out of the MSE comparison and the pick is checked over the others: one index decided the other way
    there moves an MSE at d = 8 by about a percent."""
    mse, best, parts = ops.select_signs_per_layer(cuda(q), cuda(k), cuda(v), cuda(cands), bits, causal=causal,
                                                  parts=True)
    gm, gb, gp = mse.cpu().numpy(), best.cpu().numpy(), parts.cpu().numpy()
    om, ob = oracle.select_signs_per_layer(q, k, v, cands, bits, causal=causal)
    for layer in range(q.shape[0]):
        keep = ~parity.boundary_candidates(k[layer], cands, bits) if exclude_boundary else np.ones(len(cands), bool)
        assert keep.mean() > 0.5, keep.mean()
        g, o = gm[layer, keep], om[layer, keep]
        assert np.all(np.abs(g - o) <= MSE_RTOL * o), np.max(np.abs(g - o) / o)
        assert gb[layer] == int(np.argmin(gm[layer]))
        assert o[int(np.argmin(g))] <= o.min() * (1 + PICK_RTOL)
    # the per-layer MSE is the mean of its sequences' parts
    assert np.allclose(gp.mean(axis=1), gm, rtol=1e-12, atol=0)
    return gm, gb, gp


@pytest.mark.parametrize("bits", [2, 4])
def test_per_layer_exhaustive_d8_structured_keys(bits):
    """One sign vector per layer, all 2^8 candidates at d=8, keys with a per-token outlier direction of fixed
    channel signs and layer-wise norm heterogeneity: per-layer MSEs and picks against the oracle."""
    d = 8
    q = W.normal((3, 2, 4, 100, d), 80 + bits, np.float32)
    k = W.outlier_direction_keys((3, 2, 2, 100, d), 81 + bits, 7, n_out=8)
    v = W.normal((3, 2, 2, 100, d), 82 + bits, np.float16)
    _run_per_layer(q, k, v, W.all_sign_vectors(d), bits, exclude_boundary=True)


@pytest.mark.parametrize("bits", [2, 3])
def test_per_layer_qwen3b_shaped_reduced_structured(bits):
    c = W.QWEN3B_SELECT
    inp = W.calibration_inputs(c, layers=3, seqs=1, n_cand=6, keys="outlier_direction")
    gm, gb, _ = _run_per_layer(inp["q"], inp["k"], inp["v"], inp["candidates"], bits)
    # and the whole-model selector is the mean over layers
    mse, _ = ops.select_signs(cuda(inp["q"]), cuda(inp["k"]), cuda(inp["v"]), cuda(inp["candidates"]), bits)
    assert np.allclose(mse.cpu().numpy(), gm.mean(axis=0), rtol=1e-12, atol=0)


@functools.lru_cache(maxsize=1)
def _full_calibration():
    inp = W.calibration_inputs(W.QWEN3B_SELECT)
    return inp["q"], inp["k"], inp["v"], inp["candidates"]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_qwen3b_shaped_full_size(bits):
    """The full calibration set: 36 layers x 8 sequences x 512 tokens, Hq=16, Hkv=2, d=128, 200 candidates, in
    one call.  Parity on a stated subsample of the same run: the MSE of every (layer, sequence) part for 2 layers
    x 1 sequence x 8 candidates against the oracle on exactly those slices, and the subsample's pick within
    PICK_RTOL of the oracle's minimum over it; the per-layer and whole-model MSEs are the means of the parts."""
    q, k, v, cands = _full_calibration()
    qd, kd, vd, cd = cuda(q), cuda(k), cuda(v), cuda(cands)
    mse_l, best_l, parts = ops.select_signs_per_layer(qd, kd, vd, cd, bits, parts=True)
    gm, gb, gp = mse_l.cpu().numpy(), best_l.cpu().numpy(), parts.cpu().numpy()
    assert gp.shape == (36, 8, 200) and np.all(np.isfinite(gp)) and np.all(gp > 0)
    assert np.allclose(gp.mean(axis=1), gm, rtol=1e-12, atol=0)
    for layer in range(36):
        assert gb[layer] == int(np.argmin(gm[layer]))
    if bits == 4:
        mse, best = ops.select_signs(qd, kd, vd, cd, bits)
        assert np.allclose(mse.cpu().numpy(), gm.mean(axis=0), rtol=1e-12, atol=0)
        assert int(best.item()) == int(np.argmin(mse.cpu().numpy()))
    del qd, kd, vd
    sub = np.arange(0, 200, 25)  # 8 candidates
    for layer, seq in ((0, 0), (35, 7)):
        sl = slice(layer, layer + 1), slice(seq, seq + 1)
        om, ob = oracle.select_signs(q[sl], k[sl], v[sl], cands[sub], bits)
        got = gp[layer, seq, sub]
        assert np.all(np.abs(got - om) <= MSE_RTOL * om), np.max(np.abs(got - om) / om)
        assert om[int(np.argmin(got))] <= om[ob] * (1 + PICK_RTOL)
