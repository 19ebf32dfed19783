"""Pins for the oracle's sign-pattern selector (AXELRAM Key Points 4th item / Abstract: gradient-free, one-time
selection among candidate sign patterns on calibration samples).  Checked by exhaustive search over all 2^8 sign
vectors at d=8, by the tie classes the algebra forces ({+-s*h_r}: 2d members with equal objective), and by an
independent recomputation of the objective with torch's scaled_dot_product_attention."""

import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from kv_cache_quantized_b200 import workloads as W


def _calib(d, Lyr=2, S=2, N=24, Hq=4, Hkv=2, seed=31):
    q = W.normal((Lyr, S, Hq, N, d), seed, np.float32)
    k = W.layer_scaled_keys((Lyr, S, Hkv, N, d), seed + 1)
    v = W.normal((Lyr, S, Hkv, N, d), seed + 2, np.float16)
    return q, k, v


def _class_id(s):
    """Canonical representative of {+-s * h_r}: the lexicographically smallest member."""
    d = len(s)
    Hs = scipy.linalg.hadamard(d)
    members = [tuple(int(x) for x in sign * s * Hs[r]) for r in range(d) for sign in (1, -1)]
    return min(members)


@pytest.mark.parametrize("bits", [2, 4])
def test_exhaustive_d8_and_tie_classes(bits):
    d = 8
    q, k, v = _calib(d)
    cands = W.all_sign_vectors(d)
    mse, best = oracle.select_signs(q, k, v, cands, bits)
    assert best == int(np.argmin(mse)) and mse[best] == mse.min()
    # exhaustive: the pick over every sign vector is the global minimum; any subset's pick is no better
    sub = W.rng(5).choice(len(cands), size=200, replace=False)
    msub, bsub = oracle.select_signs(q, k, v, cands[sub], bits)
    assert np.allclose(msub, mse[sub], rtol=0, atol=0)
    assert msub[bsub] >= mse[best]
    # tie classes: 256 vectors -> 16 classes of 16, one objective value per class (up to fp64 rounding)
    classes = {}
    for i, s in enumerate(cands):
        classes.setdefault(_class_id(s), []).append(mse[i])
    assert len(classes) == 16 and all(len(v_) == 16 for v_ in classes.values())
    for vals in classes.values():
        vals = np.array(vals)
        assert np.max(np.abs(vals - vals[0])) <= 1e-12 * vals[0]
    # and the classes are not all tied with one another (the objective does see the sign pattern)
    reps = np.array([vals[0] for vals in classes.values()])
    assert reps.max() > reps.min() * (1 + 1e-6)


def test_objective_matches_sdpa_recomputation():
    d, bits = 64, 3
    q, k, v = _calib(d, Lyr=2, S=1, N=40, Hq=4, Hkv=2, seed=41)
    cands = W.candidate_signs(3, d, 42)
    mse, _ = oracle.select_signs(q, k, v, cands, bits)
    G = 2
    qt = torch.from_numpy(q.astype(np.float64))
    vt = torch.from_numpy(np.repeat(v.astype(np.float64), G, axis=2))
    kt = torch.from_numpy(np.repeat(k.astype(np.float64), G, axis=2))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=1 / math.sqrt(d))
    for i, s in enumerate(cands):
        codes, n16 = oracle.write(k, s, bits)
        khat = oracle.dequantize(codes, n16, s, bits, d)
        kq = torch.from_numpy(np.repeat(khat, G, axis=2))
        out = torch.nn.functional.scaled_dot_product_attention(qt, kq, vt, is_causal=True, scale=1 / math.sqrt(d))
        want = torch.mean((out - ref) ** 2).item()
        assert abs(mse[i] - want) <= 1e-10 * want


def test_objective_is_nonnegative_and_first_minimum_wins():
    d, bits = 8, 1
    q, k, v = _calib(d, seed=51)
    s = W.sign_vector(d, 52)
    cands = np.stack([s, s, -s])  # identical and mirrored candidates tie; the first one wins
    mse, best = oracle.select_signs(q, k, v, cands, bits)
    assert np.all(mse >= 0) and best == 0
    assert mse[0] == mse[1] and abs(mse[2] - mse[0]) <= 1e-12 * mse[0]


def _structured(d, Lyr=3, S=2, N=20, Hq=4, Hkv=2, seed=61, pattern_seed=7, n_out=8):
    q = W.normal((Lyr, S, Hq, N, d), seed, np.float32)
    k = W.outlier_direction_keys((Lyr, S, Hkv, N, d), seed + 1, pattern_seed, n_out=n_out)
    v = W.normal((Lyr, S, Hkv, N, d), seed + 2, np.float16)
    return q, k, v


@pytest.mark.parametrize("bits", [2, 3])
def test_per_layer_is_the_whole_model_objective_layer_by_layer(bits):
    """Per-layer selection equals the (pinned) whole-model selector run on each layer's slice alone, and the mean
    of the per-layer MSEs over layers is the whole-model MSE (equal element counts per layer)."""
    d = 64
    q, k, v = _structured(d)
    cands = W.candidate_signs(6, d, 62)
    mse_l, best_l = oracle.select_signs_per_layer(q, k, v, cands, bits)
    assert mse_l.shape == (3, 6) and best_l.shape == (3,)
    for layer in range(3):
        m1, b1 = oracle.select_signs(q[layer:layer + 1], k[layer:layer + 1], v[layer:layer + 1], cands, bits)
        assert np.array_equal(m1, mse_l[layer]) and b1 == best_l[layer]
    m_all, _ = oracle.select_signs(q, k, v, cands, bits)
    assert np.allclose(mse_l.mean(axis=0), m_all, rtol=1e-12, atol=0)


def test_per_layer_exhaustive_d8():
    """All 2^8 sign vectors at d=8, layer by layer: every layer's pick is that layer's global minimum, and the
    algebra's tie classes (16 classes of 16) hold in every layer."""
    d, bits = 8, 2
    q, k, v = _structured(d, n_out=8)
    cands = W.all_sign_vectors(d)
    mse_l, best_l = oracle.select_signs_per_layer(q, k, v, cands, bits)
    for layer in range(q.shape[0]):
        m = mse_l[layer]
        assert m[best_l[layer]] == m.min() and best_l[layer] == int(np.argmin(m))
        classes = {}
        for i, s in enumerate(cands):
            classes.setdefault(_class_id(s), []).append(m[i])
        assert len(classes) == 16
        for vals in classes.values():
            vals = np.array(vals)
            assert np.max(np.abs(vals - vals[0])) <= 1e-12 * vals[0]


def _class_ranks_agree(kind, bits, seeds):
    """Spearman correlation of the 16 class MSEs at d=8 between a calibration set and a held-out set of the same
    distribution (different noise, same outlier patterns)."""
    import scipy.stats
    d, S, N = 8, 4, 256
    cands = W.all_sign_vectors(d)
    ids = [_class_id(s) for s in cands]
    rep = [ids.index(u) for u in sorted(set(ids))]
    out = []
    for sa, sb in seeds:
        ms = []
        for sd in (sa, sb):
            q = W.normal((1, S, 4, N, d), sd, np.float32)
            v = W.normal((1, S, 2, N, d), sd + 2, np.float16)
            if kind == "iid":
                k = W.normal((1, S, 2, N, d), sd + 1, np.float16)
            else:
                k = W.outlier_direction_keys((1, S, 2, N, d), sd + 1, 7, n_out=8, layer_scale=False)
            ms.append(oracle.select_signs(q, k, v, cands[rep], bits)[0])
        out.append(scipy.stats.spearmanr(ms[0], ms[1])[0])
    return out


@pytest.mark.slow
def test_outlier_direction_keys_make_the_pick_generalise():
    """The structured calibration keys carry real sign sensitivity: the ranking of the tie classes on one
    calibration set carries over to a held-out set drawn with the same outlier patterns (rank correlation well
    above zero), while with i.i.d. keys (all classes equivalent in expectation) it does not."""
    seeds = [(100, 200), (300, 400)]
    structured = _class_ranks_agree("structured", 2, seeds)
    iid = _class_ranks_agree("iid", 2, seeds)
    assert min(structured) > 0.6, structured
    assert max(iid) < 0.4, iid
