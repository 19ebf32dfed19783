"""Planted mistakes in the oracle (on the CPU): each plausible slip -- a dropped term, a flipped comparison, a
wrong index, a missing factor -- must make at least one pin fail.  This shows the pins constrain the oracle
rather than restating it."""

import math

import numpy as np
import pytest

import oracle
import oracle.axelram as A
import tests.test_oracle_codebook as TC
import tests.test_oracle_read as TR
import tests.test_oracle_write as TW


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(A, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def test_dropped_term_in_centroid_rule_is_caught(monkeypatch):
    def bad_lloyd(bits, tol=1e-15, max_iter=100000):
        # centroid rule with the upper pdf term dropped
        L = 1 << bits
        g = np.linspace(-2, 2, L)
        for _ in range(2000):
            t = [-math.inf] + [0.5 * (g[k - 1] + g[k]) for k in range(1, L)] + [math.inf]
            g = np.array([A._pdf(t[k]) / max(A._cell_mass(t[k], t[k + 1]), 1e-300) for k in range(L)])
        return g, 0.5 * (g[:-1] + g[1:])
    _patch(monkeypatch, "gaussian_lloyd_max", bad_lloyd)
    with pytest.raises(AssertionError):
        TC.test_optimality_conditions_by_quadrature(2)


def test_strict_comparison_is_caught(monkeypatch):
    real = A.quantize_rows

    def bad_quantize(x, signs, bits):
        idx, n, n16, u = real(x, signs, bits)
        _, t = A.codebook(np.asarray(x).shape[-1], bits)
        return np.sum(u[..., None] > t, axis=-1), n, n16, u
    _patch(monkeypatch, "quantize_rows", bad_quantize)
    with pytest.raises(AssertionError):
        TW.test_zero_vector()


def test_wrong_hadamard_order_is_caught(monkeypatch):
    real = A.hadamard

    def bad_hadamard(d):
        H = real(d).copy()
        return H[::-1]  # rows reversed: still orthogonal, no longer Sylvester order
    _patch(monkeypatch, "hadamard", bad_hadamard)
    with pytest.raises(AssertionError):
        TW.test_hadamard_matches_library(8)


def test_missing_norm_in_score_is_caught(monkeypatch):
    def bad_score(q, codes, n16, signs, bits, scale=1.0):
        q = np.asarray(q, dtype=np.float64)
        d = q.shape[-1]
        lut = A.query_lut(q, signs, bits)
        idx = A.unpack(codes, d, bits)
        return scale * lut[np.arange(d)[None, :], idx].sum(-1)
    _patch(monkeypatch, "score_lut", bad_score)
    with pytest.raises(AssertionError):
        TR.test_lut_score_equals_dequantize_then_dot(64, 2)


def test_transposed_lut_is_caught(monkeypatch):
    def bad_lut(q, signs, bits):
        q = np.asarray(q, dtype=np.float64)
        c, _ = A.codebook(q.shape[-1], bits)
        qt = A.rotate(q, signs)
        lut = qt[..., :, None] * c[None, :]
        return lut[..., ::-1, :]  # rows in the wrong coordinate order
    _patch(monkeypatch, "query_lut", bad_lut)
    with pytest.raises(AssertionError):
        TR.test_lut_score_equals_dequantize_then_dot(64, 4)


def test_wrong_gqa_mapping_is_caught(monkeypatch):
    def bad_attention(q, kcodes, kn16, signs, bits, scale, v=None, vcodes=None, vn16=None, seq_lens=None):
        q = np.asarray(q, dtype=np.float64)
        B, Hq, d = q.shape
        Hkv = kcodes.shape[1]
        out = np.zeros((B, Hq, d))
        for b in range(B):
            for h in range(Hq):
                hk = h % Hkv  # interleaved instead of contiguous groups
                vals = np.asarray(v[b, hk], dtype=np.float64)
                z = A.score_lut(q[b, h], kcodes[b, hk], kn16[b, hk], signs, bits, scale)
                out[b, h] = A._softmax_weighted_sum(z, vals)
        return out
    _patch(monkeypatch, "decode_attention", bad_attention)
    with pytest.raises(AssertionError):
        TR.test_decode_attention_matches_sdpa_on_dequantized_cache(False)


def test_sign_applied_after_transform_is_caught(monkeypatch):
    def bad_rotate(x, signs):
        x = np.asarray(x, dtype=np.float64)
        return (x @ A.hadamard(x.shape[-1]).T) * np.asarray(signs, dtype=np.float64)
    _patch(monkeypatch, "rotate", bad_rotate)
    with pytest.raises(AssertionError):
        TW.test_rotate_inverse(8)


# ---- LOOKAT oracle -------------------------------------------------------------------------------------------------

import oracle.lookat as LK  # noqa: E402
import tests.test_oracle_lookat as TL  # noqa: E402


def _patch_lk(monkeypatch, name, fn):
    monkeypatch.setattr(LK, name, fn)
    monkeypatch.setattr(oracle, name, fn)


def test_farthest_centroid_is_caught(monkeypatch):
    monkeypatch.setattr(LK, "_nearest", lambda dist: np.argmax(dist, axis=1))
    with pytest.raises(AssertionError):
        TL.test_fp32_decision_matches_fp64_nearest_except_near_ties()


def test_interleaved_subspaces_are_caught(monkeypatch):
    def bad_split(x, m):  # subspace i takes coordinates i, i + m, i + 2m, ... instead of a contiguous run
        x = np.asarray(x)
        d = x.shape[-1]
        return np.swapaxes(x.reshape(x.shape[:-1] + (d // m, m)), -1, -2)
    _patch_lk(monkeypatch, "pq_split", bad_split)
    with pytest.raises(AssertionError):
        TL.test_per_subspace_encoding_is_the_product_codebook_search()


def test_transposed_adc_table_is_caught(monkeypatch):
    real = LK.pq_table

    def bad_score(q, codes, codebooks, scale=1.0):  # the table read with the code as the row index
        tab = real(q, codebooks)
        codes = np.asarray(codes)
        m, K = tab.shape
        full = np.zeros((max(m, K), max(m, K)))
        full[:m, :K] = tab
        return scale * full.T[np.arange(m)[None, :], codes].sum(axis=-1)
    _patch_lk(monkeypatch, "pq_score", bad_score)
    with pytest.raises(AssertionError):
        TL.test_adc_score_is_the_reconstructed_dot_product(4, 16)


def test_kmeans_mean_without_division_is_caught(monkeypatch):
    def bad_kmeans(xs, init, iters):
        c = np.asarray(init, dtype=np.float32).copy()
        x64 = np.asarray(xs).astype(np.float64)
        assign = np.zeros(len(x64), dtype=np.int64)
        for _ in range(iters):
            assign = LK._nearest(LK.pq_distances_f32(xs, c))
            for k in range(c.shape[0]):
                members = x64[assign == k]
                if len(members):
                    c[k] = members.sum(axis=0).astype(np.float32)
        return c, assign
    _patch_lk(monkeypatch, "pq_kmeans", bad_kmeans)
    with pytest.raises(AssertionError):
        TL.test_kmeans_matches_scikit_learn_lloyd()


# ---- PoT oracle --------------------------------------------------------------------------------------------------------

import oracle.pot as PT  # noqa: E402
import tests.test_oracle_pot as TP  # noqa: E402


def test_log_domain_rounding_is_caught(monkeypatch):
    """Midpoints at the geometric mean of two levels (nearest in log2) instead of the arithmetic mean."""
    def bad_thresholds(E, M):
        lv = PT.pot_levels(E, M)
        return np.sqrt(lv[:-1] * lv[1:]).astype(np.float32)
    monkeypatch.setattr(PT, "pot_thresholds", bad_thresholds)
    with pytest.raises(AssertionError):
        TP.test_relative_error_of_nearest_level(3, 0, 1 / 3)


def test_dropped_sign_flip_is_caught(monkeypatch):
    real = PT.pot_score_int

    def bad_score_int(Q, codes, E, M):  # the key's sign bit ignored
        return real(Q, np.asarray(codes) & ((1 << (E + M)) - 1), E, M)
    monkeypatch.setattr(PT, "pot_score_int", bad_score_int)
    monkeypatch.setattr(oracle, "pot_score_int", bad_score_int)
    with pytest.raises(AssertionError):
        TP.test_shift_accumulate_is_the_exact_dot_product(3, 0)


def test_short_headroom_is_caught(monkeypatch):
    def bad_score_int(Q, codes, E, M):  # head-room one short: the largest level's shift is lost
        e_max = (1 << E) - 1
        codes = np.asarray(codes, dtype=np.int64)
        rank = codes & ((1 << (E + M)) - 1)
        neg = (codes >> (E + M)) & 1
        e = e_max - (rank >> M)
        mu = rank & ((1 << M) - 1)
        F = e_max + M - 1
        Qa = np.abs(np.asarray(Q, dtype=np.int64))
        mag = (Qa[None, :] << np.maximum(F - e, 0)) + mu * (Qa[None, :] << np.maximum(F - e - M, 0))
        return np.sum(np.sign(np.asarray(Q))[None, :] * np.where(neg == 1, -1, 1) * mag, axis=-1)
    monkeypatch.setattr(PT, "pot_score_int", bad_score_int)
    monkeypatch.setattr(oracle, "pot_score_int", bad_score_int)
    with pytest.raises(AssertionError):
        TP.test_shift_accumulate_is_the_exact_dot_product(3, 0)
