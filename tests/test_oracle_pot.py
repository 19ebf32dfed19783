"""Pins for the PoT shift-accumulate oracle (the arxivdaily page of the shift-accumulate attention paper): level
decisions against a brute-force nearest level, the relative-error bound of nearest power-of-two rounding, the
shift-accumulated integer against a plain fp64 dot product of the same dyadic numbers, the real score against the
dequantized dot product, the integer-log2 online softmax against its two-pass definition, and two of the page's own
findings on synthetic Gaussian keys: more exponent bits buy nothing, one mantissa bit about halves the score error."""

import math

import numpy as np
import pytest

import oracle
from kv_cache_quantized_b200 import workloads as W

FORMATS = [(3, 0), (2, 1), (2, 0), (1, 1), (3, 1)]


@pytest.mark.parametrize("E,M", FORMATS)
def test_levels_and_nearest_level_decision(E, M):
    lv = oracle.pot_levels(E, M)
    assert len(lv) == 1 << (E + M) and np.all(np.diff(lv) > 0)
    assert lv[0] == 2.0 ** -((1 << E) - 1)
    k = W.normal((3000, 64), 3, np.float16)
    codes, alpha = oracle.pot_encode(k, E, M)
    assert np.array_equal(alpha, np.max(np.abs(k), axis=-1))
    u = np.divide(k.astype(np.float32), alpha.astype(np.float32)[:, None], dtype=np.float32).astype(np.float64)
    rank = codes & ((1 << (E + M)) - 1)
    dist = np.abs(np.abs(u)[..., None] - lv)
    best = np.argmin(dist, axis=-1)
    # the nearest level, except on an exact midpoint where the larger one is taken
    diff = rank != best
    if diff.any():
        d_r = np.take_along_axis(dist, rank[..., None], -1)[..., 0][diff]
        d_b = np.take_along_axis(dist, best[..., None], -1)[..., 0][diff]
        assert np.all(d_r == d_b) and np.all(rank[diff] == best[diff] + 1)
    sign = (codes >> (E + M)) & 1
    assert np.array_equal(sign == 1, u < 0)


@pytest.mark.parametrize("E,M,bound", [(3, 0, 1 / 3), (4, 0, 1 / 3), (3, 1, 1 / 5), (2, 1, 1 / 5)])
def test_relative_error_of_nearest_level(E, M, bound):
    """Inside the covered range [2^-e_max, 1] nearest rounding to {2^-e} errs by at most 1/3 (at the midpoint
    3/4 2^-e), and with one mantissa bit ({1, 1.5} 2^-e) by at most 1/5 (at the midpoint 5/4 2^-e)."""
    g = np.random.default_rng(4)
    e_max = (1 << E) - 1
    u = 2.0 ** -g.uniform(0, e_max, size=200000)
    k = np.concatenate([np.ones(1), u]).astype(np.float16)
    k = k[: (len(k) // 8) * 8].reshape(-1, 8)
    k[:, 0] = 1.0  # alpha = 1 on every row
    codes, alpha = oracle.pot_encode(k, E, M)
    rec = oracle.pot_decode(codes, alpha, E, M)
    rel = np.abs(rec - k.astype(np.float64)) / np.abs(k.astype(np.float64))
    assert rel.max() <= bound + 1e-12 and rel.max() > 0.9 * bound


@pytest.mark.parametrize("E,M", FORMATS)
def test_shift_accumulate_is_the_exact_dot_product(E, M):
    k = W.normal((500, 128), 5, np.float16)
    q = W.normal((128,), 6, np.float32)
    codes, alpha = oracle.pot_encode(k, E, M)
    Q, s = oracle.pot_quantize_query(q)
    S = oracle.pot_score_int(Q, codes, E, M)
    # the same integer as a plain fp64 dot product of Q with the signed levels times 2^F (all dyadic: exact)
    F = (1 << E) - 1 + M
    lv = oracle.pot_levels(E, M)
    signed = np.where((codes >> (E + M)) & 1, -1.0, 1.0) * lv[codes & ((1 << (E + M)) - 1)] * 2.0 ** F
    assert np.array_equal(S.astype(np.float64), signed @ Q.astype(np.float64))
    # and the real score is the fp64 dot product of the dequantized query and key
    sc = oracle.pot_score(q, codes, alpha, E, M, scale=0.25)
    ref = 0.25 * (oracle.pot_decode(codes, alpha, E, M) @ (float(s) * Q.astype(np.float64)))
    assert np.allclose(sc, ref, rtol=1e-12, atol=1e-12)


def test_query_fixed_point():
    q = W.normal((40, 128), 7, np.float32)
    Q, s = oracle.pot_quantize_query(q)
    assert np.all(np.max(np.abs(Q), axis=-1) == 32767)
    # rint of q / s, the quotient itself rounded to fp32 first (half an ulp of numbers up to 32767: 2^-10)
    err = np.abs(q.astype(np.float64) - s[:, None].astype(np.float64) * Q)
    assert np.all(err <= (0.5 + 2.0 ** -10) * s[:, None])
    Q0, s0 = oracle.pot_quantize_query(np.zeros(8, np.float32))
    assert s0 == 0 and np.all(Q0 == 0)


@pytest.mark.parametrize("chunk", [1, 7, 64, 1000])
def test_integer_log2_online_softmax_is_the_two_pass_definition(chunk):
    g = np.random.default_rng(8)
    r = g.integers(-40, 40, size=777)
    v = g.standard_normal((777, 16))
    want = (np.ldexp(1.0, r - r.max())[:, None] * v).sum(0) / np.ldexp(1.0, r - r.max()).sum()
    assert np.allclose(oracle.pot_attention_online(r, v, chunk), want, rtol=1e-12, atol=1e-14)


def test_attention_special_cases():
    E, M = 3, 0
    B, Hkv, G, T, d = 2, 1, 2, 50, 64
    k = W.normal((B, Hkv, T, d), 9, np.float16)
    v = W.normal((B, Hkv, T, d), 10, np.float16)
    codes, alpha = oracle.pot_encode(k, E, M)
    q = np.zeros((B, Hkv * G, d), np.float32)  # zero query: every r = 0, the plain mean of the values
    out = oracle.pot_attention(q, codes, alpha, v, E, M, 1 / 8, seq_lens=[T, 0])
    assert np.allclose(out[0, 0], v[0, 0].astype(np.float64).mean(0), rtol=1e-12, atol=1e-12)
    assert np.all(out[1] == 0)


def _eps_s(E, M, seed=11):
    k = W.normal((3000, 64), seed, np.float16)
    q = W.normal((40, 64), seed + 1, np.float32)
    codes, alpha = oracle.pot_encode(k, E, M)
    s = np.stack([oracle.pot_score(q[i], codes, alpha, E, M) for i in range(len(q))])
    exact = q.astype(np.float64) @ k.astype(np.float64).T
    return np.linalg.norm(s - exact) / np.linalg.norm(exact)


def test_page_findings_on_gaussian_keys():
    """The page: nearest-PoT relative error is scale-free, so extra exponent bits buy nothing; the sub-power
    mantissa term halves the score error.  On N(0,1) keys with per-token scaling: 3 and 4 exponent bits give the
    same score error, and one mantissa bit takes it to about half."""
    e3, e4, e3m1 = _eps_s(3, 0), _eps_s(4, 0), _eps_s(3, 1)
    assert abs(e3 - e4) <= 0.01 * e3
    assert 0.4 <= e3m1 / e3 <= 0.65
