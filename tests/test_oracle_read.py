"""Pins for the oracle's read path and attention: LUT gather-sum against explicit dequantize-then-dot (AXELRAM
Abstract: table lookup on read, no inverse transform), attention against torch's scaled_dot_product_attention on
the explicitly dequantized cache (a library routine), softmax special cases, and the 102.4x count reading."""

import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantized_b200 import workloads as W


@pytest.mark.parametrize("d", [8, 64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lut_score_equals_dequantize_then_dot(d, bits):
    s = W.sign_vector(d, d + bits)
    k = W.lognormal_rows((40, d), 10 + bits, dtype=np.float32)
    q = W.normal((d,), 20 + bits, np.float64)
    codes, n16 = oracle.write(k, s, bits)
    a = oracle.score_lut(q, codes, n16, s, bits)
    b = oracle.score_bruteforce(q, codes, n16, s, bits)
    scale = np.abs(q).sum() * np.abs(n16.astype(np.float64)).max()
    assert np.max(np.abs(a - b)) <= 1e-12 * scale


def test_lut_shape_and_entries():
    d, bits = 64, 3
    s = W.sign_vector(d, 1)
    q = W.normal((d,), 2, np.float64)
    lut = oracle.query_lut(q, s, bits)
    c, _ = oracle.codebook(d, bits)
    qt = oracle.hadamard(d) @ (s * q)
    assert lut.shape == (d, 1 << bits)
    assert np.allclose(lut, np.outer(qt, c), rtol=1e-15, atol=0)


def test_score_scale_and_norm_factor():
    d, bits = 128, 4
    s = W.sign_vector(d, 3)
    k = W.normal((10, d), 4, np.float32)
    q = W.normal((d,), 5, np.float64)
    codes, n16 = oracle.write(k, s, bits)
    a = oracle.score_lut(q, codes, n16, s, bits, scale=0.25)
    b = oracle.score_lut(q, codes, np.ones_like(n16), s, bits, scale=1.0)
    assert np.allclose(a, 0.25 * n16.astype(np.float64) * b, rtol=1e-14)


def _sdpa(q, k, v, scale, G):
    """torch SDPA in fp64 on CPU; q [B,Hq,1,d], k/v [B,Hkv,T,d]."""
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(np.repeat(k, G, axis=1))
    vt = torch.from_numpy(np.repeat(v, G, axis=1))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale).numpy()


@pytest.mark.parametrize("vquant", [False, True])
def test_decode_attention_matches_sdpa_on_dequantized_cache(vquant):
    B, Hq, Hkv, T, d, bits = 2, 8, 2, 96, 64, 3
    G = Hq // Hkv
    s = W.sign_vector(d, 7)
    k = W.lognormal_rows((B, Hkv, T, d), 8, dtype=np.float16)
    v = W.normal((B, Hkv, T, d), 9, np.float16)
    q = W.normal((B, Hq, d), 10, np.float32)
    kc, kn = oracle.write(k, s, bits)
    scale = 1.0 / math.sqrt(d)
    khat = oracle.dequantize(kc, kn, s, bits, d)
    if vquant:
        vc, vn = oracle.write(v, s, bits)
        vv = oracle.dequantize(vc, vn, s, bits, d)
        out = oracle.decode_attention(q, kc, kn, s, bits, scale, vcodes=vc, vn16=vn)
    else:
        vv = v.astype(np.float64)
        out = oracle.decode_attention(q, kc, kn, s, bits, scale, v=v)
    ref = _sdpa(q.astype(np.float64)[:, :, None, :], khat, vv, scale, G)[:, :, 0, :]
    assert np.max(np.abs(out - ref)) < 1e-12


def test_quantized_v_single_inverse_transform_identity():
    """sum_t p_t * s*H(n_t c[idx_t]) == s * H(sum_t p_t n_t c[idx_t]): the one-inverse-transform form."""
    d, bits, T = 128, 4, 50
    s = W.sign_vector(d, 11)
    v = W.lognormal_rows((T, d), 12, dtype=np.float16)
    vc, vn = oracle.write(v, s, bits)
    p = W.rng(13).random(T)
    direct = (p[:, None] * oracle.dequantize(vc, vn, s, bits, d)).sum(0)
    c, _ = oracle.codebook(d, bits)
    rot = (p * vn.astype(np.float64))[:, None] * c[oracle.unpack(vc, d, bits)]
    once = s * (oracle.hadamard(d) @ rot.sum(0))
    assert np.max(np.abs(direct - once)) < 1e-12


def test_softmax_special_cases():
    d, bits = 64, 2
    s = W.sign_vector(d, 14)
    k = W.normal((1, 1, 30, d), 15, np.float16)
    v = W.normal((1, 1, 30, d), 16, np.float16)
    kc, kn = oracle.write(k, s, bits)
    # T = 1: the output is v_0
    q = W.normal((1, 1, d), 17, np.float32)
    o1 = oracle.decode_attention(q, kc[:, :, :1], kn[:, :, :1], s, bits, 0.3, v=v[:, :, :1])
    assert np.allclose(o1[0, 0], v[0, 0, 0].astype(np.float64), atol=0)
    # zero query: all scores equal -> the mean of V
    o2 = oracle.decode_attention(np.zeros((1, 1, d), np.float32), kc, kn, s, bits, 0.3, v=v)
    assert np.allclose(o2[0, 0], v[0, 0].astype(np.float64).mean(0), atol=1e-14)
    # scaling the query and dividing the scale leaves the output unchanged
    o3 = oracle.decode_attention(2 * q, kc, kn, s, bits, 0.15, v=v)
    o4 = oracle.decode_attention(q, kc, kn, s, bits, 0.3, v=v)
    assert np.allclose(o3, o4, atol=1e-13)


def test_seq_lens_truncate_and_empty_rows():
    B, Hq, Hkv, T, d, bits = 3, 4, 2, 40, 64, 4
    s = W.sign_vector(d, 18)
    k = W.normal((B, Hkv, T, d), 19, np.float16)
    v = W.normal((B, Hkv, T, d), 20, np.float16)
    q = W.normal((B, Hq, d), 21, np.float32)
    kc, kn = oracle.write(k, s, bits)
    lens = [T, 17, 0]
    out = oracle.decode_attention(q, kc, kn, s, bits, 0.125, v=v, seq_lens=lens)
    ref1 = oracle.decode_attention(q[1:2], kc[1:2, :, :17], kn[1:2, :, :17], s, bits, 0.125, v=v[1:2, :, :17])
    assert np.array_equal(out[1:2], ref1)
    assert np.all(out[2] == 0)


def test_multiplication_count_reading():
    """The 102.4x figure is reproduced exactly by T*d / (d*2^b + T) at d=128, b=4, T=8192 (the reading of the
    Key Points' identity); it is reported, not gated."""
    conv, lut = oracle.multiplication_counts(128, 4, 8192)
    assert conv / lut == pytest.approx(102.4, rel=0, abs=1e-12)
    for bits, T in ((1, 1024), (2, 2048), (3, 4096)):
        conv, lut = oracle.multiplication_counts(128, bits, T)
        assert conv / lut == pytest.approx(102.4, abs=1e-12)
