"""GPU parity of the LOOKAT product-quantized key path against the oracle: k-means training (the same initial
centroids and iteration count), encoding (the nearest-centroid decision is taken in the same fp32 order on both
sides, so indices are bit-exact), asymmetric-distance scores and decode attention over fp16 values."""

import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantized_b200 import ops
from kv_cache_quantized_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _codebooks(k, Hkv, m, K, iters=3, seed=0):
    """Per-KV-head codebooks [Hkv, m, K, d/m] learned by the oracle's k-means on keys k [B, Hkv, T, d]."""
    rng = np.random.default_rng(seed)
    out = []
    for h in range(Hkv):
        x = k[:, h].reshape(-1, k.shape[-1])
        rows = rng.choice(len(x), size=K, replace=False)
        out.append(oracle.pq_train(x, m, rows, iters))
    return np.stack(out)


@pytest.mark.parametrize("d,m,K", [(64, 4, 64), (128, 8, 256), (64, 16, 16)])
def test_train_matches_oracle_kmeans(d, m, K):
    x = W.lognormal_rows((6000, d), 11 + m, dtype=np.float16)
    rows = np.random.default_rng(12).choice(len(x), size=K, replace=False)
    want = oracle.pq_train(x, m, rows, iters=4)
    init = np.ascontiguousarray(oracle.pq_split(x, m)[rows].transpose(1, 0, 2)).astype(np.float32)
    got = ops.pq_train(cuda(x), cuda(init), 4).cpu().numpy()
    # the same assignments every iteration and fp64 sums rounded to fp32: equal but for a summation-order ulp
    assert np.allclose(got, want, rtol=2.0 ** -22, atol=0), np.max(np.abs(got - want))


@pytest.mark.parametrize("dt", [np.float16, np.float32])
def test_encode_is_bit_exact(dt):
    d, m, K, Hkv, T = 128, 8, 256, 3, 700
    k = W.lognormal_rows((2, Hkv, T, d), 13, dtype=dt)
    cbs = _codebooks(k, Hkv, m, K)
    got = ops.pq_encode(cuda(k), cuda(cbs)).cpu().numpy()
    for b in range(2):
        for h in range(Hkv):
            assert np.array_equal(got[b, h], oracle.pq_encode(k[b, h], cbs[h]))


CASES = [(64, 4, 256, 1), (64, 2, 256, 4), (128, 8, 256, 4), (128, 16, 16, 8), (128, 4, 64, 2)]


@pytest.mark.parametrize("d,m,K,G", CASES)
def test_scores_and_attention_match_oracle(d, m, K, G):
    B, Hkv, T, Tcap = 2, 2, 1500, 1536
    Hq = Hkv * G
    k = W.lognormal_rows((B, Hkv, T, d), 20 + d + m, dtype=np.float16)
    v = W.normal((B, Hkv, T, d), 21, np.float16)
    q = W.normal((B, Hq, d), 22, np.float32)
    cbs = _codebooks(k, Hkv, m, K, seed=23)
    codes = np.stack([np.stack([oracle.pq_encode(k[b, h], cbs[h]) for h in range(Hkv)]) for b in range(B)])
    cpad = np.zeros((B, Hkv, Tcap, m), np.uint8)
    cpad[:, :, :T] = codes
    vpad = np.zeros((B, Hkv, Tcap, d), np.float16)
    vpad[:, :, :T] = v
    lens = np.array([T, 333], np.int32)
    scale = 1.0 / math.sqrt(d)
    sc = ops.pq_score(cuda(q), cuda(cpad), cuda(cbs), scale=scale, seq_lens=cuda(lens), T=T).cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            hk, n = h // G, lens[b]
            want = oracle.pq_score(q[b, h], codes[b, hk, :n], cbs[hk], scale)
            tab = np.abs(oracle.pq_table(q[b, h], cbs[hk]))
            A = scale * tab[np.arange(m)[None, :], codes[b, hk, :n]].sum(-1)
            parity.check_scores(sc[b, h, :n], want, A)
            assert np.all(np.isneginf(sc[b, h, n:]))
    out = ops.pq_attend_decode(cuda(q), cuda(cpad), cuda(cbs), cuda(vpad), seq_lens=cuda(lens), T=T).cpu().numpy()
    want = oracle.pq_decode_attention(q, codes, cbs, v, scale, seq_lens=lens)
    parity.check_outputs(out, want)


def test_empty_rows_and_gpt2_shape():
    """The GPT-2 shape of the LOOKAT evaluation (12 heads, d_k = 64, up to 1024 tokens) at 32x and 64x compression
    (m = 4 and m = 2 one-byte indices against 128 bytes of fp16 key), with an empty batch row."""
    B, H, T, d = 3, 12, 1024, 64
    k = W.lognormal_rows((B, H, T, d), 30, dtype=np.float16)
    v = W.normal((B, H, T, d), 31, np.float16)
    q = W.normal((B, H, d), 32, np.float32)
    lens = np.array([1024, 0, 517], np.int32)
    for m in (4, 2):
        cbs = _codebooks(k, H, m, 256, iters=2, seed=33 + m)
        codes = ops.pq_encode(cuda(k), cuda(cbs))
        out = ops.pq_attend_decode(cuda(q), codes, cuda(cbs), cuda(v), seq_lens=cuda(lens)).cpu().numpy()
        oc = np.stack([np.stack([oracle.pq_encode(k[b, h], cbs[h]) for h in range(H)]) for b in range(B)])
        assert np.array_equal(codes.cpu().numpy(), oc)
        want = oracle.pq_decode_attention(q, oc, cbs, v, 1 / math.sqrt(d), seq_lens=lens)
        parity.check_outputs(out, want)
        assert np.all(out[1] == 0)
