"""Pins for the LOOKAT oracle (product-quantized keys, asymmetric distance computation): the fp32 nearest-centroid
decision against an fp64 brute force, per-subspace encoding against a search over the whole product codebook,
k-means against scikit-learn, the Lloyd objective never increasing, ADC scores against reconstructed-key dot
products, and attention against torch's scaled_dot_product_attention."""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantized_b200 import workloads as W


def _codebooks(m, K, ds, seed):
    return W.normal((m, K, ds), seed, np.float32)


def test_fp32_decision_matches_fp64_nearest_except_near_ties():
    x = W.normal((4000, 64), 1, np.float16)
    cb = _codebooks(4, 256, 16, 2)
    codes = oracle.pq_encode(x, cb)
    xs = oracle.pq_split(x.astype(np.float64), 4)
    n_diff = 0
    for i in range(4):
        d64 = ((xs[:, i, None, :] - cb[i].astype(np.float64)[None]) ** 2).sum(-1)
        best = np.argmin(d64, axis=1)
        diff = best != codes[:, i]
        if diff.any():  # only where the two nearest distances are within fp32 rounding of each other
            rows = np.nonzero(diff)[0]
            gap = np.abs(d64[rows, best[rows]] - d64[rows, codes[rows, i]])
            assert np.all(gap <= 1e-5 * d64[rows, best[rows]])
        n_diff += int(diff.sum())
    assert n_diff <= 2


def test_per_subspace_encoding_is_the_product_codebook_search():
    """m=2 subspaces of K=4: the nearest of all 16 reconstructions equals the per-subspace choice."""
    cb = _codebooks(2, 4, 3, 3).astype(np.float64).astype(np.float32)
    x = W.normal((300, 6), 4, np.float32)
    codes = oracle.pq_encode(x, cb)
    for n in range(len(x)):
        best, bd = None, np.inf
        for a, b in itertools.product(range(4), range(4)):
            r = np.concatenate([cb[0, a], cb[1, b]]).astype(np.float64)
            dd = np.sum((x[n].astype(np.float64) - r) ** 2)
            if dd < bd:
                best, bd = (a, b), dd
        assert tuple(codes[n]) == best


def _blobs(K, ds, per, seed):
    g = W.rng(seed)
    centers = 10.0 * g.standard_normal((K, ds))
    pts = centers[:, None, :] + g.standard_normal((K, per, ds))
    x = pts.reshape(-1, ds)
    perm = g.permutation(len(x))
    return x[perm], perm


def test_kmeans_matches_scikit_learn_lloyd():
    from sklearn.cluster import KMeans
    K, ds = 8, 4
    x, perm = _blobs(K, ds, 200, 5)
    x = x.astype(np.float32)
    # one initial centroid per blob, away from its mean
    init = np.stack([x[np.nonzero(perm // 200 == k)[0][0]] for k in range(K)]).astype(np.float32)
    c, assign = oracle.pq_kmeans(x, init, iters=30)
    km = KMeans(n_clusters=K, init=init.astype(np.float64), n_init=1, max_iter=30, tol=0.0, algorithm="lloyd")
    km.fit(x.astype(np.float64))
    assert np.allclose(c, km.cluster_centers_, rtol=0, atol=1e-5)
    assert np.array_equal(assign, km.labels_)


def test_kmeans_objective_never_increases_and_empty_cells_stay():
    x = W.normal((2000, 8), 6, np.float32)
    init = x[:64].copy()
    init[63] = 1e3  # far away: never nearest, keeps its place
    prev = np.inf
    c = init
    for _ in range(6):
        c_next, assign = oracle.pq_kmeans(x, c, iters=1)
        obj = np.sum((x.astype(np.float64) - c[assign].astype(np.float64)) ** 2)
        assert obj <= prev * (1 + 1e-12)
        prev = obj
        c = c_next
    assert np.all(c[63] == np.float32(1e3))


def test_train_uses_the_given_rows_and_k_means_per_subspace():
    x = W.normal((500, 32), 7, np.float16)
    rows = np.arange(0, 500, 50)
    cb = oracle.pq_train(x, 4, rows, iters=3)
    assert cb.shape == (4, 10, 8) and cb.dtype == np.float32
    xs = oracle.pq_split(x, 4)
    for i in range(4):
        c, _ = oracle.pq_kmeans(xs[:, i], xs[rows, i].astype(np.float32), 3)
        assert np.array_equal(c, cb[i])


@pytest.mark.parametrize("m,K", [(2, 256), (4, 16), (8, 256)])
def test_adc_score_is_the_reconstructed_dot_product(m, K):
    d = 64
    cb = _codebooks(m, K, d // m, 8 + m)
    x = W.normal((200, d), 9, np.float16)
    q = W.normal((d,), 10, np.float64)
    codes = oracle.pq_encode(x, cb)
    a = oracle.pq_score(q, codes, cb, scale=0.3)
    b = oracle.pq_score_bruteforce(q, codes, cb, scale=0.3)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
    # the table is the query's subvector against each centroid
    tab = oracle.pq_table(q, cb)
    assert tab.shape == (m, K)
    i, k = m - 1, K // 3
    assert math.isclose(tab[i, k], float(np.dot(q[i * (d // m):(i + 1) * (d // m)], cb[i, k].astype(np.float64))),
                        rel_tol=1e-13)


def test_pq_attention_matches_sdpa_on_reconstructed_keys():
    B, Hkv, G, T, d, m, K = 2, 2, 3, 90, 64, 4, 32
    cbs = np.stack([_codebooks(m, K, d // m, 20 + h) for h in range(Hkv)])
    k = W.normal((B, Hkv, T, d), 21, np.float16)
    v = W.normal((B, Hkv, T, d), 22, np.float16)
    q = W.normal((B, Hkv * G, d), 23, np.float32)
    codes = np.stack([np.stack([oracle.pq_encode(k[b, h], cbs[h]) for h in range(Hkv)]) for b in range(B)])
    lens = np.array([T, 37])
    out = oracle.pq_decode_attention(q, codes, cbs, v, 1 / math.sqrt(d), seq_lens=lens)
    for b in range(B):
        T_b = lens[b]
        khat = np.stack([oracle.pq_decode(codes[b, h, :T_b], cbs[h]) for h in range(Hkv)])
        kk = torch.from_numpy(np.repeat(khat, G, axis=0))[:, None]
        vv = torch.from_numpy(np.repeat(v[b, :, :T_b].astype(np.float64), G, axis=0))[:, None]
        qq = torch.from_numpy(q[b].astype(np.float64))[:, None, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=1 / math.sqrt(d))[:, 0, 0]
        assert np.allclose(out[b], ref.numpy(), rtol=1e-10, atol=1e-12)
