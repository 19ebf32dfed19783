"""Plain CPU oracle for LOOKAT-style product-quantized keys scored by asymmetric distance computation.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU baseline and reference arm) may import it; the product path never does, and the two share no
code.

What is computed (source: the newx.sg summary and abstract of "LOOKAT: Lookup-Optimized Key-Attention for
Memory-Efficient Transformers"; the pages give no formulas, so the textbook definitions of product quantization and
asymmetric distance computation are written out here):

* Keys are cut into m contiguous subspaces of d/m coordinates (subspace i holds coordinates [i d/m, (i+1) d/m)).
* Each subspace has a codebook of K centroids learned by k-means on keys (Lloyd's iterations from given initial
  centroids; a point goes to its nearest centroid, squared Euclidean distance, lowest index on a tie; a centroid
  becomes the mean of its points; a centroid with no points stays where it was).
* A key is stored as m indices, one per subspace: the nearest centroid of its subvector (encode).
* A query scores a stored key without reconstructing it: a table T[i][k] = q^(i) . C_i[k] is built once per query
  (m x K dot products), and the score of a key is the sum over subspaces of the table entries at its indices, times
  the softmax scale (asymmetric distance computation: the query stays exact, only the key is quantized).
* Decode attention is the softmax of those scores times fp16 values.

Precision: every floating-point step is fp64 except the two places where floating point decides an integer -- the
nearest-centroid index in encode and in the k-means assignment.  There both sides take the decision in the
kernel's precision and order: the distance is sum_j (x_j - c_j)^2 over the subspace's coordinates in increasing j,
every subtraction, product and sum rounded to fp32 (no fused multiply-add), x converted from its storage type to
fp32 exactly.  The k-means means are summed in fp64 and rounded to fp32, the codebooks' storage type.

Pins (tests/test_oracle_lookat.py): the fp32 decision against an fp64 brute-force nearest centroid; per-subspace
encoding against a brute-force search over the whole product codebook on a tiny case; k-means against
scikit-learn's Lloyd k-means from the same initial centroids; the objective never increasing; ADC scores against
the dot product with the reconstructed key; attention against torch's scaled_dot_product_attention on
reconstructed keys.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "pq_split",
    "pq_distances_f32",
    "pq_encode",
    "pq_decode",
    "pq_kmeans",
    "pq_train",
    "pq_table",
    "pq_score",
    "pq_score_bruteforce",
    "pq_decode_attention",
]


def pq_split(x, m):
    """[..., d] -> [..., m, d/m]: subspace i holds coordinates [i d/m, (i+1) d/m)."""
    x = np.asarray(x)
    d = x.shape[-1]
    if d % m:
        raise ValueError("m must divide d")
    return x.reshape(x.shape[:-1] + (m, d // m))


def pq_distances_f32(xs, cb):
    """Squared distances of subvectors xs [N, ds] to centroids cb [K, ds], as the kernel forms them: fp32, summed
    over j in increasing order, each subtraction, product and sum rounded (no fused multiply-add).  [N, K] f32."""
    xs = np.asarray(xs).astype(np.float32)
    cb = np.asarray(cb, dtype=np.float32)
    acc = np.zeros((xs.shape[0], cb.shape[0]), dtype=np.float32)
    for j in range(xs.shape[1]):
        diff = np.subtract(xs[:, j:j + 1], cb[None, :, j], dtype=np.float32)
        acc = np.add(acc, np.multiply(diff, diff, dtype=np.float32), dtype=np.float32)
    return acc


def _nearest(dist):
    """First index of the minimum of each row (ties go to the lowest index)."""
    return np.argmin(dist, axis=1)


def pq_encode(x, codebooks):
    """Indices [..., m] (int64) of the nearest centroid of every subvector; codebooks [m, K, d/m] f32."""
    codebooks = np.asarray(codebooks, dtype=np.float32)
    m = codebooks.shape[0]
    xs = pq_split(x, m)
    lead = xs.shape[:-2]
    flat = xs.reshape((-1, m, xs.shape[-1]))
    out = np.zeros((flat.shape[0], m), dtype=np.int64)
    for i in range(m):
        out[:, i] = _nearest(pq_distances_f32(flat[:, i], codebooks[i]))
    return out.reshape(lead + (m,))


def pq_decode(codes, codebooks):
    """Reconstructed keys [..., d] (fp64) from indices [..., m]."""
    codebooks = np.asarray(codebooks, dtype=np.float64)
    m = codebooks.shape[0]
    codes = np.asarray(codes)
    parts = [codebooks[i][codes[..., i]] for i in range(m)]
    return np.concatenate(parts, axis=-1)


def pq_kmeans(xs, init, iters):
    """Lloyd's k-means of subvectors xs [N, ds] from centroids init [K, ds] for a fixed number of iterations.

    Each iteration: assign every point to its nearest centroid (pq_distances_f32, lowest index on a tie); move every
    centroid with at least one point to the fp64 mean of its points, rounded to fp32; a centroid with no points
    stays.  Returns (centroids [K, ds] f32, assignments [N] of the last iteration).
    """
    c = np.asarray(init, dtype=np.float32).copy()
    x64 = np.asarray(xs).astype(np.float64)
    assign = np.zeros(len(x64), dtype=np.int64)
    for _ in range(iters):
        assign = _nearest(pq_distances_f32(xs, c))
        for k in range(c.shape[0]):
            members = x64[assign == k]
            if len(members):
                c[k] = (members.sum(axis=0) / len(members)).astype(np.float32)
    return c, assign


def pq_train(x, m, init_rows, iters):
    """Codebooks [m, K, d/m] f32 learned on keys x [N, d]: per subspace, k-means from the subvectors of the rows
    init_rows (K row indices of x) as initial centroids."""
    xs = pq_split(np.asarray(x), m)
    init_rows = np.asarray(init_rows)
    out = []
    for i in range(m):
        sub = xs[:, i]
        c, _ = pq_kmeans(sub, sub[init_rows].astype(np.float32), iters)
        out.append(c)
    return np.stack(out)


def pq_table(q, codebooks):
    """T[i][k] = q^(i) . C_i[k] (fp64) for one query q [d]: [m, K]."""
    codebooks = np.asarray(codebooks, dtype=np.float64)
    qs = pq_split(np.asarray(q, dtype=np.float64), codebooks.shape[0])
    return np.einsum("ij,ikj->ik", qs, codebooks)


def pq_score(q, codes, codebooks, scale=1.0):
    """ADC scores of one query q [d] against codes [T, m]: scale * sum_i T[i][codes_i]  -> [T]."""
    tab = pq_table(q, codebooks)
    codes = np.asarray(codes)
    m = tab.shape[0]
    return scale * tab[np.arange(m)[None, :], codes].sum(axis=-1)


def pq_score_bruteforce(q, codes, codebooks, scale=1.0):
    """scale * q . decode(codes): the dot product with the reconstructed key."""
    return scale * (pq_decode(codes, codebooks) @ np.asarray(q, dtype=np.float64))


def pq_decode_attention(q, codes, codebooks, v, scale, seq_lens=None):
    """Decode attention over product-quantized keys: one query per (batch, query head).

    q [B, Hq, d]; codes [B, Hkv, Tc, m]; codebooks [Hkv, m, K, d/m] (one set per KV head); v [B, Hkv, Tc, d] fp16.
    Query head h reads KV head h // (Hq/Hkv); row b attends to its first seq_lens[b] tokens (0 gives 0).
    z_t = scale * ADC score, two-pass softmax, out = sum_t p_t v_t / sum_t p_t.  Returns f64 [B, Hq, d].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv, Tc = codes.shape[1], codes.shape[2]
    G = Hq // Hkv
    lens = [Tc] * B if seq_lens is None else [int(n) for n in seq_lens]
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        T = lens[b]
        if T == 0:
            continue
        for hk in range(Hkv):
            vals = np.asarray(v[b, hk, :T], dtype=np.float64)
            for g in range(G):
                h = hk * G + g
                z = pq_score(q[b, h], codes[b, hk, :T], codebooks[hk], scale)
                p = np.exp(z - z.max())
                out[b, h] = (p[:, None] * vals).sum(axis=0) / p.sum()
    return out
