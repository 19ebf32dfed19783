"""Plain, slow fp64 CPU oracle for AXELRAM decode-time attention from quantized key indices.

TEST INFRASTRUCTURE ONLY.  The only code that may import, call or execute anything in this package is
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference``
arm).  The product path (``kv_cache_quantized_b200``) never imports it and shares no code with it: no kernels,
headers, helpers, tables or constant generators.  Inputs come from the caller (seeded generators in
``kv_cache_quantized_b200.workloads``, which hold none of the method's arithmetic).

What the method computes (source: "AXELRAM: Quantize Once, Never Dequantize", arXiv 2604.02638, as carried by the
ai-navigate-news digest -- Key Points and Abstract -- and by the mlsanity index card -- Abstract):

* Write path, "transform on write" (Key Points, 2nd item; Abstract): each key is passed through a fixed orthogonal
  transform, which makes every coordinate of the unit vector close to N(0, 1/d); each coordinate is then replaced by
  the index of its cell in a scalar quantizer that is optimal for N(0, 1/d) and therefore depends only on (d, b)
  (Abstract: design-time fixed codebook).  Concrete choices taken here (the pages name none): the transform is a
  +-1 sign diagonal D_s followed by the Sylvester Walsh-Hadamard matrix scaled by 1/sqrt(d); the codebook is the
  Lloyd-Max quantizer of N(0,1) scaled by 1/sqrt(d); the key's L2 norm is kept as an fp16 number; the indices are
  bit-packed LSB-first.
* Read path, "table lookup on read with no inverse transform" (Key Points, 2nd item; Abstract): the query is
  transformed once, a d x 2^b table of products q~_j * c_k is built, and each cached token's score is its stored
  norm times the sum over j of the table entries picked by its indices.  No key is reconstructed (Key Points, 1st
  item: scores come straight from the quantized indices).
* Softmax and the value product are not on the pages (an SRAM macro only scores).  The oracle uses their textbook
  definitions: two-pass softmax, weighted sum of the values (fp16 values, or values quantized the same way and
  reconstructed explicitly).
* Sign-pattern selection (Key Points, 4th item; Abstract): a one-time, gradient-free choice among candidate sign
  vectors on a few calibration samples.  Objective taken here: attention-output MSE of quantized-K attention
  against unquantized fp64 attention; the first index of the minimum wins.  Over the whole model (one sign
  vector), or layer by layer (one sign vector per layer: the pages trace the sensitivity to layer-wise norm
  heterogeneity).

Every function below is pinned by a ``-m "not gpu"`` test against closed forms, library routines or invariants
(tests/test_oracle_*.py).  Nothing here is "parity unpinned".
"""

from __future__ import annotations

import functools
import math
from statistics import NormalDist

import numpy as np

__all__ = [
    "gaussian_lloyd_max",
    "codebook",
    "hadamard",
    "rotate",
    "quantize_rows",
    "pack",
    "unpack",
    "write",
    "query_lut",
    "score_lut",
    "dequantize",
    "score_bruteforce",
    "decode_attention",
    "attention",
    "select_signs",
    "select_signs_per_layer",
    "multiplication_counts",
]


# ---------------------------------------------------------------------------------------------------------------
# a0. Design-time codebook (Abstract: the optimal quantizer for N(0, 1/d) depends only on d and b).
# ---------------------------------------------------------------------------------------------------------------

def _pdf(x: float) -> float:
    """Standard normal density; 0 at +-inf."""
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _upper_tail(x: float) -> float:
    """P(X >= x) for X ~ N(0,1), through erfc so that the upper tail keeps its precision."""
    if x == math.inf:
        return 0.0
    if x == -math.inf:
        return 1.0
    return 0.5 * math.erfc(x / math.sqrt(2.0))


def _cell_mass(a: float, b: float) -> float:
    """P(a <= X < b) for X ~ N(0,1), computed on the side of zero where it does not cancel."""
    if a >= 0.0:
        return _upper_tail(a) - _upper_tail(b)
    return _upper_tail(-b) - _upper_tail(-a)


@functools.lru_cache(maxsize=None)
def gaussian_lloyd_max(bits: int, tol: float = 1e-15, max_iter: int = 1_000_000):
    """Lloyd-Max quantizer of N(0,1) with L = 2^bits levels (Lloyd's method I, Max 1960).

    Alternates the two optimality conditions until no level moves by more than ``tol``:
      thresholds  tau_k = (gamma_{k-1} + gamma_k) / 2,                    k = 1..L-1
      levels      gamma_k = (pdf(tau_k) - pdf(tau_{k+1})) / P(tau_k <= X < tau_{k+1}),   tau_0=-inf, tau_L=+inf
    (the second is E[X | cell k] for the Gaussian, since d/dx pdf(x) = -x pdf(x)).
    Starts from the cell midpoints of the equal-probability partition.

    Returns (gamma [L], tau [L-1]) as float64 arrays, increasing.
    """
    if bits < 1 or bits > 8:
        raise ValueError("bits must be in 1..8")
    L = 1 << bits
    nd = NormalDist()
    gamma = [nd.inv_cdf((k + 0.5) / L) for k in range(L)]
    for _ in range(max_iter):
        tau = [-math.inf] + [0.5 * (gamma[k - 1] + gamma[k]) for k in range(1, L)] + [math.inf]
        new = [(_pdf(tau[k]) - _pdf(tau[k + 1])) / _cell_mass(tau[k], tau[k + 1]) for k in range(L)]
        moved = max(abs(a - b) for a, b in zip(new, gamma))
        gamma = new
        if moved < tol:
            break
    else:  # pragma: no cover - the Gaussian iteration converges in < 2000 steps for bits <= 4
        raise RuntimeError("Lloyd-Max iteration did not converge")
    tau = [0.5 * (gamma[k - 1] + gamma[k]) for k in range(1, L)]
    return np.array(gamma, dtype=np.float64), np.array(tau, dtype=np.float64)


def codebook(d: int, bits: int):
    """Unit-scale codebook for N(0, 1/d): centroids c_k = gamma_k / sqrt(d), thresholds t_k = tau_k / sqrt(d)."""
    gamma, tau = gaussian_lloyd_max(bits)
    s = 1.0 / math.sqrt(d)
    return gamma * s, tau * s


# ---------------------------------------------------------------------------------------------------------------
# a1. Orthogonal transform: y = H_d (s * x), H_d the Sylvester Walsh-Hadamard matrix scaled by 1/sqrt(d).
#     Written as a dense matrix-vector product on purpose (no fast transform).
# ---------------------------------------------------------------------------------------------------------------

@functools.lru_cache(maxsize=None)
def _hadamard_cached(d: int) -> np.ndarray:
    if d < 1 or (d & (d - 1)) != 0:
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1), dtype=np.float64)
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])  # Sylvester doubling
    H = H / math.sqrt(d)
    H.setflags(write=False)
    return H


def hadamard(d: int) -> np.ndarray:
    """Normalised Sylvester Walsh-Hadamard matrix H_d (symmetric, H_d @ H_d = I)."""
    return _hadamard_cached(d)


def rotate(x, signs) -> np.ndarray:
    """y = H_d (s * x) for every row of x (last axis = d)."""
    x = np.asarray(x, dtype=np.float64)
    s = np.asarray(signs, dtype=np.float64)
    H = hadamard(x.shape[-1])
    return (x * s) @ H.T


# ---------------------------------------------------------------------------------------------------------------
# a2. Norm and scalar quantization of the unit vector.
# ---------------------------------------------------------------------------------------------------------------

def quantize_rows(x, signs, bits):
    """Quantize rows of x.

    n = ||x||_2 (fp64); u = H(s*x) / n (u = 0 when n = 0); idx_j = number of thresholds t_k with u_j >= t_k,
    so index 0 is the most negative centroid and a value exactly on a threshold goes up.  The stored norm is
    fp16(n), round to nearest even.

    Returns (idx int64 [..., d], n float64 [...], n16 float16 [...], u float64 [..., d]).
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    _, t = codebook(d, bits)
    n = np.sqrt(np.sum(x * x, axis=-1))
    y = rotate(x, signs)
    safe = np.where(n > 0.0, n, 1.0)
    u = np.where(n[..., None] > 0.0, y / safe[..., None], 0.0)
    idx = np.sum(u[..., None] >= t, axis=-1).astype(np.int64)
    n16 = n.astype(np.float16)
    return idx, n, n16, u


# ---------------------------------------------------------------------------------------------------------------
# a3. Bit packing: one LSB-first bitstream per row; coordinate j occupies bits [j*b, j*b + b).
# ---------------------------------------------------------------------------------------------------------------

def pack(idx, bits) -> np.ndarray:
    idx = np.asarray(idx, dtype=np.int64)
    d = idx.shape[-1]
    nbits = d * bits
    if nbits % 8:
        raise ValueError("d*bits must be a multiple of 8")
    stream = np.zeros(idx.shape[:-1] + (nbits,), dtype=np.uint8)
    for j in range(d):
        for i in range(bits):
            stream[..., j * bits + i] = (idx[..., j] >> i) & 1
    out = np.zeros(idx.shape[:-1] + (nbits // 8,), dtype=np.uint8)
    for byte in range(nbits // 8):
        acc = np.zeros(idx.shape[:-1], dtype=np.int64)
        for i in range(8):
            acc |= stream[..., 8 * byte + i].astype(np.int64) << i
        out[..., byte] = acc.astype(np.uint8)
    return out


def unpack(codes, d, bits) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    if codes.shape[-1] * 8 != d * bits:
        raise ValueError("row length does not match d*bits/8")
    idx = np.zeros(codes.shape[:-1] + (d,), dtype=np.int64)
    for j in range(d):
        for i in range(bits):
            pos = j * bits + i
            bit = (codes[..., pos // 8].astype(np.int64) >> (pos % 8)) & 1
            idx[..., j] |= bit << i
    return idx


def write(x, signs, bits):
    """Write path a1-a3: returns (codes uint8 [..., d*b/8], n16 float16 [...])."""
    idx, _, n16, _ = quantize_rows(x, signs, bits)
    return pack(idx, bits), n16


# ---------------------------------------------------------------------------------------------------------------
# a4-a6. Read path: query transform, table, gather-sum score.
# ---------------------------------------------------------------------------------------------------------------

def query_lut(q, signs, bits) -> np.ndarray:
    """Table LUT[..., j, k] = q~_j * c_k with q~ = H(s*q)."""
    q = np.asarray(q, dtype=np.float64)
    c, _ = codebook(q.shape[-1], bits)
    qt = rotate(q, signs)
    return qt[..., :, None] * c[None, :]


def score_lut(q, codes, n16, signs, bits, scale=1.0) -> np.ndarray:
    """Scores of one query against rows of codes: scale * n16_t * sum_j LUT[j, idx_{t,j}].

    q: [d]; codes: [T, d*b/8]; n16: [T] -> [T].
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    lut = query_lut(q, signs, bits)
    idx = unpack(codes, d, bits)
    gathered = lut[np.arange(d)[None, :], idx]  # [T, d]
    return scale * np.asarray(n16, dtype=np.float64) * gathered.sum(axis=-1)


def dequantize(codes, n16, signs, bits, d) -> np.ndarray:
    """Explicit reconstruction k^ = s * H(n16 * c[idx]) in the original domain (H is its own inverse)."""
    c, _ = codebook(d, bits)
    idx = unpack(codes, d, bits)
    rot = np.asarray(n16, dtype=np.float64)[..., None] * c[idx]
    H = hadamard(d)
    return (rot @ H.T) * np.asarray(signs, dtype=np.float64)


def score_bruteforce(q, codes, n16, signs, bits) -> np.ndarray:
    """Dequantize-then-dot: q . k^_t for every row."""
    q = np.asarray(q, dtype=np.float64)
    khat = dequantize(codes, n16, signs, bits, q.shape[-1])
    return khat @ q


# ---------------------------------------------------------------------------------------------------------------
# a7-a10. Decode attention over a quantized key cache.
# ---------------------------------------------------------------------------------------------------------------

def _softmax_weighted_sum(z, values):
    """Two-pass softmax of z [T] (max, then sum) and the weighted sum of values [T, d]."""
    m = np.max(z)
    p = np.exp(z - m)
    return (p[:, None] * values).sum(axis=0) / p.sum()


def decode_attention(q, kcodes, kn16, signs, bits, scale, v=None, vcodes=None, vn16=None, seq_lens=None):
    """Decode attention of one query per (batch, query head) over a quantized key cache.

    q [B, Hq, d]; kcodes [B, Hkv, Tc, R]; kn16 [B, Hkv, Tc]; values either v [B, Hkv, Tc, d] (fp16) or
    vcodes/vn16 (quantized the same way as keys, same sign vector).  Query head h reads KV head h // (Hq/Hkv).
    seq_lens [B] (default: Tc for every row) limits the tokens each batch row attends to; an empty row gives 0.
    z_t = scale * score_t, out = sum_t softmax(z)_t v_t.
    Returns float64 [B, Hq, d].
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    Hkv = kcodes.shape[1]
    G = Hq // Hkv
    Tc = kcodes.shape[2]
    lens = [Tc] * B if seq_lens is None else [int(x) for x in seq_lens]
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        T = lens[b]
        if T == 0:
            continue
        for hk in range(Hkv):
            if v is not None:
                vals = np.asarray(v[b, hk, :T], dtype=np.float64)
            else:
                vals = dequantize(vcodes[b, hk, :T], vn16[b, hk, :T], signs, bits, d)
            for g in range(G):
                h = hk * G + g
                z = score_lut(q[b, h], kcodes[b, hk, :T], kn16[b, hk, :T], signs, bits, scale)
                out[b, h] = _softmax_weighted_sum(z, vals)
    return out


# ---------------------------------------------------------------------------------------------------------------
# a11. Sign-pattern selection (Key Points, 4th item; Abstract).
# ---------------------------------------------------------------------------------------------------------------

def attention(q, k, v, causal=True, scale=None):
    """Plain softmax attention in fp64. q [..., Hq, N, d]; k, v [..., Hkv, N, d]; query head h reads KV head
    h // (Hq/Hkv); with causal=True position i sees keys 0..i.  Two-pass softmax per row."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Hq, N, d = q.shape[-3:]
    Hkv = k.shape[-3]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    kk = np.repeat(k, G, axis=-3)
    vv = np.repeat(v, G, axis=-3)
    z = scale * (q @ np.swapaxes(kk, -1, -2))  # [..., Hq, N, N]
    if causal:
        mask = np.triu(np.ones((N, z.shape[-1]), dtype=bool), k=1)
        z = np.where(mask, -np.inf, z)
    m = np.max(z, axis=-1, keepdims=True)
    p = np.exp(z - m)
    return (p @ vv) / p.sum(axis=-1, keepdims=True)


def select_signs(q, k, v, candidates, bits, causal=True):
    """Score every candidate sign vector by the attention-output MSE of quantized-K attention against fp64
    unquantized attention (V unquantized), averaged over every (layer, sequence, query head, position, dim).

    q [Lyr, S, Hq, N, d]; k, v [Lyr, S, Hkv, N, d]; candidates [C, d] of +-1.
    Returns (mse float64 [C], index of the first minimum).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q.shape[-1]
    ref = attention(q, k, v, causal)
    mse = np.zeros(len(candidates), dtype=np.float64)
    for ci, s in enumerate(candidates):
        codes, n16 = write(k, s, bits)
        khat = dequantize(codes, n16, s, bits, d)
        out = attention(q, khat, v, causal)
        mse[ci] = np.mean((out - ref) ** 2)
    return mse, int(np.argmin(mse))


def select_signs_per_layer(q, k, v, candidates, bits, causal=True):
    """One sign vector per layer (the sensitivity is traced to layer-wise norm heterogeneity: AXELRAM Abstract;
    Key Points, 3rd and 4th items).  For every layer l and candidate c, the MSE of quantized-K attention against
    fp64 unquantized attention over every (sequence, query head, position, dim) of layer l only; each layer picks
    the first index of its own minimum.

    q [Lyr, S, Hq, N, d]; k, v [Lyr, S, Hkv, N, d]; candidates [C, d] of +-1.
    Returns (mse float64 [Lyr, C], best int64 [Lyr]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    d = q.shape[-1]
    Lyr = q.shape[0]
    mse = np.zeros((Lyr, len(candidates)), dtype=np.float64)
    for layer in range(Lyr):
        ref = attention(q[layer], k[layer], v[layer], causal)
        for ci, s in enumerate(candidates):
            codes, n16 = write(k[layer], s, bits)
            khat = dequantize(codes, n16, s, bits, d)
            out = attention(q[layer], khat, v[layer], causal)
            mse[layer, ci] = np.mean((out - ref) ** 2)
    return mse, np.argmin(mse, axis=1)


# ---------------------------------------------------------------------------------------------------------------
# The per-query multiplication count (Key Points, 2nd item: a 102.4x reduction stated as an identity).
# ---------------------------------------------------------------------------------------------------------------

def multiplication_counts(d, bits, T):
    """(conventional, table) multiplications for one query over T keys.

    Reading (no formula is printed): a dense score costs d products per key; the table costs d * 2^b products to
    build plus one norm product per key.
    """
    return d * T, d * (1 << bits) + T
