"""Plain CPU oracle for the power-of-two (PoT) shift-accumulate key codec and its integer-log2 softmax.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py`` (its CPU baseline and reference arm) may import it; the product path never does, and the two share no
code.

Source: the arxivdaily page of the shift-accumulate attention paper (its English abstract).  The key cache is
quantized to signed power-of-two fixed-point codes, so that every product in QK^T is a sign flip, a shift and an
integer accumulation; a fixed-point head-room F >= e_max makes every shift a non-negative left shift and the
accumulation exact; a sub-power mantissa term adds one shift-add; the online softmax keeps its running maximum in
an integer log2 domain so every rescaling is an exact shift; and the attention-value product is log-quantized.  The
page prints no formulas.  The plainest reading, taken here:

* Key codec, per token: alpha = max_j |k_j| (exact in fp16 for fp16 keys, stored as fp16); u_j = k_j / alpha in
  fp32; the magnitude levels are 2^-e (1 + mu / 2^M) for e in [0, 2^E - 1] and mu in [0, 2^M - 1] (E exponent bits,
  M mantissa bits); |u_j| goes to the nearest level in linear value (a value on a midpoint between two levels goes
  up), its sign to a sign bit (u_j < 0 is negative).  The code of a coordinate is sign << (E + M) | l, l the
  level's rank from the smallest (l = (e_max - e) 2^M + mu, e_max = 2^E - 1): 1 + E + M bits, packed LSB-first like
  the AXELRAM codes.
* Query: fixed point, Q_j = rint(q_j / s_q) with s_q = max_j |q_j| / 32767 (fp32; Q = 0 when q = 0).
* Score: with F = e_max + M, S = sum_j sigma_j (Q_j 2^(F - e_j) + mu_j Q_j 2^(F - e_j - M)), an exact integer
  (the sign flip, the shifts and the integer sum), and the real score is s_q alpha 2^-F S.
* Softmax: w_t = float(S) * (s_q * mult * alpha_t) * 2^-F in fp32 with mult = fp32(scale) * fp32(log2 e) (the
  kernel's order), r_t = rint(w_t) an integer; the weights are 2^(r_t - R), R = max_t r_t (exact powers of two: the
  log-quantized product), and out = sum_t 2^(r_t - R) v_t / sum_t 2^(r_t - R).

Floating point decides integers at three places -- the key's level index, the query's Q_j and the exponent r_t --
and there the oracle uses the kernel's fp32 operations in the kernel's order (numpy float32 arithmetic rounds each
operation to nearest, like the kernel's explicit round-to-nearest operations).  Everything after the integers is
fp64.

Pins (tests/test_oracle_pot.py): the level decision against a brute-force nearest level; the relative-error bounds
of nearest power-of-two rounding (1/3 without mantissa, 1/5 with one mantissa bit); the shift-accumulated integer
against the exact integer dot product and, times its scale factors, against the fp64 dot product of the dequantized
query and key; the online softmax with an integer running maximum against the two-pass definition; special cases.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "pot_levels",
    "pot_thresholds",
    "pot_encode",
    "pot_decode",
    "pot_quantize_query",
    "pot_mult",
    "pot_score_int",
    "pot_score",
    "pot_exponents",
    "pot_attention",
    "pot_attention_online",
]

LOG2E = 1.4426950408889634


def pot_levels(E, M):
    """Magnitude levels 2^-e (1 + mu / 2^M), ascending (rank l = (e_max - e) 2^M + mu), f64."""
    e_max = (1 << E) - 1
    out = []
    for l in range(1 << (E + M)):
        e = e_max - (l >> M)
        mu = l & ((1 << M) - 1)
        out.append(2.0 ** -e * (1.0 + mu / (1 << M)))
    return np.array(out, dtype=np.float64)


def pot_thresholds(E, M):
    """Midpoints between consecutive levels, exact dyadic numbers (fp32 holds them exactly)."""
    lv = pot_levels(E, M)
    return ((lv[:-1] + lv[1:]) / 2).astype(np.float32)


def pot_encode(k, E, M):
    """Key rows k [..., d] (fp16) -> (codes int64 [..., d] = sign << (E+M) | rank, alpha fp16 [...]).

    alpha = max |k_j| (exact); u = k / alpha in fp32 (0 when alpha = 0); rank = number of midpoints <= |u|."""
    k = np.asarray(k)
    if k.dtype != np.float16:
        raise ValueError("the PoT codec takes fp16 keys (alpha is stored exactly as fp16)")
    k32 = k.astype(np.float32)
    alpha = np.max(np.abs(k32), axis=-1)
    safe = np.where(alpha > 0, alpha, np.float32(1)).astype(np.float32)
    u = np.where(alpha[..., None] > 0, np.divide(k32, safe[..., None], dtype=np.float32), np.float32(0))
    mag = np.abs(u)
    rank = np.sum(mag[..., None] >= pot_thresholds(E, M), axis=-1).astype(np.int64)
    sign = (u < 0).astype(np.int64)
    return (sign << (E + M)) | rank, alpha.astype(np.float16)


def pot_decode(codes, alpha, E, M):
    """Dequantized keys alpha * (-1)^sign * level[rank], f64."""
    codes = np.asarray(codes)
    lv = pot_levels(E, M)
    rank = codes & ((1 << (E + M)) - 1)
    sign = np.where((codes >> (E + M)) & 1, -1.0, 1.0)
    return np.asarray(alpha, dtype=np.float64)[..., None] * sign * lv[rank]


def pot_quantize_query(q):
    """(Q int64 [..., d], s_q f32 [...]): s_q = max|q| / 32767 in fp32, Q = rint(q / s_q) in fp32 (0 if q = 0)."""
    q32 = np.asarray(q, dtype=np.float32)
    s = np.divide(np.max(np.abs(q32), axis=-1), np.float32(32767), dtype=np.float32)
    safe = np.where(s > 0, s, np.float32(1)).astype(np.float32)
    Q = np.where(s[..., None] > 0, np.rint(np.divide(q32, safe[..., None], dtype=np.float32)), np.float32(0))
    return Q.astype(np.int64), s


def pot_mult(scale):
    """The fp32 factor scale * log2(e) (each operand rounded to fp32, the product rounded to fp32)."""
    return np.float32(np.float32(scale) * np.float32(LOG2E))


def pot_score_int(Q, codes, E, M):
    """S = sum_j sigma_j ((Q_j << (F - e_j)) + mu_j (Q_j << (F - e_j - M))), F = e_max + M, with Python-exact
    integers: the shift-accumulate form.  Q [d]; codes [T, d] -> int64 [T]."""
    e_max = (1 << E) - 1
    F = e_max + M
    codes = np.asarray(codes, dtype=np.int64)
    rank = codes & ((1 << (E + M)) - 1)
    neg = (codes >> (E + M)) & 1
    e = e_max - (rank >> M)
    mu = rank & ((1 << M) - 1)
    Qa = np.abs(np.asarray(Q, dtype=np.int64))
    Qs = np.sign(np.asarray(Q, dtype=np.int64))
    mag = (Qa[None, :] << (F - e)) + mu * (Qa[None, :] << np.maximum(F - e - M, 0))
    sgn = Qs[None, :] * np.where(neg == 1, -1, 1)  # the sign flip
    return np.sum(sgn * mag, axis=-1)


def pot_score(q, codes, alpha, E, M, scale=1.0):
    """Real scores scale * s_q * alpha_t * 2^-F * S_t (f64) of one query q [d] against codes [T, d]."""
    Q, s = pot_quantize_query(q)
    S = pot_score_int(Q, codes, E, M)
    F = (1 << E) - 1 + M
    return scale * float(s) * np.asarray(alpha, dtype=np.float64) * 2.0 ** -F * S.astype(np.float64)


def pot_exponents(q, codes, alpha, E, M, scale):
    """The integer log2 weights r_t = rint(w_t), w_t = float(S_t) * (s_q * mult * alpha_t) * 2^-F in fp32."""
    Q, s = pot_quantize_query(q)
    S = pot_score_int(Q, codes, E, M)
    F = (1 << E) - 1 + M
    c = np.multiply(np.multiply(s, pot_mult(scale), dtype=np.float32), np.asarray(alpha, np.float32),
                    dtype=np.float32)
    w = np.multiply(S.astype(np.float32), c, dtype=np.float32)
    w = np.multiply(w, np.float32(2.0 ** -F), dtype=np.float32)
    return np.rint(w).astype(np.int64)


def pot_attention(q, codes, alpha, v, E, M, scale, seq_lens=None):
    """Decode attention with PoT keys and log-quantized weights.  q [B, Hq, d]; codes [B, Hkv, Tc, d]; alpha
    [B, Hkv, Tc]; v [B, Hkv, Tc, d] fp16.  out = sum_t 2^(r_t - R) v_t / sum_t 2^(r_t - R) (two passes: R, then the
    sums), 0 for an empty row.  f64 [B, Hq, d]."""
    q = np.asarray(q)
    B, Hq, d = q.shape
    Hkv, Tc = codes.shape[1], codes.shape[2]
    G = Hq // Hkv
    lens = [Tc] * B if seq_lens is None else [int(n) for n in seq_lens]
    out = np.zeros((B, Hq, d))
    for b in range(B):
        T = lens[b]
        if T == 0:
            continue
        for hk in range(Hkv):
            vals = np.asarray(v[b, hk, :T], dtype=np.float64)
            for g in range(G):
                h = hk * G + g
                r = pot_exponents(q[b, h], codes[b, hk, :T], alpha[b, hk, :T], E, M, scale)
                p = np.ldexp(1.0, r - r.max())
                out[b, h] = (p[:, None] * vals).sum(axis=0) / p.sum()
    return out


def pot_attention_online(r, v, chunk):
    """The same weighted mean streamed in chunks with a running integer maximum R (log2 domain): on a new maximum
    the running sums are rescaled by 2^(R_old - R_new), an exact power of two.  r [T] int; v [T, d]."""
    R = None
    l = 0.0
    o = np.zeros(v.shape[-1])
    for t0 in range(0, len(r), chunk):
        rc = np.asarray(r[t0:t0 + chunk])
        Rn = int(rc.max()) if R is None else max(R, int(rc.max()))
        if R is not None:
            f = math.ldexp(1.0, R - Rn)
            l *= f
            o = o * f
        R = Rn
        p = np.ldexp(1.0, rc - R)
        l += p.sum()
        o = o + (p[:, None] * np.asarray(v[t0:t0 + chunk], dtype=np.float64)).sum(axis=0)
    return o / l
