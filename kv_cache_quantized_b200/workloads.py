"""Seeded synthetic inputs shaped like the decode workloads the AXELRAM pages discuss.

This module holds no arithmetic of the method (no transform, codebook, quantizer or attention): it only draws
random tensors.  Both the CUDA path and the fp64 oracle are fed from it, so they see the same bytes.

Distributions (the pages give none; these are the stated synthetic stand-ins):
  * keys: i.i.d. N(0,1) per coordinate, times one lognormal(0, 0.5) factor per token (per row), or with a few
    seeded "outlier" channels scaled x10 (the same channels for every head), or times a per-layer factor
    10^U(-1,1) (layer-wise norm heterogeneity, AXELRAM Abstract);
  * queries and values: i.i.d. N(0,1);
  * sign vectors: i.i.d. uniform +-1 as int8.

Host generators use numpy PCG64 (``seed`` fixes every byte).  ``*_device`` variants draw the same distributions
with a seeded torch CUDA generator, for benchmark-size tensors that the oracle only samples.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BASE_SEED = 20260403


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def sign_vector(d: int, seed: int) -> np.ndarray:
    """One +-1 sign vector [d] int8."""
    return np.where(rng(seed).random(d) < 0.5, -1, 1).astype(np.int8)


def candidate_signs(n: int, d: int, seed: int) -> np.ndarray:
    """n candidate sign vectors [n, d] int8."""
    return np.where(rng(seed).random((n, d)) < 0.5, -1, 1).astype(np.int8)


def all_sign_vectors(d: int) -> np.ndarray:
    """Every +-1 vector of length d (2^d rows), row i having -1 where bit j of i is set."""
    i = np.arange(1 << d)[:, None]
    j = np.arange(d)[None, :]
    return np.where((i >> j) & 1, -1, 1).astype(np.int8)


def normal(shape, seed: int, dtype=np.float32) -> np.ndarray:
    return rng(seed).standard_normal(shape).astype(dtype)


def lognormal_rows(shape, seed: int, sigma: float = 0.5, dtype=np.float32) -> np.ndarray:
    """N(0,1) entries, each row (last axis) times exp(N(0, sigma))."""
    g = rng(seed)
    x = g.standard_normal(shape)
    f = np.exp(sigma * g.standard_normal(shape[:-1]))
    return (x * f[..., None]).astype(dtype)


def outlier_channels(d: int, n: int, seed: int) -> np.ndarray:
    """n distinct channel indices out of d."""
    return np.sort(rng(seed).choice(d, size=n, replace=False))


def outlier_keys(shape, seed: int, n_outliers: int = 4, factor: float = 10.0, dtype=np.float16) -> np.ndarray:
    """N(0,1) keys with n_outliers seeded channels (shared by every head and token) scaled by factor."""
    x = rng(seed).standard_normal(shape)
    ch = outlier_channels(shape[-1], n_outliers, seed + 7919)
    x[..., ch] *= factor
    return x.astype(dtype)


def layer_scaled_keys(shape, seed: int, dtype=np.float16) -> np.ndarray:
    """Keys [Lyr, ...]: N(0,1) times a per-layer factor 10^U(-1,1) (log-uniform over [0.1, 10])."""
    g = rng(seed)
    x = g.standard_normal(shape)
    f = 10.0 ** g.uniform(-1.0, 1.0, size=shape[0])
    return (x * f.reshape((-1,) + (1,) * (len(shape) - 1))).astype(dtype)


def outlier_direction_keys(shape, seed: int, pattern_seed: int, n_out: int = 8, m: float = 4.0,
                           layer_scale: bool = True, dtype=np.float16) -> np.ndarray:
    """Keys [Lyr, S, Hkv, N, d] with structure the sign pattern can see: N(0,1) noise plus a per-token multiple of a
    fixed outlier direction, x_t = z_t + a_t mu, a_t ~ N(0,1), where mu (one per layer and KV head) is +-m on n_out
    channels with fixed signs and 0 elsewhere (outlier channels with fixed sign relations), the whole layer times
    10^U(-1,1) if layer_scale (layer-wise norm heterogeneity).  The outlier patterns and layer factors come from
    pattern_seed alone, so calibration and held-out sets drawn with different `seed` share them.  Under the
    transform mu becomes H(s * mu), and the sign pattern decides whether that varying direction lands on a few
    coordinates (clipped by the codebook) or spreads over many."""
    g = rng(seed)
    gp = rng(pattern_seed)
    Lyr, S, Hkv, N, d = shape
    x = g.standard_normal(shape)
    a = g.standard_normal((Lyr, S, Hkv, N))
    nb = min(n_out, d)
    for layer in range(Lyr):
        for h in range(Hkv):
            ch = gp.choice(d, size=nb, replace=False)
            mu = np.zeros(d)
            mu[ch] = m * np.where(gp.random(nb) < 0.5, -1.0, 1.0)
            x[layer, :, h] += a[layer, :, h, :, None] * mu
    if layer_scale:
        f = 10.0 ** gp.uniform(-1.0, 1.0, size=Lyr)
        x *= f.reshape((-1,) + (1,) * (len(shape) - 1))
    return x.astype(dtype)


# ---------------------------------------------------------------------------------------------------------------
# Named workloads.
# ---------------------------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class Decode:
    """One decode step over a KV cache: one query per (batch row, query head)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    d: int
    bits: int
    v_quant: bool
    keys: str  # "lognormal" | "outlier"
    seed: int
    k_fp32: bool = False  # keys handed to the write path as fp32 instead of fp16

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


SINGLE_HEAD = Decode("single_head_d128_b2_t1024", 1, 1, 1, 1024, 128, 2, False, "lognormal", BASE_SEED + 1,
                     k_fp32=True)
LLAMA8B_DECODE = Decode("llama8b_decode_b8_t8192_hq32_hkv8_d128_b4_v16", 8, 32, 8, 8192, 128, 4, False, "outlier",
                        BASE_SEED + 2)
LONG_CONTEXT = Decode("long_context_b8_t32768_hq32_hkv8_d128_b4_kvquant", 8, 32, 8, 32768, 128, 4, True,
                      "lognormal", BASE_SEED + 4)


def sweep_case(B: int, T: int, bits: int, d: int) -> Decode:
    """One row of the decode sweep: Hq=32, Hkv=8, fp16 V, lognormal keys and values."""
    return Decode(f"sweep_b{B}_t{T}_b{bits}_d{d}", B, 32, 8, T, d, bits, False, "lognormal",
                  BASE_SEED + 5 + 1000 * bits + 10 * d + B + T)


SWEEP = [sweep_case(B, T, b, d) for B in (1, 8, 64) for T in (4096, 32768, 131072) for b in (1, 2, 3, 4)
         for d in (64, 128)]


@dataclass(frozen=True)
class Calibration:
    """Sign-selection calibration set: per-layer Q/K/V of a few sequences."""
    name: str
    layers: int
    seqs: int
    tokens: int
    Hq: int
    Hkv: int
    d: int
    bits: tuple
    n_cand: int
    seed: int


QWEN3B_SELECT = Calibration("qwen3b_select_l36_s8_n512_hq16_hkv2_d128", 36, 8, 512, 16, 2, 128, (2, 3, 4), 200,
                            BASE_SEED + 3)


def decode_inputs(w: Decode, T: int | None = None, B: int | None = None):
    """Host tensors of a decode workload (optionally truncated to B rows and T tokens).

    Returns dict with q [B,Hq,d] f32, k [B,Hkv,T,d] (f32 for the single-head case, else f16), v [B,Hkv,T,d] f16,
    signs [d] int8.
    """
    B = w.B if B is None else B
    T = w.T if T is None else T
    kshape = (B, w.Hkv, T, w.d)
    if w.keys == "outlier":
        k = outlier_keys(kshape, w.seed)
    else:
        k = lognormal_rows(kshape, w.seed, dtype=np.float32 if w.k_fp32 else np.float16)
    if w.v_quant:
        v = lognormal_rows(kshape, w.seed + 2, dtype=np.float16)
    else:
        v = normal(kshape, w.seed + 2, dtype=np.float16)
    q = normal((B, w.Hq, w.d), w.seed + 3, dtype=np.float32)
    return {"q": q, "k": k, "v": v, "signs": sign_vector(w.d, w.seed + 4)}


def calibration_inputs(c: Calibration, layers: int | None = None, seqs: int | None = None,
                       tokens: int | None = None, n_cand: int | None = None, keys: str = "layer_scaled"):
    """Host tensors of a calibration set (optionally reduced).  q f32, k/v f16, candidates int8.  keys:
    "layer_scaled" (i.i.d. N(0,1) times the per-layer factor) or "outlier_direction" (outlier_direction_keys)."""
    Lyr = c.layers if layers is None else layers
    S = c.seqs if seqs is None else seqs
    N = c.tokens if tokens is None else tokens
    C = c.n_cand if n_cand is None else n_cand
    q = normal((Lyr, S, c.Hq, N, c.d), c.seed, dtype=np.float32)
    if keys == "outlier_direction":
        k = outlier_direction_keys((Lyr, S, c.Hkv, N, c.d), c.seed + 1, c.seed + 5)
    else:
        k = layer_scaled_keys((Lyr, S, c.Hkv, N, c.d), c.seed + 1)
    v = normal((Lyr, S, c.Hkv, N, c.d), c.seed + 2, dtype=np.float16)
    return {"q": q, "k": k, "v": v, "candidates": candidate_signs(C, c.d, c.seed + 3)}


# ---------------------------------------------------------------------------------------------------------------
# Device generators for benchmark-size tensors (torch is plumbing here).
# ---------------------------------------------------------------------------------------------------------------

def _torch_gen(seed: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def lognormal_rows_device(shape, seed: int, device, sigma: float = 0.5, dtype=None):
    import torch
    dtype = torch.float16 if dtype is None else dtype
    g = _torch_gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    f = torch.exp(sigma * torch.randn(shape[:-1], generator=g, device=device, dtype=torch.float32))
    return (x * f.unsqueeze(-1)).to(dtype)


def normal_device(shape, seed: int, device, dtype=None):
    import torch
    dtype = torch.float16 if dtype is None else dtype
    g = _torch_gen(seed, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def outlier_keys_device(shape, seed: int, device, n_outliers: int = 4, factor: float = 10.0, dtype=None):
    import torch
    dtype = torch.float16 if dtype is None else dtype
    g = _torch_gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    ch = torch.as_tensor(outlier_channels(shape[-1], n_outliers, seed + 7919), device=device)
    x[..., ch] *= factor
    return x.to(dtype)


def layer_scaled_keys_device(shape, seed: int, device, dtype=None):
    """layer_scaled_keys' distribution drawn on the device: N(0,1) times a per-layer factor 10^U(-1,1)."""
    import torch
    dtype = torch.float16 if dtype is None else dtype
    g = _torch_gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    f = 10.0 ** (2.0 * torch.rand(shape[0], generator=g, device=device, dtype=torch.float32) - 1.0)
    return (x * f.view((-1,) + (1,) * (len(shape) - 1))).to(dtype)
