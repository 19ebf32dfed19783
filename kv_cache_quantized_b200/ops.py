"""Torch-tensor front end of libaxr: argument marshalling only.

Every function here checks devices, dtypes and shapes, passes raw device pointers and the current CUDA stream to
the C ABI (include/axr.h), and raises AxrError on a non-OK status.  All arithmetic runs in the library's kernels;
tensors on the CPU are rejected (there is no fallback).

Layouts (see include/axr.h): codes [B, Hkv, Tcap, d*b/8] uint8, norms [B, Hkv, Tcap] float16, values
[B, Hkv, Tcap, d] float16, q [B, Hq, d] float32.
"""

from __future__ import annotations

import ctypes
import math

import numpy as np
import torch

from . import _abi


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need_cuda(name: str, t: torch.Tensor, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libaxr has no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def row_bytes(d: int, bits: int) -> int:
    return d * bits // 8


def codebook(d: int, bits: int):
    """(centroids [2^b], thresholds [2^b - 1]) float64 numpy arrays from the library's host codebook."""
    L = 1 << bits
    c = np.zeros(L, dtype=np.float64)
    t = np.zeros(max(L - 1, 1), dtype=np.float64)
    st = _abi.lib().axr_codebook(d, bits, c.ctypes.data_as(ctypes.c_void_p), t.ctypes.data_as(ctypes.c_void_p))
    _abi.check(st, "axr_codebook")
    return c, t[: L - 1]


def write_keys(x: torch.Tensor, signs: torch.Tensor, bits: int, codes: torch.Tensor | None = None,
               norms: torch.Tensor | None = None, dst_rows: torch.Tensor | None = None):
    """Quantize rows of x [..., d] (float16 or float32).  Returns (codes uint8 [..., d*b/8], norms float16 [...]).

    With dst_rows (int64 [n_vec]) the rows land at those row indices of the given codes/norms buffers (e.g. a cache
    viewed as [B*Hkv*Tcap, R]); codes and norms are then required.
    """
    _need_cuda("x", x)
    _need_cuda("signs", signs, torch.int8)
    if x.dtype not in (torch.float16, torch.float32):
        raise TypeError("x must be float16 or float32")
    d = x.shape[-1]
    n_vec = x.numel() // d if d else 0
    R = row_bytes(d, bits)
    if dst_rows is None:
        if codes is None:
            codes = torch.empty(x.shape[:-1] + (R,), dtype=torch.uint8, device=x.device)
        if norms is None:
            norms = torch.empty(x.shape[:-1], dtype=torch.float16, device=x.device)
    else:
        _need_cuda("dst_rows", dst_rows, torch.int64)
        if codes is None or norms is None:
            raise ValueError("dst_rows needs the destination codes and norms buffers")
        if dst_rows.numel() != n_vec:
            raise ValueError("dst_rows must hold one row index per vector")
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("norms", norms, torch.float16)
    if dst_rows is None and (codes.numel() != n_vec * R or norms.numel() != n_vec):
        raise ValueError("codes/norms do not match x")
    dt = _abi.F16 if x.dtype == torch.float16 else _abi.F32
    st = _abi.lib().axr_write_keys(_ptr(x), dt, n_vec, d, bits, _ptr(signs), _ptr(dst_rows), _ptr(codes),
                                   _ptr(norms), _stream())
    _abi.check(st, "axr_write_keys")
    return codes, norms


TILE = 128  # tokens per tile of the tiled value layout


def tiled_shape(B, Hkv, Tcap, d, bits):
    """Shape of value codes in the tiled layout: [B, Hkv, Tcap/128, d, 16*b] uint8."""
    if Tcap % TILE:
        raise ValueError("the tiled layout needs Tcap to be a multiple of 128")
    return (B, Hkv, Tcap // TILE, d, TILE * bits // 8)


def write_values_tiled(x: torch.Tensor, signs: torch.Tensor, bits: int, codes: torch.Tensor | None = None,
                       norms: torch.Tensor | None = None, dst_rows: torch.Tensor | None = None, Tcap: int | None = None):
    """Quantize value vectors like write_keys, storing the codes tiled for the tensor-core value product.

    Without dst_rows x is the whole cache [B, Hkv, Tcap, d] (Tcap a multiple of 128) and (codes [B, Hkv, Tcap/128,
    d, 16*b], norms [B, Hkv, Tcap]) are returned.  With dst_rows (int64, rows (b*Hkv + h)*Tcap + t) the vectors x
    [n, d] are written into the given codes/norms in place.
    """
    _need_cuda("x", x)
    _need_cuda("signs", signs, torch.int8)
    if x.dtype not in (torch.float16, torch.float32):
        raise TypeError("x must be float16 or float32")
    d = x.shape[-1]
    n_vec = x.numel() // d if d else 0
    if dst_rows is None:
        if x.dim() != 4:
            raise ValueError("x must be [B, Hkv, Tcap, d] without dst_rows")
        B, Hkv, Tc, _ = x.shape
        Tcap = Tc
        if codes is None:
            codes = torch.empty(tiled_shape(B, Hkv, Tcap, d, bits), dtype=torch.uint8, device=x.device)
        if norms is None:
            norms = torch.empty((B, Hkv, Tcap), dtype=torch.float16, device=x.device)
    else:
        _need_cuda("dst_rows", dst_rows, torch.int64)
        if codes is None or norms is None:
            raise ValueError("dst_rows needs the destination codes and norms buffers")
        if dst_rows.numel() != n_vec:
            raise ValueError("dst_rows must hold one row index per vector")
        if codes.dim() != 5:
            raise ValueError("codes must be [B, Hkv, Tcap/128, d, 16*b]")
        Tcap = codes.shape[2] * TILE
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("norms", norms, torch.float16)
    dt = _abi.F16 if x.dtype == torch.float16 else _abi.F32
    st = _abi.lib().axr_write_values_tiled(_ptr(x), dt, n_vec, d, bits, _ptr(signs), _ptr(dst_rows), int(Tcap),
                                           _ptr(codes), _ptr(norms), _stream())
    _abi.check(st, "axr_write_values_tiled")
    return codes, norms


def _cache_dims(q, kcodes, knorms, d, bits, T):
    _need_cuda("q", q, torch.float32)
    _need_cuda("kcodes", kcodes, torch.uint8)
    _need_cuda("knorms", knorms, torch.float16)
    if q.dim() != 3 or kcodes.dim() != 4 or knorms.dim() != 3:
        raise ValueError("q [B,Hq,d], kcodes [B,Hkv,Tcap,R], knorms [B,Hkv,Tcap] expected")
    B, Hq, _ = q.shape
    _, Hkv, Tcap, R = kcodes.shape
    if R != row_bytes(d, bits) or kcodes.shape[0] != B or tuple(knorms.shape) != (B, Hkv, Tcap):
        raise ValueError("cache shapes do not match q, d and bits")
    T = Tcap if T is None else int(T)
    return B, Hq, Hkv, Tcap, T


def _lens(seq_lens, B):
    if seq_lens is None:
        return None
    _need_cuda("seq_lens", seq_lens, torch.int32)
    if seq_lens.numel() != B:
        raise ValueError("seq_lens must have B entries")
    return seq_lens


def score(q, kcodes, knorms, signs, bits, scale=1.0, seq_lens=None, T=None, out=None):
    """Scores [B, Hq, T] float32 = scale * norm_t * sum_j LUT[j][idx_{t,j}] (tokens >= seq_lens[b] get -inf)."""
    d = q.shape[-1]
    B, Hq, Hkv, Tcap, T = _cache_dims(q, kcodes, knorms, d, bits, T)
    _need_cuda("signs", signs, torch.int8)
    seq_lens = _lens(seq_lens, B)
    if out is None:
        out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    _need_cuda("out", out, torch.float32)
    st = _abi.lib().axr_score(_ptr(q), _ptr(kcodes), _ptr(knorms), _ptr(seq_lens), B, Hq, Hkv, T, Tcap, d, bits,
                              _ptr(signs), float(scale), _ptr(out), _stream())
    _abi.check(st, "axr_score")
    return out


GATHER_MODES = {"tensor": _abi.GATHER_TENSOR, "factored": _abi.GATHER_FACTORED, "table": _abi.GATHER_TABLE,
                "mma": _abi.GATHER_MMA, "direct": _abi.GATHER_DIRECT}


def set_gather(mode: str) -> None:
    """Table read mode of score(): "mma" (default: warp-level MMAs on hi/lo fp16 operands), "factored" (packed fp32
    FMAs), "tensor" (tcgen05 MMAs from tensor memory) or "table" (the materialised table, gathered per entry)."""
    _abi.check(_abi.lib().axr_set_gather(GATHER_MODES[mode]), "axr_set_gather")


def get_gather() -> str:
    code = _abi.lib().axr_get_gather()
    return {v: k for k, v in GATHER_MODES.items()}[code]


def attend_workspace_bytes(B, Hq, Hkv, T, d) -> int:
    return int(_abi.lib().axr_attend_workspace_bytes(B, Hq, Hkv, T, d))


def _workspace(nbytes, device, ws):
    if ws is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _need_cuda("workspace", ws, torch.uint8)
    return ws


def attend_decode(q, kcodes, knorms, signs, bits, v=None, vcodes=None, vnorms=None, scale=None, seq_lens=None,
                  T=None, out=None, workspace=None):
    """One decode step over a quantized key cache.  Values: v (float16 [B,Hkv,Tcap,d]) or vcodes/vnorms (quantized
    like the keys with the same signs, in the keys' row layout or -- 5-D -- in write_values_tiled's layout, which
    runs the value product on the tensor cores).  Returns out [B, Hq, d] float32."""
    d = q.shape[-1]
    B, Hq, Hkv, Tcap, T = _cache_dims(q, kcodes, knorms, d, bits, T)
    _need_cuda("signs", signs, torch.int8)
    seq_lens = _lens(seq_lens, B)
    if (v is None) == (vcodes is None):
        raise ValueError("pass exactly one of v or vcodes")
    if v is not None:
        _need_cuda("v", v, torch.float16)
        if tuple(v.shape) != (B, Hkv, Tcap, d):
            raise ValueError("v must be [B, Hkv, Tcap, d]")
        vkind, vptr, vnptr = _abi.V_F16, _ptr(v), None
    else:
        _need_cuda("vcodes", vcodes, torch.uint8)
        _need_cuda("vnorms", vnorms, torch.float16)
        if vnorms.shape != knorms.shape:
            raise ValueError("vnorms must have the key norms' shape")
        if vcodes.dim() == 5:  # tiled layout (write_values_tiled)
            if tuple(vcodes.shape) != tiled_shape(B, Hkv, Tcap, d, bits):
                raise ValueError("tiled vcodes must be [B, Hkv, Tcap/128, d, 16*b]")
            vkind = _abi.V_QUANT_TILED
        else:
            if vcodes.shape != kcodes.shape:
                raise ValueError("vcodes must have the key cache's shape")
            vkind = _abi.V_QUANT
        vptr, vnptr = _ptr(vcodes), _ptr(vnorms)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _need_cuda("out", out, torch.float32)
    nbytes = attend_workspace_bytes(B, Hq, Hkv, T, d)
    ws = _workspace(nbytes, q.device, workspace)
    st = _abi.lib().axr_attend_decode(_ptr(q), _ptr(kcodes), _ptr(knorms), vkind, vptr, vnptr, _ptr(seq_lens), B, Hq,
                                      Hkv, T, Tcap, d, bits, _ptr(signs), scale, _ptr(out), _ptr(ws), ws.numel(),
                                      _stream())
    _abi.check(st, "axr_attend_decode")
    return out


def decode_step(q, k_new, v_new, kcodes, knorms, signs, bits, v=None, vcodes=None, vnorms=None, scale=None,
                seq_lens=None, T=None, out=None, workspace=None):
    """One decode step in one launch: k_new, v_new (float16 [B, Hkv, d]) are written into the cache at position
    seq_lens[b] - 1 of each batch row (T - 1 without seq_lens) -- keys as codes and norms, values the same way
    (vcodes/vnorms) or as they are (v) -- and attention then runs over positions [0, seq_lens[b]).  Row value
    layouts only.  Returns out [B, Hq, d] float32; the cache tensors are updated in place."""
    d = q.shape[-1]
    B, Hq, Hkv, Tcap, T = _cache_dims(q, kcodes, knorms, d, bits, T)
    _need_cuda("signs", signs, torch.int8)
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _need_cuda(name, t, torch.float16)
        if tuple(t.shape) != (B, Hkv, d) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [B, Hkv, d] float16 tensor")
    seq_lens = _lens(seq_lens, B)
    if (v is None) == (vcodes is None):
        raise ValueError("pass exactly one of v or vcodes")
    if v is not None:
        _need_cuda("v", v, torch.float16)
        if tuple(v.shape) != (B, Hkv, Tcap, d):
            raise ValueError("v must be [B, Hkv, Tcap, d]")
        vkind, vptr, vnptr = _abi.V_F16, _ptr(v), None
    else:
        _need_cuda("vcodes", vcodes, torch.uint8)
        _need_cuda("vnorms", vnorms, torch.float16)
        if vcodes.shape != kcodes.shape or vnorms.shape != knorms.shape:
            raise ValueError("vcodes / vnorms must have the key cache's shapes (row layout)")
        vkind, vptr, vnptr = _abi.V_QUANT, _ptr(vcodes), _ptr(vnorms)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _need_cuda("out", out, torch.float32)
    nbytes = attend_workspace_bytes(B, Hq, Hkv, T, d)
    ws = _workspace(nbytes, q.device, workspace)
    st = _abi.lib().axr_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kcodes), _ptr(knorms), vkind, vptr, vnptr,
                                    _ptr(seq_lens), B, Hq, Hkv, T, Tcap, d, bits, _ptr(signs), scale, _ptr(out),
                                    _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_decode_step")
    return out


def dense_decode(q, k, v, scale=None, seq_lens=None, T=None, out=None, workspace=None):
    """Decode attention over an unquantized float16 K/V cache [B, Hkv, Tcap, d] (the bandwidth reference)."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("k", k, torch.float16)
    _need_cuda("v", v, torch.float16)
    B, Hq, d = q.shape
    _, Hkv, Tcap, _ = k.shape
    if tuple(v.shape) != tuple(k.shape) or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k, v must be [B, Hkv, Tcap, d]")
    T = Tcap if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    nbytes = attend_workspace_bytes(B, Hq, Hkv, T, d)
    ws = _workspace(nbytes, q.device, workspace)
    st = _abi.lib().axr_dense_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_lens), B, Hq, Hkv, T, Tcap, d, scale,
                                     _ptr(out), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_dense_decode")
    return out


def select_workspace_bytes(layers, seqs, tokens, Hq, Hkv, d, n_cand) -> int:
    return int(_abi.lib().axr_select_workspace_bytes(layers, seqs, tokens, Hq, Hkv, d, n_cand))


def select_signs(q, k, v, candidates, bits, causal=True, workspace=None):
    """Score candidate sign vectors [C, d] int8 on calibration q [Ly,S,Hq,N,d] f32, k/v [Ly,S,Hkv,N,d] f16.
    Returns (mse float64 [C], best int32 [1]) as CUDA tensors."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("k", k, torch.float16)
    _need_cuda("v", v, torch.float16)
    _need_cuda("candidates", candidates, torch.int8)
    Ly, S, Hq, N, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (Ly, S, Hkv, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k, v must be [Ly, S, Hkv, N, d]")
    C = candidates.shape[0]
    if tuple(candidates.shape) != (C, d):
        raise ValueError("candidates must be [C, d]")
    mse = torch.empty(C, dtype=torch.float64, device=q.device)
    best = torch.empty(1, dtype=torch.int32, device=q.device)
    nbytes = select_workspace_bytes(Ly, S, N, Hq, Hkv, d, C)
    ws = _workspace(nbytes, q.device, workspace)
    st = _abi.lib().axr_select_signs(_ptr(q), _ptr(k), _ptr(v), Ly, S, N, Hq, Hkv, d, bits, _ptr(candidates), C,
                                     1 if causal else 0, _ptr(mse), _ptr(best), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_select_signs")
    return mse, best


def select_signs_per_layer(q, k, v, candidates, bits, causal=True, parts=False, workspace=None):
    """One sign vector per layer: per-layer MSE of every candidate (the mean over that layer's sequences, heads,
    positions and coordinates) and each layer's first argmin.  Returns (mse [Ly, C] float64, best [Ly] int32) and,
    with parts, also the MSE of each (layer, sequence) [Ly, S, C] float64, as CUDA tensors."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("k", k, torch.float16)
    _need_cuda("v", v, torch.float16)
    _need_cuda("candidates", candidates, torch.int8)
    Ly, S, Hq, N, d = q.shape
    Hkv = k.shape[2]
    if tuple(k.shape) != (Ly, S, Hkv, N, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("k, v must be [Ly, S, Hkv, N, d]")
    C = candidates.shape[0]
    if tuple(candidates.shape) != (C, d):
        raise ValueError("candidates must be [C, d]")
    mse = torch.empty((Ly, C), dtype=torch.float64, device=q.device)
    best = torch.empty(Ly, dtype=torch.int32, device=q.device)
    mparts = torch.empty((Ly, S, C), dtype=torch.float64, device=q.device) if parts else None
    nbytes = select_workspace_bytes(Ly, S, N, Hq, Hkv, d, C)
    ws = _workspace(nbytes, q.device, workspace)
    st = _abi.lib().axr_select_signs_per_layer(_ptr(q), _ptr(k), _ptr(v), Ly, S, N, Hq, Hkv, d, bits,
                                               _ptr(candidates), C, 1 if causal else 0, _ptr(mse), _ptr(best),
                                               _ptr(mparts), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_select_signs_per_layer")
    return (mse, best, mparts) if parts else (mse, best)


def device_status(clear: bool = False) -> int:
    """The current device's status word (synchronizes the device): AXR_STATUS_WAIT_TIMEOUT (1) if a kernel's bounded
    wait gave up since the word was last cleared (its outputs hold NaN), else 0.  clear resets it."""
    flags = ctypes.c_uint(0)
    st = _abi.lib().axr_device_status(ctypes.byref(flags), 1 if clear else 0)
    if st not in (0, 3):
        _abi.check(st, "axr_device_status")
    if st == 3 and not (flags.value & _abi.STATUS_WAIT_TIMEOUT):
        _abi.check(st, "axr_device_status")
    return int(flags.value)


def _paged_dims(q, kcodes, knorms, block_table, bits):
    _need_cuda("q", q, torch.float32)
    _need_cuda("kcodes", kcodes, torch.uint8)
    _need_cuda("knorms", knorms, torch.float16)
    _need_cuda("block_table", block_table, torch.int32)
    if q.dim() != 3 or kcodes.dim() != 4 or knorms.dim() != 3 or block_table.dim() != 2:
        raise ValueError("q [B,Hq,d], kcodes [blocks,Hkv,bt,R], knorms [blocks,Hkv,bt], block_table [B,max_blocks]")
    B, Hq, d = q.shape
    nb, Hkv, bt, R = kcodes.shape
    if R != row_bytes(d, bits) or tuple(knorms.shape) != (nb, Hkv, bt) or block_table.shape[0] != B:
        raise ValueError("pool shapes do not match q, d, bits and the block table")
    return B, Hq, Hkv, d, bt, block_table.shape[1]


def _paged_values(v, vcodes, vnorms, kcodes, knorms, d):
    if (v is None) == (vcodes is None):
        raise ValueError("pass exactly one of v or vcodes")
    if v is not None:
        _need_cuda("v", v, torch.float16)
        if tuple(v.shape) != tuple(kcodes.shape[:3]) + (d,):
            raise ValueError("v must be [blocks, Hkv, bt, d]")
        return _abi.V_F16, _ptr(v), None
    _need_cuda("vcodes", vcodes, torch.uint8)
    _need_cuda("vnorms", vnorms, torch.float16)
    if vcodes.shape != kcodes.shape or vnorms.shape != knorms.shape:
        raise ValueError("vcodes / vnorms must have the key pools' shapes")
    return _abi.V_QUANT, _ptr(vcodes), _ptr(vnorms)


def attend_decode_paged(q, kcodes, knorms, signs, bits, block_table, seq_lens=None, T=None, v=None, vcodes=None,
                        vnorms=None, scale=None, out=None, workspace=None):
    """axr_attend_decode over paged pools: kcodes [blocks, Hkv, bt, R], knorms [blocks, Hkv, bt], values v [blocks,
    Hkv, bt, d] float16 or vcodes/vnorms shaped like the key pools; block_table [B, max_blocks] int32 maps logical
    block j of batch row b to its pool block.  T (default max_blocks * bt) bounds seq_lens.  Returns out [B, Hq, d]."""
    B, Hq, Hkv, d, bt, mb = _paged_dims(q, kcodes, knorms, block_table, bits)
    _need_cuda("signs", signs, torch.int8)
    T = mb * bt if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    vkind, vptr, vnptr = _paged_values(v, vcodes, vnorms, kcodes, knorms, d)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _need_cuda("out", out, torch.float32)
    ws = _workspace(attend_workspace_bytes(B, Hq, Hkv, T, d), q.device, workspace)
    st = _abi.lib().axr_attend_decode_paged(_ptr(q), _ptr(kcodes), _ptr(knorms), vkind, vptr, vnptr, _ptr(block_table),
                                            mb, bt, _ptr(seq_lens), B, Hq, Hkv, T, d, bits, _ptr(signs), scale,
                                            _ptr(out), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_attend_decode_paged")
    return out


def decode_step_paged(q, k_new, v_new, kcodes, knorms, signs, bits, block_table, seq_lens=None, T=None, v=None,
                      vcodes=None, vnorms=None, scale=None, out=None, workspace=None):
    """axr_decode_step over paged pools: k_new, v_new (float16 [B, Hkv, d]) are written at position seq_lens[b] - 1
    through the block table, then attention runs over [0, seq_lens[b]).  The pools are updated in place."""
    B, Hq, Hkv, d, bt, mb = _paged_dims(q, kcodes, knorms, block_table, bits)
    _need_cuda("signs", signs, torch.int8)
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _need_cuda(name, t, torch.float16)
        if tuple(t.shape) != (B, Hkv, d):
            raise ValueError(f"{name} must be a contiguous [B, Hkv, d] float16 tensor")
    T = mb * bt if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    vkind, vptr, vnptr = _paged_values(v, vcodes, vnorms, kcodes, knorms, d)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    _need_cuda("out", out, torch.float32)
    ws = _workspace(attend_workspace_bytes(B, Hq, Hkv, T, d), q.device, workspace)
    st = _abi.lib().axr_decode_step_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(kcodes), _ptr(knorms), vkind, vptr,
                                          vnptr, _ptr(block_table), mb, bt, _ptr(seq_lens), B, Hq, Hkv, T, d, bits,
                                          _ptr(signs), scale, _ptr(out), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_decode_step_paged")
    return out


# ---- LOOKAT product quantization ------------------------------------------------------------------------------------

def pq_train(x, codebooks, iters, workspace=None):
    """Lloyd k-means of one head's keys x [n, d] (float16/float32), per subspace, from the initial centroids in
    codebooks [m, K, d/m] float32, which are updated in place and returned."""
    _need_cuda("x", x)
    _need_cuda("codebooks", codebooks, torch.float32)
    if x.dtype not in (torch.float16, torch.float32):
        raise TypeError("x must be float16 or float32")
    m, K, ds = codebooks.shape
    d = x.shape[-1]
    if m * ds != d:
        raise ValueError("codebooks do not match d")
    n = x.numel() // d
    nbytes = int(_abi.lib().axr_pq_train_workspace_bytes(d, m, K))
    ws = _workspace(nbytes, x.device, workspace)
    dt = _abi.F16 if x.dtype == torch.float16 else _abi.F32
    st = _abi.lib().axr_pq_train(_ptr(x), dt, n, d, m, K, int(iters), _ptr(codebooks), _ptr(ws), ws.numel(),
                                 _stream())
    _abi.check(st, "axr_pq_train")
    return codebooks


def pq_encode(x, codebooks, head_period=None, codes=None, dst_rows=None):
    """Indices (uint8 [..., m]) of the nearest centroids of x [..., d]; codebooks [heads, m, K, d/m] float32, vector
    r using set (r / head_period) % heads (default head_period: x.shape[-2] for a [B, Hkv, T, d] cache, i.e. the
    head axis is x.shape[-3])."""
    _need_cuda("x", x)
    _need_cuda("codebooks", codebooks, torch.float32)
    if codebooks.dim() == 3:
        codebooks = codebooks.unsqueeze(0)
    H, m, K, ds = codebooks.shape
    d = x.shape[-1]
    n = x.numel() // d
    if head_period is None:
        head_period = x.shape[-2] if (H > 1 and x.dim() >= 3) else max(n, 1)
    if dst_rows is None:
        if codes is None:
            codes = torch.empty(x.shape[:-1] + (m,), dtype=torch.uint8, device=x.device)
    else:
        _need_cuda("dst_rows", dst_rows, torch.int64)
        if codes is None:
            raise ValueError("dst_rows needs the destination codes buffer")
    _need_cuda("codes", codes, torch.uint8)
    dt = _abi.F16 if x.dtype == torch.float16 else _abi.F32
    st = _abi.lib().axr_pq_encode(_ptr(x), dt, n, d, m, K, _ptr(codebooks), H, int(head_period), _ptr(dst_rows),
                                  _ptr(codes), _stream())
    _abi.check(st, "axr_pq_encode")
    return codes


def pq_score(q, codes, codebooks, scale=1.0, seq_lens=None, T=None, out=None):
    """ADC scores [B, Hq, T]: q [B, Hq, d] float32, codes [B, Hkv, Tcap, m] uint8, codebooks [Hkv, m, K, d/m]."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("codebooks", codebooks, torch.float32)
    B, Hq, d = q.shape
    _, Hkv, Tcap, m = codes.shape
    K = codebooks.shape[2]
    T = Tcap if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    if out is None:
        out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    st = _abi.lib().axr_pq_score(_ptr(q), _ptr(codes), _ptr(codebooks), _ptr(seq_lens), B, Hq, Hkv, T, Tcap, d, m, K,
                                 float(scale), _ptr(out), _stream())
    _abi.check(st, "axr_pq_score")
    return out


def pq_attend_decode(q, codes, codebooks, v, scale=None, seq_lens=None, T=None, out=None, workspace=None):
    """Decode attention over product-quantized keys and float16 values v [B, Hkv, Tcap, d]."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("codebooks", codebooks, torch.float32)
    _need_cuda("v", v, torch.float16)
    B, Hq, d = q.shape
    _, Hkv, Tcap, m = codes.shape
    K = codebooks.shape[2]
    T = Tcap if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    ws = _workspace(attend_workspace_bytes(B, Hq, Hkv, T, d), q.device, workspace)
    st = _abi.lib().axr_pq_attend_decode(_ptr(q), _ptr(codes), _ptr(codebooks), _ptr(v), _ptr(seq_lens), B, Hq, Hkv,
                                         T, Tcap, d, m, K, scale, _ptr(out), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_pq_attend_decode")
    return out


# ---- power-of-two shift-accumulate keys -------------------------------------------------------------------------------

def pot_row_bytes(d: int, E: int, M: int) -> int:
    return d * (1 + E + M) // 8


def pot_write(x, E, M, codes=None, alpha=None, dst_rows=None):
    """PoT codes of float16 rows x [..., d]: (codes uint8 [..., d(1+E+M)/8], alpha float16 [...])."""
    _need_cuda("x", x, torch.float16)
    d = x.shape[-1]
    n = x.numel() // d
    R = pot_row_bytes(d, E, M)
    if dst_rows is None:
        codes = torch.empty(x.shape[:-1] + (R,), dtype=torch.uint8, device=x.device) if codes is None else codes
        alpha = torch.empty(x.shape[:-1], dtype=torch.float16, device=x.device) if alpha is None else alpha
    else:
        _need_cuda("dst_rows", dst_rows, torch.int64)
        if codes is None or alpha is None:
            raise ValueError("dst_rows needs the destination codes and alpha buffers")
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("alpha", alpha, torch.float16)
    st = _abi.lib().axr_pot_write(_ptr(x), n, d, E, M, _ptr(dst_rows), _ptr(codes), _ptr(alpha), _stream())
    _abi.check(st, "axr_pot_write")
    return codes, alpha


def pot_score(q, codes, alpha, E, M, scale=1.0, seq_lens=None, T=None, integers=False):
    """PoT scores [B, Hq, T] float32 (and, with integers, the exact shift-accumulated int32 sums S as well)."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("alpha", alpha, torch.float16)
    B, Hq, d = q.shape
    _, Hkv, Tcap, _ = codes.shape
    T = Tcap if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    out = torch.empty((B, Hq, T), dtype=torch.float32, device=q.device)
    S = torch.empty((B, Hq, T), dtype=torch.int32, device=q.device) if integers else None
    st = _abi.lib().axr_pot_score(_ptr(q), _ptr(codes), _ptr(alpha), _ptr(seq_lens), B, Hq, Hkv, T, Tcap, d, E, M,
                                  float(scale), _ptr(S), _ptr(out), _stream())
    _abi.check(st, "axr_pot_score")
    return (out, S) if integers else out


def pot_attend_decode(q, codes, alpha, v, E, M, scale=None, seq_lens=None, T=None, out=None, workspace=None):
    """Decode attention over PoT keys (integer-log2 weights) and float16 values v [B, Hkv, Tcap, d]."""
    _need_cuda("q", q, torch.float32)
    _need_cuda("codes", codes, torch.uint8)
    _need_cuda("alpha", alpha, torch.float16)
    _need_cuda("v", v, torch.float16)
    B, Hq, d = q.shape
    _, Hkv, Tcap, _ = codes.shape
    T = Tcap if T is None else int(T)
    seq_lens = _lens(seq_lens, B)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    ws = _workspace(attend_workspace_bytes(B, Hq, Hkv, T, d), q.device, workspace)
    st = _abi.lib().axr_pot_attend_decode(_ptr(q), _ptr(codes), _ptr(alpha), _ptr(v), _ptr(seq_lens), B, Hq, Hkv, T,
                                          Tcap, d, E, M, scale, _ptr(out), _ptr(ws), ws.numel(), _stream())
    _abi.check(st, "axr_pot_attend_decode")
    return out
