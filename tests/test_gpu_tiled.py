"""GPU parity of the tiled value layout and the tensor-core value product.

* axr_write_values_tiled against the oracle's write path (the tiles are re-read into rows on the host);
* its scattered form (dst_rows, used to append a token) against the whole-tile form, byte for byte;
* axr_attend_decode with tiled values (AXR_V_QUANT_TILED) against the oracle's decode attention on the oracle's own
  codes, over several tiles, several splits and ragged lengths, and at the long-context size in the benchmark's
  launch configuration on sampled (batch, head) outputs."""

import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantized_b200 import ops
from kv_cache_quantized_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

TILE = 128


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def tiles_to_indices(codes_t, bits):
    """Tiled codes [B, Hkv, NT, d, 16 b] -> indices [B, Hkv, NT * 128, d] (token o at bits [o b, o b + b))."""
    c = np.asarray(codes_t)
    B, Hkv, NT, d, _ = c.shape
    bit = np.unpackbits(c, axis=-1, bitorder="little").reshape(B, Hkv, NT, d, TILE, bits).astype(np.int64)
    idx = (bit << np.arange(bits)).sum(-1)
    return np.moveaxis(idx, -1, -2).reshape(B, Hkv, NT * TILE, d)


def indices_to_tiles(idx, bits):
    """Indices [B, Hkv, Tcap, d] -> tiled codes [B, Hkv, Tcap / 128, d, 16 b]."""
    B, Hkv, Tcap, d = idx.shape
    t = np.moveaxis(np.asarray(idx, np.int64).reshape(B, Hkv, Tcap // TILE, TILE, d), -1, -2)
    bit = ((t[..., None] >> np.arange(bits)) & 1).astype(np.uint8)
    return np.packbits(bit.reshape(B, Hkv, Tcap // TILE, d, TILE * bits), axis=-1, bitorder="little")


def test_tile_helpers_round_trip():
    rng = np.random.default_rng(3)
    for bits in (1, 2, 3, 4):
        idx = rng.integers(0, 1 << bits, size=(2, 1, 256, 128))
        assert np.array_equal(tiles_to_indices(indices_to_tiles(idx, bits), bits), idx)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_write_tiled_matches_oracle(bits, dtype):
    B, Hkv, Tcap, d = 2, 2, 384, 128
    x = W.lognormal_rows((B, Hkv, Tcap, d), 40 + bits, dtype=dtype)
    s = W.sign_vector(d, 41)
    codes, norms = ops.write_values_tiled(cuda(x), cuda(s), bits)
    idx = tiles_to_indices(codes.cpu().numpy(), bits)
    parity.check_indices(oracle.pack(idx, bits), x, s, d, bits)
    parity.check_norms(norms.cpu().numpy(), x)


@pytest.mark.parametrize("bits", [3, 4])
def test_write_tiled_scatter_matches_whole_tiles(bits):
    B, Hkv, Tcap, d = 2, 2, 256, 128
    x = W.normal((B, Hkv, Tcap, d), 50, np.float16)
    s = cuda(W.sign_vector(d, 51))
    whole, wn = ops.write_values_tiled(cuda(x), s, bits)
    # every token written one by one (random order) into a buffer full of garbage
    rng = np.random.default_rng(52)
    codes = torch.from_numpy(rng.integers(0, 256, size=whole.shape, dtype=np.uint8)).cuda()
    norms = torch.zeros_like(wn)
    rows = rng.permutation(B * Hkv * Tcap)
    xr = x.reshape(-1, d)[rows]
    ops.write_values_tiled(cuda(xr), s, bits, codes=codes, norms=norms, dst_rows=cuda(rows.astype(np.int64)))
    assert torch.equal(codes, whole)
    assert torch.equal(norms.view(torch.int16), wn.view(torch.int16))
    # appending: one new token per (batch, KV head) replaces exactly its own codes
    t = 200
    xn = W.normal((B, Hkv, d), 53, np.float16)
    dst = (np.arange(B * Hkv) * Tcap + t).astype(np.int64)
    ops.write_values_tiled(cuda(xn.reshape(-1, d)), s, bits, codes=codes, norms=norms, dst_rows=cuda(dst))
    x2 = x.copy()
    x2[:, :, t] = xn
    want, wn2 = ops.write_values_tiled(cuda(x2), s, bits)
    assert torch.equal(codes, want)
    assert torch.equal(norms.view(torch.int16), wn2.view(torch.int16))


def tiled_case(B, Hkv, T, Tcap, d, bits, seed, G):
    k = W.lognormal_rows((B, Hkv, T, d), seed, dtype=np.float16)
    v = W.lognormal_rows((B, Hkv, T, d), seed + 1, dtype=np.float16)
    s = W.sign_vector(d, seed + 2)
    kc, kn = oracle.write(k, s, bits)
    vidx, _, vn, _ = oracle.quantize_rows(v, s, bits)
    vc = oracle.pack(vidx, bits)
    pad = lambda a, fill=0: np.pad(a, [(0, 0), (0, 0), (0, Tcap - T)] + [(0, 0)] * (a.ndim - 3),
                                   constant_values=fill)
    vt = indices_to_tiles(pad(vidx), bits)
    q = W.normal((B, Hkv * G, d), seed + 3, np.float32)
    return q, s, kc, kn, vc, vn, pad(kc), pad(kn), vt, pad(vn)


CASES = [(b, g) for b in (1, 2, 3, 4) for g in (4,)] + [(4, 1), (4, 2), (4, 8), (3, 8), (2, 1)]


@pytest.mark.parametrize("bits,G", CASES)
def test_attend_tiled_matches_oracle(bits, G):
    B, Hkv, T, Tcap, d = 2, 2, 2500, 2560, 128
    q, s, kc, kn, vc, vn, kcp, knp, vt, vnp = tiled_case(B, Hkv, T, Tcap, d, bits, 700 + 10 * bits + G, G)
    lens = np.array([T, 777], np.int32)
    scale = 1.0 / math.sqrt(d)
    out = ops.attend_decode(cuda(q), cuda(kcp), cuda(knp), cuda(s), bits, vcodes=cuda(vt), vnorms=cuda(vnp),
                            seq_lens=cuda(lens), T=T, scale=scale).cpu().numpy()
    want = oracle.decode_attention(q, kc, kn, s, bits, scale, vcodes=vc, vn16=vn, seq_lens=lens)
    parity.check_outputs(out, want)


def test_attend_tiled_edge_cases():
    d, bits, Hkv, G = 128, 4, 2, 4
    B, T, Tcap = 5, 300, 384
    q, s, kc, kn, vc, vn, kcp, knp, vt, vnp = tiled_case(B, Hkv, T, Tcap, d, bits, 900, G)
    q[3] = 0.0  # zero query: uniform weights
    lens = np.array([1, 0, 300, 129, 128], np.int32)
    args = dict(vcodes=cuda(vt), vnorms=cuda(vnp), T=T)
    out = ops.attend_decode(cuda(q), cuda(kcp), cuda(knp), cuda(s), bits, seq_lens=cuda(lens), **args).cpu().numpy()
    want = oracle.decode_attention(q, kc, kn, s, bits, 1 / math.sqrt(d), vcodes=vc, vn16=vn, seq_lens=lens)
    parity.check_outputs(out, want)
    assert np.all(out[1] == 0.0)  # empty row
    # the same rows through the row-layout kernel agree to fp16-rounding noise of the value centroids
    rows = ops.attend_decode(cuda(q), cuda(kcp), cuda(knp), cuda(s), bits, vcodes=cuda(np.pad(
        vc, [(0, 0), (0, 0), (0, Tcap - T), (0, 0)])), vnorms=cuda(vnp), seq_lens=cuda(lens), T=T).cpu().numpy()
    parity.check_outputs(out, rows.astype(np.float64))


def test_attend_tiled_split_invariance():
    """B = 1 (many splits) and B = 8 (fewer splits) give the same row up to the rounding of the fp16 weights
    p * n^V (each split rounds its weights against its own running maximum): unit roundoff 2^-11, so a row may move
    by a few 1e-4 of its norm, well inside the 2e-3 parity bound."""
    d, bits, Hkv, G, T = 128, 4, 8, 4, 32768
    dev = torch.device("cuda")
    k = W.lognormal_rows_device((8, Hkv, T, d), 910, dev)
    v = W.lognormal_rows_device((8, Hkv, T, d), 911, dev)
    s = cuda(W.sign_vector(d, 912))
    q = cuda(W.normal((8, Hkv * G, d), 913, np.float32))
    kc, kn = ops.write_keys(k, s, bits)
    vt, vn = ops.write_values_tiled(v, s, bits)
    full = ops.attend_decode(q, kc, kn, s, bits, vcodes=vt, vnorms=vn)
    one = ops.attend_decode(q[:1].contiguous(), kc[:1].contiguous(), kn[:1].contiguous(), s, bits,
                            vcodes=vt[:1].contiguous(), vnorms=vn[:1].contiguous())
    a, b = full[0].cpu().numpy().astype(np.float64), one[0].cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(a - b, axis=-1) / np.linalg.norm(a, axis=-1)
    assert rel.max() <= 2.0 ** -11


def test_long_context_tiled_full_size():
    """The long-context workload (B = 8, T = 32768, K and V at b = 4) as the benchmark runs it: cache written on the
    GPU (keys in rows, values tiled), attention on the GPU; sampled outputs recomputed by the oracle."""
    w = W.LONG_CONTEXT
    inp = W.decode_inputs(w)
    k, v, q, s = inp["k"], inp["v"], inp["q"], inp["signs"]
    st = cuda(s)
    kc, kn = ops.write_keys(cuda(k), st, w.bits)
    vt, vn = ops.write_values_tiled(cuda(v), st, w.bits)
    out = ops.attend_decode(cuda(q), kc, kn, st, w.bits, vcodes=vt, vnorms=vn).cpu().numpy()
    vt_h = vt.cpu().numpy()
    scale = 1.0 / math.sqrt(w.d)
    for b, h in [(0, 1), (4, 17), (7, 31)]:
        hk = h // w.G
        parity.check_indices(oracle.pack(tiles_to_indices(vt_h[b:b + 1, hk:hk + 1], w.bits)[0, 0], w.bits),
                             v[b, hk], s, w.d, w.bits)
        okc, okn = oracle.write(k[b, hk], s, w.bits)
        ovc, ovn = oracle.write(v[b, hk], s, w.bits)
        want = oracle.decode_attention(q[b:b + 1, h:h + 1], okc[None, None], okn[None, None], s, w.bits, scale,
                                       vcodes=ovc[None, None], vn16=ovn[None, None])
        parity.check_outputs(out[b:b + 1, h:h + 1], want)
