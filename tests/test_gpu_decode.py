"""GPU parity of the read path: LUT scores (axr_score), split-T decode attention over fp16 or quantized values
(axr_attend_decode) and the dense fp16 reference (axr_dense_decode), against the oracle on the same inputs.

Small cases span several 256-token tiles, several splits and a ragged tail; the full-size workloads run in the
launch configuration the benchmark uses and are checked on sampled (batch, head) outputs."""

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


def padded(a, Tcap, axis=2, fill=0):
    pad = [(0, 0)] * a.ndim
    pad[axis] = (0, Tcap - a.shape[axis])
    return np.pad(a, pad, constant_values=fill)


def oracle_cache(B, Hkv, T, d, bits, seed, vq, keys="lognormal"):
    """Host inputs and oracle-written codes for a small decode case."""
    shape = (B, Hkv, T, d)
    k = W.outlier_keys(shape, seed) if keys == "outlier" else W.lognormal_rows(shape, seed, dtype=np.float16)
    v = W.lognormal_rows(shape, seed + 1, dtype=np.float16) if vq else W.normal(shape, seed + 1, np.float16)
    s = W.sign_vector(d, seed + 2)
    kc, kn = oracle.write(k, s, bits)
    vc, vn = oracle.write(v, s, bits) if vq else (None, None)
    return k, v, s, kc, kn, vc, vn


SMALL = [(d, b, 4, vq) for d in (64, 128) for b in (1, 2, 3, 4) for vq in (False, True)]
SMALL += [(128, 3, g, vq) for g in (1, 2, 8) for vq in (False, True)]
SMALL += [(64, 4, g, False) for g in (1, 2, 8)]


SCORE_CASES = [(d, b, g, m) for m in ("tensor", "mma", "direct") for d, b, g in sorted({(d, b, g) for d, b, g, _ in SMALL})]
SCORE_CASES += [(d, b, g, m) for m in ("factored", "table") for d, b, g in [(128, 4, 4), (64, 3, 4), (128, 2, 8),
                                                                             (128, 1, 1)]]
SCORE_CASES += [(d, b, g, "table") for d, b, g in [(128, 2, 4), (128, 4, 1), (64, 1, 8), (128, 3, 8), (64, 2, 2)]]


# the attend kernels follow the gather mode: "mma" (the default) scores keys through warp-level MMAs, "factored" on
# CUDA cores
ATTEND_CASES = [(d, b, g, vq, "mma") for d, b, g, vq in SMALL]
ATTEND_CASES += [(d, b, g, vq, "factored") for d, b, g, vq in [(128, 4, 4, True), (128, 4, 4, False), (64, 3, 4, True),
                                                                (128, 2, 8, False), (128, 1, 1, True)]]
# the literal table (fp16 values): fields of 8 bits at b <= 2, 6 at b = 3, 8 or 4 at b = 4
ATTEND_CASES += [(d, b, g, False, "table") for d, b, g in [(128, 4, 4), (128, 4, 2), (128, 2, 4), (128, 2, 8), (64, 3, 4),
                                                           (128, 1, 8), (64, 1, 1)]]


@pytest.fixture
def gather_mode(request):
    ops.set_gather(request.param)
    yield request.param
    ops.set_gather("mma")


@pytest.mark.parametrize("d,bits,G,gather_mode", SCORE_CASES, indirect=["gather_mode"])
def test_score_matches_oracle(d, bits, G, gather_mode):
    B, Hkv, T, Tcap = 2, 2, 2500, 2560
    Hq = G * Hkv
    k, v, s, kc, kn, _, _ = oracle_cache(B, Hkv, T, d, bits, 300 + d + bits + G, False)
    q = W.normal((B, Hq, d), 400 + G, np.float32)
    lens = np.array([T, 1111], np.int32)
    scale = 0.7
    out = ops.score(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits, scale=scale,
                    seq_lens=cuda(lens), T=T).cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            Tb = lens[b]
            want = oracle.score_lut(q[b, h], kc[b, hk, :Tb], kn[b, hk, :Tb], s, bits, scale)
            A = parity.abs_score_scale(q[b, h].astype(np.float64), kc[b, hk, :Tb], kn[b, hk, :Tb], s, bits, scale)
            parity.check_scores(out[b, h, :Tb], want, A)
            assert np.all(np.isneginf(out[b, h, Tb:]))


@pytest.mark.parametrize("d,bits,G,vq,gather_mode", ATTEND_CASES, indirect=["gather_mode"])
def test_attend_matches_oracle(d, bits, G, vq, gather_mode):
    B, Hkv, T, Tcap = 2, 2, 2500, 2600
    Hq = G * Hkv
    k, v, s, kc, kn, vc, vn = oracle_cache(B, Hkv, T, d, bits, 500 + d + bits + G, vq)
    q = W.normal((B, Hq, d), 600 + G, np.float32)
    lens = np.array([T, 777], np.int32)
    scale = 1.0 / math.sqrt(d)
    args = dict(seq_lens=cuda(lens), T=T, scale=scale)
    if vq:
        out = ops.attend_decode(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits,
                                vcodes=cuda(padded(vc, Tcap)), vnorms=cuda(padded(vn, Tcap)), **args)
        want = oracle.decode_attention(q, kc, kn, s, bits, scale, vcodes=vc, vn16=vn, seq_lens=lens)
    else:
        out = ops.attend_decode(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits,
                                v=cuda(padded(v, Tcap)), **args)
        want = oracle.decode_attention(q, kc, kn, s, bits, scale, v=v, seq_lens=lens)
    parity.check_outputs(out.cpu().numpy(), want)


@pytest.mark.parametrize("gather_mode", ["mma", "factored"], indirect=True)
@pytest.mark.parametrize("vq", [False, True])
def test_attend_edge_cases(vq, gather_mode):
    d, bits, Hkv, G = 128, 4, 2, 4
    Hq = Hkv * G
    B, T, Tcap = 4, 300, 320
    k, v, s, kc, kn, vc, vn = oracle_cache(B, Hkv, T, d, bits, 700, vq)
    q = W.normal((B, Hq, d), 701, np.float32)
    q[3] = 0.0  # zero query: uniform softmax
    lens = np.array([1, 0, 300, 257], np.int32)
    vargs = dict(vcodes=cuda(padded(vc, Tcap)), vnorms=cuda(padded(vn, Tcap))) if vq else dict(v=cuda(padded(v, Tcap)))
    out = ops.attend_decode(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits, seq_lens=cuda(lens),
                            T=T, **vargs).cpu().numpy()
    okw = dict(vcodes=vc, vn16=vn) if vq else dict(v=v)
    want = oracle.decode_attention(q, kc, kn, s, bits, 1 / math.sqrt(d), seq_lens=lens, **okw)
    parity.check_outputs(out, want)
    assert np.all(out[1] == 0.0)  # empty row
    # T = 0 gives zeros
    out0 = ops.attend_decode(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits, T=0,
                             **vargs).cpu().numpy()
    assert np.all(out0 == 0.0)


@pytest.mark.parametrize("vq", [False, True])
def test_unaligned_norm_rows(vq):
    """An odd cache capacity leaves most norm rows off 16-byte alignment: the kernels then load norms per lane
    instead of staging them with the codes; scores and outputs stay the same."""
    d, bits, Hkv, G = 128, 4, 3, 4
    Hq = Hkv * G
    B, T, Tcap = 2, 1000, 1003
    k, v, s, kc, kn, vc, vn = oracle_cache(B, Hkv, T, d, bits, 750, vq)
    q = W.normal((B, Hq, d), 751, np.float32)
    lens = np.array([1000, 613], np.int32)
    vargs = dict(vcodes=cuda(padded(vc, Tcap)), vnorms=cuda(padded(vn, Tcap))) if vq else dict(v=cuda(padded(v, Tcap)))
    out = ops.attend_decode(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits, seq_lens=cuda(lens),
                            T=T, **vargs).cpu().numpy()
    okw = dict(vcodes=vc, vn16=vn) if vq else dict(v=v)
    parity.check_outputs(out, oracle.decode_attention(q, kc, kn, s, bits, 1 / math.sqrt(d), seq_lens=lens, **okw))
    if not vq:
        sc = ops.score(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits, scale=0.5,
                       seq_lens=cuda(lens), T=T).cpu().numpy()
        for b in range(B):
            for h in range(Hq):
                Tb = lens[b]
                want = oracle.score_lut(q[b, h], kc[b, h // G, :Tb], kn[b, h // G, :Tb], s, bits, 0.5)
                A = parity.abs_score_scale(q[b, h].astype(np.float64), kc[b, h // G, :Tb], kn[b, h // G, :Tb], s,
                                           bits, 0.5)
                parity.check_scores(sc[b, h, :Tb], want, A)


@pytest.mark.parametrize("vq", [False, True])
@pytest.mark.parametrize("d,bits,G,Tcap", [(128, 4, 4, 912), (64, 2, 8, 912), (128, 3, 1, 912), (128, 4, 4, 1003),
                                           (64, 2, 8, 1003), (64, 3, 4, 912), (64, 1, 2, 1003)])
def test_decode_step(vq, d, bits, G, Tcap):
    """axr_decode_step writes the new token exactly as axr_write_keys does and attends over it: the same bits in the
    cache, the same output as a separate append + attend, and parity with the oracle over the full cache.  Tcap 1003
    leaves the norm rows unaligned (norms read from global memory rather than staged with the tiles); with rows of
    8 or 24 bytes (d = 64, b = 1, 3) an even capacity takes the streaming kernel and an odd one the row kernel."""
    B, Hkv, T = 3, 2, 900
    Hq = Hkv * G
    k, v, s, kc, kn, vc, vn = oracle_cache(B, Hkv, T, d, bits, 950 + d + bits + G, vq)
    q = W.normal((B, Hq, d), 951, np.float32)
    lens = np.array([900, 1, 517], np.int32)  # the new token: the last position, the first, a middle one
    pos = lens - 1
    knew = np.stack([k[b, :, pos[b]] for b in range(B)])  # [B, Hkv, d]
    vnew = np.stack([v[b, :, pos[b]] for b in range(B)])
    # cache copies with garbage at each new token's position
    def stale(a, fill):
        a = padded(a, Tcap).copy()
        for b in range(B):
            a[b, :, pos[b]] = fill
        return a
    kc_g, kn_g = cuda(stale(kc, 0x5a)), cuda(stale(kn, np.float16(3.0)))
    if vq:
        vargs = dict(vcodes=cuda(stale(vc, 0xa5)), vnorms=cuda(stale(vn, np.float16(2.0))))
    else:
        vargs = dict(v=cuda(stale(v, np.float16(7.0))))
    out = ops.decode_step(cuda(q), cuda(knew), cuda(vnew), kc_g, kn_g, cuda(s), bits, seq_lens=cuda(lens), T=T,
                          **vargs).cpu().numpy()
    # the written token matches axr_write_keys on the same vectors
    st = cuda(s)
    wk_c, wk_n = ops.write_keys(cuda(knew.reshape(-1, d)), st, bits)
    for b in range(B):
        for h in range(Hkv):
            i = b * Hkv + h
            assert np.array_equal(kc_g[b, h, pos[b]].cpu().numpy(), wk_c[i].cpu().numpy())
            assert kn_g[b, h, pos[b]].item() == wk_n[i].item()
    if vq:
        wv_c, wv_n = ops.write_keys(cuda(vnew.reshape(-1, d)), st, bits)
        for b in range(B):
            for h in range(Hkv):
                i = b * Hkv + h
                assert np.array_equal(vargs["vcodes"][b, h, pos[b]].cpu().numpy(), wv_c[i].cpu().numpy())
                assert vargs["vnorms"][b, h, pos[b]].item() == wv_n[i].item()
    else:
        for b in range(B):
            assert np.array_equal(vargs["v"][b, :, pos[b]].cpu().numpy(), vnew[b])
    # the same output as attend over the now complete cache
    again = ops.attend_decode(cuda(q), kc_g, kn_g, cuda(s), bits, seq_lens=cuda(lens), T=T, **vargs).cpu().numpy()
    # the same kernel for quantized values (identical bits); fp16 values may take the other kernel, whose warps split
    # the tokens differently: fp16 weights rounded against other running maxima (2^-11 relative each)
    num = np.linalg.norm((out - again).reshape(B * Hq, d), axis=1)
    den = np.linalg.norm(again.reshape(B * Hq, d), axis=1)
    assert np.all(num <= 2.0 ** -11 * np.maximum(den, 1e-30)), (num / np.maximum(den, 1e-30)).max()
    # parity with the oracle over the whole cache (codes of the new token: the write path's own)
    kc_w = kc_g.cpu().numpy()[:, :, :T]
    kn_w = kn_g.cpu().numpy()[:, :, :T]
    if vq:
        okw = dict(vcodes=vargs["vcodes"].cpu().numpy()[:, :, :T], vn16=vargs["vnorms"].cpu().numpy()[:, :, :T])
    else:
        okw = dict(v=v)
    want = oracle.decode_attention(q, kc_w, kn_w, s, bits, 1 / math.sqrt(d), seq_lens=lens, **okw)
    parity.check_outputs(out, want)


@pytest.mark.parametrize("B,T", [(8, 4096), (40, 1024)])
@pytest.mark.parametrize("vq", [False, True])
def test_decode_step_many_items(vq, B, T):
    """More (batch row, KV head, split) items than resident blocks, ragged rows (one full, one of a single token):
    blocks carry several items, some of them holding a new token.  The step writes each token exactly as
    axr_write_keys does and gives the output of attend over the completed cache.  Both shapes hold at least 2^18
    (token, KV head) units, so quantized values take the streaming kernel as fp16 values do."""
    Hkv, G, d, bits = 8, 4, 128, 4
    Tcap = T + 8
    Hq = Hkv * G
    rng = np.random.default_rng(977)
    lens = rng.integers(1, T + 1, size=B).astype(np.int32)
    lens[0], lens[1] = T, 1
    st = cuda(W.sign_vector(d, 978))
    k = cuda(W.lognormal_rows((B, Hkv, Tcap, d), 979, dtype=np.float16))
    v = cuda(W.lognormal_rows((B, Hkv, Tcap, d), 980, dtype=np.float16))
    q = cuda(W.normal((B, Hq, d), 981, np.float32))
    kc, kn = ops.write_keys(k, st, bits)
    pos = torch.from_numpy(lens.astype(np.int64) - 1)
    bi = torch.arange(B)
    knew = k[bi, :, pos].contiguous()  # [B, Hkv, d]
    vnew = v[bi, :, pos].contiguous()
    kc[bi, :, pos] = 0x5a
    kn[bi, :, pos] = 3.0
    if vq:
        vc, vn = ops.write_keys(v, st, bits)
        vc[bi, :, pos] = 0xa5
        vn[bi, :, pos] = 2.0
        vargs = dict(vcodes=vc, vnorms=vn)
    else:
        vv = v.clone()
        vv[bi, :, pos] = 7.0
        vargs = dict(v=vv)
    sl = cuda(lens)
    out = ops.decode_step(q, knew, vnew, kc, kn, st, bits, seq_lens=sl, T=T, **vargs)
    wk_c, wk_n = ops.write_keys(knew, st, bits)
    assert torch.equal(kc[bi, :, pos], wk_c) and torch.equal(kn[bi, :, pos], wk_n)
    if vq:
        wv_c, wv_n = ops.write_keys(vnew, st, bits)
        assert torch.equal(vc[bi, :, pos], wv_c) and torch.equal(vn[bi, :, pos], wv_n)
    else:
        assert torch.equal(vv[bi, :, pos], vnew)
    again = ops.attend_decode(q, kc, kn, st, bits, seq_lens=sl, T=T, **vargs)
    num = torch.linalg.vector_norm(out - again, dim=-1)
    den = torch.linalg.vector_norm(again, dim=-1)
    assert bool(torch.all(num <= 2.0 ** -11 * den)), float((num / den).max())


@pytest.mark.parametrize("d,bits", [(128, 4), (128, 2), (64, 4)])
def test_attend_many_units_quantized_values(d, bits):
    """Quantized values over 40 x 8 x 1024 >= 2^18 (token, KV head) units: the streaming kernel's quantized-value
    path at four query heads per KV head, ragged rows (empty, one token, full), against the oracle on sampled batch
    rows."""
    B, Hkv, G, T, Tcap = 40, 8, 4, 1024, 1040
    Hq = Hkv * G
    k = W.lognormal_rows((B, Hkv, T, d), 1200 + d + bits, dtype=np.float16)
    v = W.lognormal_rows((B, Hkv, T, d), 1201 + d + bits, dtype=np.float16)
    s = W.sign_vector(d, 1202)
    q = W.normal((B, Hq, d), 1203, np.float32)
    lens = np.random.default_rng(1204).integers(1, T + 1, size=B).astype(np.int32)
    lens[0], lens[1], lens[2] = T, 1, 0
    kc, kn = oracle.write(k, s, bits)
    vc, vn = oracle.write(v, s, bits)
    out = ops.attend_decode(cuda(q), cuda(padded(kc, Tcap)), cuda(padded(kn, Tcap)), cuda(s), bits,
                            vcodes=cuda(padded(vc, Tcap)), vnorms=cuda(padded(vn, Tcap)), seq_lens=cuda(lens),
                            T=T).cpu().numpy()
    assert np.all(out[2] == 0)
    for b in [0, 1, 5, 17, 39]:
        want = oracle.decode_attention(q[b:b + 1], kc[b:b + 1], kn[b:b + 1], s, bits, 1.0 / math.sqrt(d),
                                       vcodes=vc[b:b + 1], vn16=vn[b:b + 1], seq_lens=lens[b:b + 1])
        parity.check_outputs(out[b:b + 1], want)


@pytest.mark.parametrize("d,G,Hkv", [(128, 4, 2), (64, 8, 1), (128, 1, 3), (64, 2, 2), (128, 8, 1)])
def test_dense_matches_oracle_attention(d, G, Hkv):
    """The dense fp16 kernel (per-warp streaming workers) against the oracle's attention on the same fp16 cache:
    every (d, G) family, rows of 0, 1, 5 and ragged lengths (tails inside a 32-token tile, chunks split over
    several workers), and garbage past each row's length that must not be read."""
    B, T, Tcap = 5, 2100, 2200
    k = W.lognormal_rows((B, Hkv, T, d), 800 + d + G, dtype=np.float16)
    v = W.normal((B, Hkv, T, d), 801 + d + G, np.float16)
    q = W.normal((B, Hkv * G, d), 802 + d + G, np.float32)
    lens = np.array([T, 5, 1500, 0, 1], np.int32)
    kp, vp = padded(k, Tcap, fill=np.nan), padded(v, Tcap, fill=np.nan)
    for b in range(B):  # positions past the row's length hold NaN: a read of one would show in the output
        kp[b, :, lens[b]:] = np.nan
        vp[b, :, lens[b]:] = np.nan
    out = ops.dense_decode(cuda(q), cuda(kp), cuda(vp), seq_lens=cuda(lens), T=T).cpu().numpy()
    for b in range(B):
        Tb = lens[b]
        if Tb == 0:
            assert np.all(out[b] == 0)
            continue
        want = oracle.attention(q[b][:, None, :], k[b, :, :Tb], v[b, :, :Tb], causal=False)[:, 0, :]
        parity.check_outputs(out[b], want)


def test_dense_full_size_sampled():
    """The long-context shape (B=8, T=32768, 32/8 heads, d=128) through the dense kernel, in the launch
    configuration the benchmark times; sampled (batch row, KV head) pairs against the oracle."""
    B, Hkv, G, T, d = 8, 8, 4, 32768, 128
    dev = torch.device("cuda", 0)
    k = W.lognormal_rows_device((B, Hkv, T, d), 810, dev)
    v = W.normal_device((B, Hkv, T, d), 811, dev, dtype=torch.float16)
    q = W.normal_device((B, Hkv * G, d), 812, dev, dtype=torch.float32)
    out = ops.dense_decode(q, k, v).cpu().numpy()
    for b, hk in [(0, 0), (3, 5), (7, 7)]:
        kk = k[b, hk].cpu().numpy()
        vv = v[b, hk].cpu().numpy()
        qq = q[b, hk * G:(hk + 1) * G].cpu().numpy()
        want = oracle.attention(qq[:, None, :], kk[None], vv[None], causal=False)[:, 0, :]
        parity.check_outputs(out[b, hk * G:(hk + 1) * G], want)


def test_split_count_invariance():
    """The same row attended with B=1 (many splits) and inside B=8 (fewer splits) agrees to fp32 noise."""
    d, bits, Hkv, G, T = 128, 4, 8, 4, 32768
    shape = (8, Hkv, T, d)
    k = W.lognormal_rows(shape, 900, dtype=np.float16)
    v = W.normal(shape, 901, np.float16)
    s = W.sign_vector(d, 902)
    q = W.normal((8, Hkv * G, d), 903, np.float32)
    kc, kn = ops.write_keys(cuda(k), cuda(s), bits)
    vt = cuda(v)
    qt = cuda(q)
    st = cuda(s)
    full = ops.attend_decode(qt, kc, kn, st, bits, v=vt)
    one = ops.attend_decode(qt[:1].contiguous(), kc[:1].contiguous(), kn[:1].contiguous(), st, bits,
                            v=vt[:1].contiguous())
    assert ops.attend_workspace_bytes(1, 32, 8, T, d) // 1 != ops.attend_workspace_bytes(8, 32, 8, T, d) // 8
    a, b = full[0].cpu().numpy(), one[0].cpu().numpy()
    assert np.max(np.abs(a - b)) <= 1e-5 * np.max(np.abs(a))


def _full_size(w, samples, seed_q=None, step=False):
    """Full-size workload in the benchmark's launch configuration: the cache is written on the GPU, attention runs
    on the GPU; sampled (batch, head) outputs are recomputed by the oracle from the same host inputs.  With step,
    also the call the benchmark times: axr_decode_step writing token T - 1 itself over a cache whose position T - 1
    is stale must leave the cache as the writer does, and its sampled outputs must match the oracle too."""
    inp = W.decode_inputs(w)
    k, v, q, s = inp["k"], inp["v"], inp["q"], inp["signs"]
    st = cuda(s)
    kc, kn = ops.write_keys(cuda(k), st, w.bits)
    if w.v_quant:
        vc, vn = ops.write_keys(cuda(v), st, w.bits)
        out = ops.attend_decode(cuda(q), kc, kn, st, w.bits, vcodes=vc, vnorms=vn)
    else:
        out = ops.attend_decode(cuda(q), kc, kn, st, w.bits, v=cuda(v))
    out = out.cpu().numpy()
    got = None
    if step:
        kc_s, kn_s = kc.clone(), kn.clone()
        kc_s[:, :, -1] = 0x5a
        kn_s[:, :, -1] = 3.0
        knew, vnew = cuda(k[:, :, -1]), cuda(v[:, :, -1])  # [B, Hkv, d]
        if w.v_quant:
            vc_s, vn_s = vc.clone(), vn.clone()
            vc_s[:, :, -1] = 0xa5
            vn_s[:, :, -1] = 2.0
            vargs = dict(vcodes=vc_s, vnorms=vn_s)
        else:
            v_s = cuda(v)
            v_s[:, :, -1] = 7.0
            vargs = dict(v=v_s)
        got = ops.decode_step(cuda(q), knew, vnew, kc_s, kn_s, st, w.bits, **vargs).cpu().numpy()
        assert torch.equal(kc_s, kc) and torch.equal(kn_s, kn)
        if w.v_quant:
            assert torch.equal(vc_s, vc) and torch.equal(vn_s, vn)
        else:
            assert torch.equal(v_s, cuda(v))
    kc_h, kn_h = kc.cpu().numpy(), kn.cpu().numpy()
    vc_h = vn_h = None
    if w.v_quant:
        vc_h, vn_h = vc.cpu().numpy(), vn.cpu().numpy()
    scale = 1.0 / math.sqrt(w.d)
    for b, h in samples:
        hk = h // w.G
        nmk, _ = parity.check_indices(kc_h[b, hk], k[b, hk], s, w.d, w.bits)
        parity.check_norms(kn_h[b, hk], k[b, hk])
        okc, okn = oracle.write(k[b, hk], s, w.bits)
        if w.v_quant:
            parity.check_indices(vc_h[b, hk], v[b, hk], s, w.d, w.bits)
            ovc, ovn = oracle.write(v[b, hk], s, w.bits)
            want = oracle.decode_attention(q[b:b + 1, h:h + 1], okc[None, None], okn[None, None], s, w.bits, scale,
                                           vcodes=ovc[None, None], vn16=ovn[None, None])
        else:
            want = oracle.decode_attention(q[b:b + 1, h:h + 1], okc[None, None], okn[None, None], s, w.bits, scale,
                                           v=v[b:b + 1, hk:hk + 1])
        parity.check_outputs(out[b:b + 1, h:h + 1], want)
        if got is not None:
            parity.check_outputs(got[b:b + 1, h:h + 1], want)
        # and the scores of this head against the oracle on the oracle's codes
        sc = ops.score(cuda(q[b:b + 1, hk * w.G:(hk + 1) * w.G]), cuda(okc[None, None]), cuda(okn[None, None]), st,
                       w.bits, scale=scale).cpu().numpy()[0, h - hk * w.G]
        want_s = oracle.score_lut(q[b, h], okc, okn, s, w.bits, scale)
        A = parity.abs_score_scale(q[b, h].astype(np.float64), okc, okn, s, w.bits, scale)
        parity.check_scores(sc, want_s, A)


def test_llama8b_shaped_decode_full_size():
    _full_size(W.LLAMA8B_DECODE, [(0, 0), (3, 13), (7, 31)], step=True)


def test_long_context_kv_quantized_full_size():
    _full_size(W.LONG_CONTEXT, [(0, 1), (5, 22), (7, 31)], step=True)


@pytest.mark.parametrize("B,T,bits,d", [(1, 131072, 1, 64), (1, 131072, 3, 128), (64, 4096, 2, 128),
                                        (8, 32768, 4, 64)])
def test_sweep_rows_sampled(B, T, bits, d):
    w = W.sweep_case(B, T, bits, d)
    _full_size(w, [(0, 0), (B - 1, 31)])


def _sweep_device(w, samples):
    """A decode-sweep row at its full size with inputs drawn on the device by the benchmark's own generators (one
    batch row at a time, as the benchmark does; the host could not hold B=64 x T=131072 in numpy).  The attend
    runs in the benchmark's launch configuration; each sampled (batch row, query head) is recomputed by the oracle
    from that unit's inputs copied back to the host: indices and norms of the GPU writer, scores of the GPU scorer
    on the oracle's codes, and the attention output."""
    B, Hq, Hkv, T, d, bits, G = w.B, w.Hq, w.Hkv, w.T, w.d, w.bits, w.G
    dev = torch.device("cuda")
    st = cuda(W.sign_vector(d, w.seed + 4))
    s = st.cpu().numpy()
    k = torch.empty((B, Hkv, T, d), dtype=torch.float16, device=dev)
    v = torch.empty((B, Hkv, T, d), dtype=torch.float16, device=dev)
    for b in range(B):
        k[b] = W.lognormal_rows_device((Hkv, T, d), w.seed + 7919 * b, dev)
        v[b] = W.lognormal_rows_device((Hkv, T, d), w.seed + 2 + 7919 * b, dev)
    q = W.normal_device((B, Hq, d), w.seed + 3, dev, dtype=torch.float32)
    kc, kn = ops.write_keys(k, st, bits)
    out = ops.attend_decode(q, kc, kn, st, bits, v=v).cpu().numpy()
    scale = 1.0 / math.sqrt(d)
    qh = q.cpu().numpy()
    for b, h in samples:
        hk = h // G
        kh, vh = k[b, hk].cpu().numpy(), v[b, hk].cpu().numpy()
        parity.check_indices(kc[b, hk].cpu().numpy(), kh, s, d, bits)
        parity.check_norms(kn[b, hk].cpu().numpy(), kh)
        okc, okn = oracle.write(kh, s, bits)
        want = oracle.decode_attention(qh[b:b + 1, h:h + 1], okc[None, None], okn[None, None], s, bits, scale,
                                       v=vh[None, None])
        parity.check_outputs(out[b:b + 1, h:h + 1], want)
        sc = ops.score(q[b:b + 1, hk * G:(hk + 1) * G].contiguous(), cuda(okc[None, None]), cuda(okn[None, None]),
                       st, bits, scale=scale).cpu().numpy()[0, h - hk * G]
        want_s = oracle.score_lut(qh[b, h], okc, okn, s, bits, scale)
        A = parity.abs_score_scale(qh[b, h].astype(np.float64), okc, okn, s, bits, scale)
        parity.check_scores(sc, want_s, A)
    del k, v, kc, kn
    torch.cuda.empty_cache()


# With test_sweep_rows_sampled every (b, d) pair of the sweep appears at least once, the largest row
# (B=64, T=131072, b=4, d=128: 21.6 GB of cache) included.
@pytest.mark.parametrize("B,T,bits,d", [(64, 131072, 4, 128), (8, 4096, 1, 128), (64, 32768, 2, 64),
                                        (8, 131072, 3, 64)])
def test_sweep_rows_sampled_device_inputs(B, T, bits, d):
    w = W.sweep_case(B, T, bits, d)
    _sweep_device(w, [(0, 0), (B // 2, 13), (B - 1, 31)])
