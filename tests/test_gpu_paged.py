"""GPU parity of decode attention over paged caches (axr_attend_decode_paged, axr_decode_step_paged): pools of
blocks addressed through a shuffled block table, ragged lengths, block sizes below and above the kernel's 128-token
tile, fp16 and quantized values, against the oracle on the same tokens and against the contiguous-cache path."""

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


def paginate(cache, lens, bt, table_seed, spare=3):
    """Scatter a contiguous cache [B, Hkv, T, ...] into a pool [num_blocks, Hkv, bt, ...] through a shuffled block
    table [B, max_blocks]; blocks no row uses hold noise.  Returns (pool, table)."""
    B, Hkv, T = cache.shape[:3]
    mb = -(-T // bt)
    need = [-(-int(n) // bt) for n in lens]
    nblocks = sum(need) + spare
    rng = np.random.default_rng(table_seed)
    perm = rng.permutation(nblocks)
    table = np.zeros((B, mb), np.int32)  # entries past a row's blocks stay 0, a valid block that is never read
    pool = rng.integers(0, 255, size=(nblocks, Hkv, bt) + cache.shape[3:]).astype(cache.dtype)
    k = 0
    for b in range(B):
        for j in range(need[b]):
            p = perm[k]
            k += 1
            table[b, j] = p
            n = min(bt, T - j * bt)
            pool[p, :, :n] = cache[b, :, j * bt:j * bt + n]
    return pool, table


CASES = [(128, 4, 4, 16, True), (128, 4, 4, 128, False), (128, 4, 4, 256, True), (128, 2, 8, 32, False),
         (64, 3, 4, 64, True), (64, 1, 2, 16, False), (128, 3, 1, 512, True), (64, 4, 4, 128, True)]


@pytest.mark.parametrize("d,bits,G,bt,vq", CASES)
def test_paged_attend_matches_oracle_and_contiguous(d, bits, G, bt, vq):
    B, Hkv, T = 3, 2, 1100
    Hq = Hkv * G
    shape = (B, Hkv, T, d)
    k = W.lognormal_rows(shape, 40 + d + bits + bt, dtype=np.float16)
    v = W.lognormal_rows(shape, 41 + d + bits + bt, dtype=np.float16)
    s = W.sign_vector(d, 42)
    q = W.normal((B, Hq, d), 43, np.float32)
    lens = np.array([T, 1, 517], np.int32)
    kc, kn = oracle.write(k, s, bits)
    kcp, table = paginate(kc, lens, bt, 7)
    knp, _ = paginate(kn, lens, bt, 7)
    scale = 1.0 / math.sqrt(d)
    st, tq, tt, tl = cuda(s), cuda(q), cuda(table), cuda(lens)
    if vq:
        vc, vn = oracle.write(v, s, bits)
        vargs = dict(vcodes=cuda(paginate(vc, lens, bt, 7)[0]), vnorms=cuda(paginate(vn, lens, bt, 7)[0]))
        cargs = dict(vcodes=cuda(vc), vnorms=cuda(vn))
        want = oracle.decode_attention(q, kc, kn, s, bits, scale, vcodes=vc, vn16=vn, seq_lens=lens)
    else:
        vargs = dict(v=cuda(paginate(v, lens, bt, 7)[0]))
        cargs = dict(v=cuda(v))
        want = oracle.decode_attention(q, kc, kn, s, bits, scale, v=v, seq_lens=lens)
    out = ops.attend_decode_paged(tq, cuda(kcp), cuda(knp), st, bits, tt, seq_lens=tl, T=T, **vargs).cpu().numpy()
    parity.check_outputs(out, want)
    assert np.all(out[1] != 0) and np.all(np.isfinite(out))
    # the contiguous cache through the library gives the same result up to rounding: it may take the streaming
    # kernel (other split points).  fp16 values carry fp32-level weights there; quantized values carry fp16 weights
    # p n^V / sqrt(d) in both kernels, each rounded to half an fp16 ulp (2^-11) against its own split maxima.
    ref = ops.attend_decode(tq, cuda(kc), cuda(kn), st, bits, seq_lens=tl, T=T, **cargs).cpu().numpy()
    num = np.linalg.norm((out - ref).reshape(-1, d), axis=1)
    den = np.linalg.norm(ref.reshape(-1, d), axis=1)
    assert np.all(num <= (2.0 ** -10 if vq else 2.0 ** -11) * den), float(np.max(num / den))


@pytest.mark.parametrize("vq", [False, True])
@pytest.mark.parametrize("bt", [16, 128])
def test_paged_decode_step_writes_through_the_table(vq, bt):
    d, bits, G, B, Hkv, T = 128, 4, 4, 4, 2, 700
    Hq = Hkv * G
    shape = (B, Hkv, T, d)
    k = W.lognormal_rows(shape, 60 + bt, dtype=np.float16)
    v = W.lognormal_rows(shape, 61 + bt, dtype=np.float16)
    s = W.sign_vector(d, 62)
    q = W.normal((B, Hq, d), 63, np.float32)
    lens = np.array([700, 1, 129, 0], np.int32)  # the new token at the last, the first and a block's first position
    pos = np.maximum(lens - 1, 0)
    kc, kn = oracle.write(k, s, bits)
    vc, vn = oracle.write(v, s, bits)
    knew = np.stack([k[b, :, pos[b]] for b in range(B)])
    vnew = np.stack([v[b, :, pos[b]] for b in range(B)])
    kcp, table = paginate(kc, lens, bt, 9)
    knp, _ = paginate(kn, lens, bt, 9)
    # stale bytes at each new token's row in the pools
    def stale(pool, fill):
        pool = pool.copy()
        for b in range(B):
            if lens[b] > 0:
                pool[table[b, pos[b] // bt], :, pos[b] % bt] = fill
        return pool
    kcp_d, knp_d = cuda(stale(kcp, 0x5a)), cuda(stale(knp, np.float16(3.0)))
    if vq:
        vargs = dict(vcodes=cuda(stale(paginate(vc, lens, bt, 9)[0], 0xa5)),
                     vnorms=cuda(stale(paginate(vn, lens, bt, 9)[0], np.float16(2.0))))
    else:
        vargs = dict(v=cuda(stale(paginate(v, lens, bt, 9)[0], np.float16(7.0))))
    st = cuda(s)
    out = ops.decode_step_paged(cuda(q), cuda(knew), cuda(vnew), kcp_d, knp_d, st, bits, cuda(table),
                                seq_lens=cuda(lens), T=T, **vargs).cpu().numpy()
    # the written rows equal the oracle's codes and norms of those tokens (rows with len 0 are untouched)
    for b in range(B):
        if lens[b] == 0:
            continue
        p, o = table[b, pos[b] // bt], pos[b] % bt
        for h in range(Hkv):
            assert np.array_equal(kcp_d[p, h, o].cpu().numpy(), kc[b, h, pos[b]])
            if vq:
                assert np.array_equal(vargs["vcodes"][p, h, o].cpu().numpy(), vc[b, h, pos[b]])
            else:
                assert np.array_equal(vargs["v"][p, h, o].cpu().numpy(), v[b, h, pos[b]])
    okw = dict(vcodes=vc, vn16=vn) if vq else dict(v=v)
    want = oracle.decode_attention(q, kc, kn, s, bits, 1 / math.sqrt(d), seq_lens=lens, **okw)
    parity.check_outputs(out, want)
    assert np.all(out[3] == 0)


def test_paged_argument_errors():
    d, bits, B, Hkv, G, bt = 128, 4, 2, 2, 4, 64
    kc = torch.zeros((8, Hkv, bt, d * bits // 8), dtype=torch.uint8, device="cuda")
    kn = torch.zeros((8, Hkv, bt), dtype=torch.float16, device="cuda")
    q = torch.zeros((B, Hkv * G, d), dtype=torch.float32, device="cuda")
    s = torch.ones(d, dtype=torch.int8, device="cuda")
    table = torch.zeros((B, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(Exception, match="exceeds"):
        ops.attend_decode_paged(q, kc, kn, s, bits, table, T=4 * bt + 1, vcodes=kc, vnorms=kn)
    kc2 = torch.zeros((8, Hkv, 48, d * bits // 8), dtype=torch.uint8, device="cuda")
    kn2 = torch.zeros((8, Hkv, 48), dtype=torch.float16, device="cuda")
    with pytest.raises(Exception, match="power of two"):
        ops.attend_decode_paged(q, kc2, kn2, s, bits, table, vcodes=kc2, vnorms=kn2)


# Pools the streaming kernel takes: quantized values, at least 2^18 (token, KV head) units or eight query heads per
# KV head, and blocks of at least its 32-token tile.  (d, bits, G, B, Hkv, T, bt)
STREAM_CASES = [(128, 4, 4, 4, 8, 8192, 32), (128, 4, 4, 4, 8, 8192, 256), (64, 3, 8, 2, 2, 1000, 64)]


@pytest.mark.parametrize("d,bits,G,B,Hkv,T,bt", STREAM_CASES)
def test_paged_streaming_kernel(d, bits, G, B, Hkv, T, bt):
    """Paged pools through the streaming kernel: attend and decode step give the contiguous cache's results bit for
    bit (the same kernel arithmetic, split plan and rows, only addressed through a shuffled block table), the step
    writes its token through the table, and sampled heads match the oracle on the host inputs."""
    Hq = Hkv * G
    shape = (B, Hkv, T, d)
    k = W.lognormal_rows(shape, 70 + bt + d, dtype=np.float16)
    v = W.lognormal_rows(shape, 71 + bt + d, dtype=np.float16)
    s = W.sign_vector(d, 72)
    q = W.normal((B, Hq, d), 73, np.float32)
    lens = np.array([T, T // 2 + 1, 33, T - 7][:B], np.int32)
    st, tq, tl = cuda(s), cuda(q), cuda(lens)
    kc, kn = ops.write_keys(cuda(k), st, bits)
    vc, vn = ops.write_keys(cuda(v), st, bits)
    mb = -(-T // bt)
    nblocks = B * mb + 5
    rng = np.random.default_rng(bt + d)
    table = cuda(rng.permutation(nblocks)[:B * mb].reshape(B, mb).astype(np.int32))

    def pool(x, noise):
        """x [B, Hkv, T, ...] scattered into a pool [nblocks, Hkv, bt, ...] through the table; spare blocks hold
        noise."""
        pad = torch.zeros((B, Hkv, mb * bt) + tuple(x.shape[3:]), dtype=x.dtype, device="cuda")
        pad[:, :, :T] = x
        p = noise((nblocks, Hkv, bt) + tuple(x.shape[3:]))
        blocks = pad.reshape((B, Hkv, mb, bt) + tuple(x.shape[3:])).transpose(1, 2)
        p[table.long().reshape(-1)] = blocks.reshape((B * mb, Hkv, bt) + tuple(x.shape[3:]))
        return p

    codes_noise = lambda shp: torch.randint(0, 256, shp, dtype=torch.uint8, device="cuda")
    norms_noise = lambda shp: (torch.rand(shp, device="cuda") * 4).half()
    kcp, knp = pool(kc, codes_noise), pool(kn, norms_noise)
    vcp, vnp = pool(vc, codes_noise), pool(vn, norms_noise)

    out_c = ops.attend_decode(tq, kc, kn, st, bits, vcodes=vc, vnorms=vn, seq_lens=tl, T=T)
    out_p = ops.attend_decode_paged(tq, kcp, knp, st, bits, table, seq_lens=tl, T=T, vcodes=vcp, vnorms=vnp)
    assert torch.equal(out_p, out_c)

    # the decode step over stale rows at each row's last position, in both layouts
    pos = lens - 1
    knew = cuda(np.stack([k[b, :, pos[b]] for b in range(B)]))
    vnew = cuda(np.stack([v[b, :, pos[b]] for b in range(B)]))
    kc_s, kn_s, vc_s, vn_s = kc.clone(), kn.clone(), vc.clone(), vn.clone()
    kcp_s, knp_s, vcp_s, vnp_s = kcp.clone(), knp.clone(), vcp.clone(), vnp.clone()
    tab = table.cpu().numpy()
    for b in range(B):
        p, o = tab[b, pos[b] // bt], pos[b] % bt
        kc_s[b, :, pos[b]] = 0x5a; kn_s[b, :, pos[b]] = 3.0; vc_s[b, :, pos[b]] = 0xa5; vn_s[b, :, pos[b]] = 2.0
        kcp_s[p, :, o] = 0x5a; knp_s[p, :, o] = 3.0; vcp_s[p, :, o] = 0xa5; vnp_s[p, :, o] = 2.0
    step_c = ops.decode_step(tq, knew, vnew, kc_s, kn_s, st, bits, vcodes=vc_s, vnorms=vn_s, seq_lens=tl, T=T)
    step_p = ops.decode_step_paged(tq, knew, vnew, kcp_s, knp_s, st, bits, table, seq_lens=tl, T=T, vcodes=vcp_s,
                                   vnorms=vnp_s)
    assert torch.equal(step_p, step_c)
    for got, want in ((kcp_s, kcp), (knp_s, knp), (vcp_s, vcp), (vnp_s, vnp)):
        assert torch.equal(got, want)  # the written rows are the writer's, the rest untouched

    out, got = out_p.cpu().numpy(), step_p.cpu().numpy()
    scale = 1.0 / math.sqrt(d)
    for b, h in [(0, 0), (B - 1, Hq - 1), (1, Hq // 2 + 1), (B - 1, 3)]:
        hk, n = h // G, lens[b]
        okc, okn = oracle.write(k[b, hk, :n], s, bits)
        ovc, ovn = oracle.write(v[b, hk, :n], s, bits)
        want = oracle.decode_attention(q[b:b + 1, h:h + 1], okc[None, None], okn[None, None], s, bits, scale,
                                       vcodes=ovc[None, None], vn16=ovn[None, None])
        parity.check_outputs(out[b:b + 1, h:h + 1], want)
        parity.check_outputs(got[b:b + 1, h:h + 1], want)
