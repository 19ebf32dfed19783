"""GPU parity of the power-of-two shift-accumulate codec against the oracle: the writer's codes and alpha bit for
bit, the shift-accumulated integer sums bit for bit, the real scores, and decode attention with integer-log2
weights.  Every integer is decided in fp32 in the same order on both sides; every weight is an exact power of two,
so the attention outputs differ only by the order of fp32 sums (checked at 1e-4 relative L2, well inside 2e-3)."""

import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_quantized_b200 import ops
from kv_cache_quantized_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu

FORMATS = [(3, 0), (2, 1), (2, 0), (1, 1), (1, 0)]
POT_OUT_REL_L2 = 1e-4


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("E,M", FORMATS)
def test_writer_is_bit_exact(d, E, M):
    k = W.lognormal_rows((2500, d), 50 + d + 10 * E + M, dtype=np.float16)
    k[7] = 0  # a zero row: alpha 0
    codes, alpha = ops.pot_write(cuda(k), E, M)
    oc, oa = oracle.pot_encode(k, E, M)
    assert np.array_equal(alpha.cpu().numpy().view(np.uint16), oa.view(np.uint16))
    assert np.array_equal(codes.cpu().numpy(), oracle.pack(oc, 1 + E + M))


@pytest.mark.parametrize("d,E,M,G", [(128, 3, 0, 4), (128, 2, 1, 4), (64, 3, 0, 8), (64, 2, 0, 1), (128, 1, 1, 2)])
def test_integer_sums_scores_and_attention(d, E, M, G):
    B, Hkv, T, Tcap = 2, 2, 1700, 1792
    Hq = Hkv * G
    k = W.lognormal_rows((B, Hkv, T, d), 60 + d + E, dtype=np.float16)
    v = W.normal((B, Hkv, T, d), 61, np.float16)
    q = W.normal((B, Hq, d), 62, np.float32)
    bits = 1 + E + M
    oc, oa = oracle.pot_encode(k, E, M)
    cpad = np.zeros((B, Hkv, Tcap, d * bits // 8), np.uint8)
    cpad[:, :, :T] = oracle.pack(oc, bits)
    apad = np.zeros((B, Hkv, Tcap), np.float16)
    apad[:, :, :T] = oa
    vpad = np.zeros((B, Hkv, Tcap, d), np.float16)
    vpad[:, :, :T] = v
    lens = np.array([T, 901], np.int32)
    scale = 1.0 / math.sqrt(d)
    sc, S = ops.pot_score(cuda(q), cuda(cpad), cuda(apad), E, M, scale=scale, seq_lens=cuda(lens), T=T, integers=True)
    sc, S = sc.cpu().numpy(), S.cpu().numpy()
    for b in range(B):
        for h in range(Hq):
            hk, n = h // G, lens[b]
            Q, _ = oracle.pot_quantize_query(q[b, h])
            assert np.array_equal(S[b, h, :n], oracle.pot_score_int(Q, oc[b, hk, :n], E, M))
            assert np.all(S[b, h, n:] == 0) and np.all(np.isneginf(sc[b, h, n:]))
            want = oracle.pot_score(q[b, h], oc[b, hk, :n], oa[b, hk, :n], E, M, scale)
            assert np.allclose(sc[b, h, :n], want, rtol=1e-6, atol=1e-30)
    out = ops.pot_attend_decode(cuda(q), cuda(cpad), cuda(apad), cuda(vpad), E, M, seq_lens=cuda(lens), T=T)
    want = oracle.pot_attention(q, oc, oa, v, E, M, scale, seq_lens=lens)
    got = out.cpu().numpy()
    rel = np.linalg.norm(got - want, axis=-1) / np.linalg.norm(want, axis=-1)
    assert rel.max() <= POT_OUT_REL_L2, rel.max()
    parity.check_outputs(got, want)


def test_many_splits_and_empty_rows():
    """Several splits per row (the integer maxima of the splits merged by exact powers of two) and an empty row."""
    E, M, d, G = 3, 0, 128, 4
    B, Hkv, T = 3, 2, 20000
    Hq = Hkv * G
    k = W.lognormal_rows((B, Hkv, T, d), 70, dtype=np.float16)
    v = W.normal((B, Hkv, T, d), 71, np.float16)
    q = 3.0 * W.normal((B, Hq, d), 72, np.float32)  # sharper weights: many tokens far below the maximum
    lens = np.array([T, 0, 12345], np.int32)
    codes, alpha = ops.pot_write(cuda(k), E, M)
    out = ops.pot_attend_decode(cuda(q), codes, alpha, cuda(v), E, M, seq_lens=cuda(lens)).cpu().numpy()
    oc, oa = oracle.pot_encode(k, E, M)
    want = oracle.pot_attention(q, oc, oa, v, E, M, 1 / math.sqrt(d), seq_lens=lens)
    assert np.all(out[1] == 0)
    keep = [0, 2]
    rel = np.linalg.norm(out[keep] - want[keep], axis=-1) / np.linalg.norm(want[keep], axis=-1)
    assert rel.max() <= POT_OUT_REL_L2, rel.max()
