"""GPU parity of the write path (axr_write_keys) against the oracle: indices, fp16 norms, packing, scatter rows."""

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


@pytest.mark.parametrize("d", [8, 64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("dt", [np.float16, np.float32])
def test_write_matches_oracle(d, bits, dt):
    x = W.lognormal_rows((3001, d), 100 + d + bits, dtype=dt)
    s = W.sign_vector(d, 200 + d)
    codes, norms = ops.write_keys(cuda(x), cuda(s), bits)
    torch.cuda.synchronize()
    assert codes.shape == (3001, d * bits // 8) and norms.shape == (3001,)
    parity.check_indices(codes.cpu().numpy(), x, s, d, bits)
    parity.check_norms(norms.cpu().numpy(), x)


def test_outlier_keys_and_grid_stride():
    """More vectors than one grid pass covers (the kernel strides), with x10 outlier channels."""
    d, bits = 128, 4
    x = W.outlier_keys((40_000, d), 7)
    s = W.sign_vector(d, 8)
    codes, norms = ops.write_keys(cuda(x), cuda(s), bits)
    parity.check_indices(codes.cpu().numpy(), x, s, d, bits)
    parity.check_norms(norms.cpu().numpy(), x)


def test_zero_vectors():
    for bits in (1, 2, 3, 4):
        x = np.zeros((5, 128), np.float16)
        codes, norms = ops.write_keys(cuda(x), cuda(np.ones(128, np.int8)), bits)
        idx = oracle.unpack(codes.cpu().numpy(), 128, bits)
        assert np.all(idx == (1 << bits) // 2) and np.all(norms.cpu().numpy() == 0)


def test_dst_rows_scatter_into_cache():
    """Appending one token per (batch, KV head) into a [B, Hkv, Tcap] cache at per-row positions."""
    B, Hkv, Tcap, d, bits = 3, 4, 50, 128, 3
    R = d * bits // 8
    x = W.normal((B, Hkv, d), 9, np.float16)
    s = W.sign_vector(d, 10)
    pos = np.array([0, 17, 49])
    dst = ((np.arange(B)[:, None] * Hkv + np.arange(Hkv)[None, :]) * Tcap + pos[:, None]).reshape(-1)
    codes = torch.full((B, Hkv, Tcap, R), 0xAB, dtype=torch.uint8, device="cuda")
    norms = torch.zeros((B, Hkv, Tcap), dtype=torch.float16, device="cuda")
    ops.write_keys(cuda(x), cuda(s), bits, codes=codes.view(-1, R), norms=norms.view(-1), dst_rows=cuda(dst))
    c = codes.cpu().numpy()
    n = norms.cpu().numpy()
    want_c, want_n = oracle.write(x, s, bits)
    for b in range(B):
        assert np.array_equal(c[b, :, pos[b]], want_c[b])
        assert np.array_equal(n[b, :, pos[b]].view(np.uint16), want_n[b].view(np.uint16))
    untouched = np.ones((B, Hkv, Tcap), bool)
    for b in range(B):
        untouched[b, :, pos[b]] = False
    assert np.all(c[untouched] == 0xAB) and np.all(n[untouched] == 0)


def test_single_head_config_write_then_score():
    """Single head, d=128, b=2, 1024 fp32 keys x lognormal(0,0.5) norms: write on the GPU, then LUT scores on the
    GPU.  The scores are checked twice, whatever the index parity found: the GPU scorer on the oracle's own codes
    against the oracle's brute-force dequantize-then-dot, and the GPU scorer on the GPU's codes against the
    oracle's brute force on those same codes."""
    w = W.SINGLE_HEAD
    inp = W.decode_inputs(w)
    k = inp["k"][0, 0]  # [T, d] fp32
    q = inp["q"]        # [1, 1, d]
    s = inp["signs"]
    st = cuda(s)
    codes, norms = ops.write_keys(cuda(k), st, w.bits)
    parity.check_indices(codes.cpu().numpy(), k, s, w.d, w.bits)
    parity.check_norms(norms.cpu().numpy(), k)
    oc, on = oracle.write(k, s, w.bits)
    # the scorer on the oracle's codes
    sc = ops.score(cuda(q), cuda(oc[None, None]), cuda(on[None, None]), st, w.bits, scale=1.0)
    want = oracle.score_bruteforce(q[0, 0], oc, on, s, w.bits)
    A = parity.abs_score_scale(q[0, 0].astype(np.float64), oc, on, s, w.bits, 1.0)
    parity.check_scores(sc.cpu().numpy()[0, 0], want, A)
    # the scorer on the GPU's own codes
    gc, gn = codes.cpu().numpy(), norms.cpu().numpy()
    sc2 = ops.score(cuda(q), codes.view(1, 1, w.T, -1), norms.view(1, 1, w.T), st, w.bits, scale=1.0)
    want2 = oracle.score_bruteforce(q[0, 0], gc, gn, s, w.bits)
    A2 = parity.abs_score_scale(q[0, 0].astype(np.float64), gc, gn, s, w.bits, 1.0)
    parity.check_scores(sc2.cpu().numpy()[0, 0], want2, A2)
