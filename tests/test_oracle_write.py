"""Pins for the oracle's write path (AXELRAM Key Points / Abstract: transform on write, fixed codebook, indices):
the transform against a library Hadamard routine and orthogonality, the quantizer against brute-force nearest
centroid, the packing against numpy.packbits and hand-worked bytes, and the fp16 norm against numpy's rounding."""

import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from kv_cache_quantized_b200 import workloads as W

HERE = os.path.dirname(__file__)


@pytest.mark.parametrize("d", [1, 2, 8, 64, 128])
def test_hadamard_matches_library(d):
    H = oracle.hadamard(d)
    assert np.array_equal(H * math.sqrt(d), scipy.linalg.hadamard(d).astype(np.float64))


@pytest.mark.parametrize("d", [8, 64, 128])
def test_hadamard_orthogonal_symmetric_involutory(d):
    H = oracle.hadamard(d)
    I = np.eye(d)
    assert np.max(np.abs(H @ H.T - I)) < 1e-12
    assert np.array_equal(H, H.T)
    assert np.max(np.abs(H @ H - I)) < 1e-12
    x = W.normal((16, d), 1, np.float64)
    assert np.allclose(np.linalg.norm(oracle.rotate(x, np.ones(d)), axis=-1), np.linalg.norm(x, axis=-1),
                       rtol=1e-13)


@pytest.mark.parametrize("d", [8, 128])
def test_rotate_inverse(d):
    s = W.sign_vector(d, 5).astype(np.float64)
    x = W.normal((4, d), 2, np.float64)
    y = oracle.rotate(x, s)
    back = (y @ oracle.hadamard(d).T) * s  # (H D_s)^-1 = D_s H
    assert np.max(np.abs(back - x)) < 1e-12


@pytest.mark.parametrize("d", [8, 64])
def test_walsh_row_sign_is_a_permutation(d):
    """H diag(h_r) = P_r H with (P_r y)_i = y_{i xor r}: a Walsh row in the sign vector only permutes coordinates."""
    Hs = scipy.linalg.hadamard(d)
    x = W.normal((3, d), 3, np.float64)
    s = W.sign_vector(d, 9).astype(np.float64)
    y = oracle.rotate(x, s)
    for r in range(d):
        y2 = oracle.rotate(x, s * Hs[r])
        perm = np.arange(d) ^ r
        assert np.max(np.abs(y2 - y[:, perm])) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_threshold_count_is_nearest_centroid(bits):
    d = 128
    c, t = oracle.codebook(d, bits)
    g = W.rng(bits)
    x = g.standard_normal((200, d))
    idx, n, n16, u = oracle.quantize_rows(x, np.ones(d), bits)
    nearest = np.argmin(np.abs(u[..., None] - c), axis=-1)
    gap = np.min(np.abs(u[..., None] - t), axis=-1)
    ok = gap > 1e-12
    assert np.array_equal(idx[ok], nearest[ok])
    assert idx.min() >= 0 and idx.max() < (1 << bits)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_tie_goes_up(bits):
    """A unit coordinate exactly on threshold t_k maps to index k (the upper cell)."""
    d = 8
    c, t = oracle.codebook(d, bits)
    H = oracle.hadamard(d)
    for k, tk in enumerate(t, start=1):
        # build x with u = H x / |x| having coordinate 0 equal to tk exactly is awkward; check the rule itself
        u = np.array([tk])
        assert int(np.sum(u[..., None] >= t, axis=-1)[0]) == k
    # and through the full path: x = e_0 with all signs +1 gives u_j = 1/sqrt(d) for every j
    x = np.zeros((1, d))
    x[0, 0] = 1.0
    idx, n, n16, u = oracle.quantize_rows(x, np.ones(d), bits)
    assert np.allclose(u, H[:, 0][None, :])
    want = int(np.sum(1.0 / math.sqrt(d) >= t))
    assert np.all(idx == want)


def test_worked_example_e0_b2():
    """d=8, b=2, x = e_0, s = +1: every u_j = 1/sqrt(8), i.e. 1.0 in N(0,1) units, which is above the top
    threshold 0.9816 -> every index is 3; the norm is 1."""
    x = np.zeros((1, 8))
    x[0, 0] = 1.0
    idx, n, n16, u = oracle.quantize_rows(x, np.ones(8), 2)
    assert np.all(idx == 3) and n[0] == 1.0 and n16[0] == np.float16(1.0)


def test_zero_vector():
    for bits in (1, 2, 3, 4):
        idx, n, n16, u = oracle.quantize_rows(np.zeros((2, 64)), np.ones(64), bits)
        assert np.all(idx == (1 << bits) // 2) and np.all(n == 0) and np.all(n16 == 0)


def test_norm16_is_round_to_nearest_even():
    x = W.lognormal_rows((500, 128), 4, dtype=np.float32)
    _, n, n16, _ = oracle.quantize_rows(x, np.ones(128), 4)
    ref = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1))
    assert np.array_equal(n, ref)
    import torch
    assert np.array_equal(n16, torch.from_numpy(ref).to(torch.float16).numpy())


def _golden_pack():
    rows = []
    with open(os.path.join(HERE, "golden", "pack_lsb_first.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b, c = line.split("|")
            d, bits = map(int, a.split())
            rows.append((d, bits, [int(x) for x in b.split()], [int(x, 16) for x in c.split()]))
    return rows


def test_pack_hand_worked():
    for d, bits, idx, want in _golden_pack():
        got = oracle.pack(np.array([idx]), bits)[0]
        assert list(got) == want, (d, bits)
        assert list(oracle.unpack(got[None], d, bits)[0]) == idx


@pytest.mark.parametrize("d,bits", [(8, 1), (8, 3), (64, 3), (128, 1), (128, 2), (128, 3), (128, 4)])
def test_pack_matches_packbits_and_roundtrips(d, bits):
    idx = W.rng(d * bits).integers(0, 1 << bits, size=(50, d))
    stream = ((idx[..., :, None] >> np.arange(bits)) & 1).reshape(50, d * bits).astype(np.uint8)
    want = np.packbits(stream, axis=-1, bitorder="little")
    got = oracle.pack(idx, bits)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.unpack(got, d, bits), idx)
