"""The arithmetic the MMA read paths rely on for the score tolerance, checked on the host in exact arithmetic.

AXELRAM Key Points (1st, 2nd items): a score is the gather-sum of q~_j c_k at the stored indices.  The warp-level
MMA paths form each product from fp16 operands, so both factors are carried as two fp16 planes, hi = fp16(x) and
lo = fp16(x - hi), and the four plane products are accumulated in fp32.  These tests pin the premises of that
reading: the planes represent the Lloyd-Max centroids and the power-of-two-scaled query coordinates to about
2^-22 relative, and a score formed from the four plane products (exactly, in fp64) stays far inside the score
tolerance that the parity tests apply (1e-6 absolute + 1e-5 relative to the sum of |terms|)."""

import math

import numpy as np
import pytest

import oracle
from kv_cache_quantized_b200 import workloads as W
from tests import parity


def planes(x):
    """hi = fp16(x), lo = fp16(x - hi), as fp64 values (round to nearest even, like __float2half_rn)."""
    x = np.asarray(x, np.float64)
    hi = x.astype(np.float16).astype(np.float64)
    lo = (x - hi).astype(np.float16).astype(np.float64)
    return hi, lo


def head_scale(qt):
    """2^(14 - e) with ||q~|| in [2^(e-1), 2^e): the power of two the MMA paths scale each head's operand by."""
    _, e = math.frexp(float(np.linalg.norm(qt)))
    return 2.0 ** (14 - e)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_centroid_planes(bits):
    gamma, _ = oracle.gaussian_lloyd_max(bits)  # the N(0, 1) levels the tables hold
    hi, lo = planes(gamma)
    rel = np.abs(gamma - (hi + lo)) / np.abs(gamma)
    assert np.all(rel <= 2.0 ** -22)
    assert np.all(np.abs(lo) <= 2.0 ** -11 * np.abs(gamma))


@pytest.mark.parametrize("d", [64, 128])
def test_query_planes_after_head_scale(d):
    rng = np.random.default_rng(5 + d)
    for trial in range(20):
        qt = rng.standard_normal(d) * 10.0 ** rng.uniform(-3, 3)
        sc = head_scale(qt)
        y = qt * sc
        assert np.abs(y).max() < 2.0 ** 15  # far from the fp16 overflow at 65504
        hi, lo = planes(y)
        err = np.abs(y - (hi + lo))
        # each coordinate to 2^-22 of the vector's scale (coordinates far below it may lose relative precision,
        # and then carry no weight in the score)
        assert np.all(err <= 2.0 ** -22 * np.abs(y).max())


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 4), (128, 1), (64, 3)])
def test_score_from_four_plane_products_meets_tolerance(d, bits):
    gamma, _ = oracle.gaussian_lloyd_max(bits)
    s = W.sign_vector(d, 31 + d + bits)
    k = W.lognormal_rows((200, d), 32 + bits, dtype=np.float32)
    q = W.normal((d,), 33 + bits, np.float64)
    codes, n16 = oracle.write(k, s, bits)
    scale = 1.0 / math.sqrt(d)
    want = oracle.score_lut(q, codes, n16, s, bits, scale)
    A = parity.abs_score_scale(q, codes, n16, s, bits, scale)
    # the same score through the planes: q~ = H (s .* q) scaled by a power of two, centroids at the N(0, 1) levels
    # (the 1/sqrt(d) of the unit-scale codebook and the softmax scale folded into one factor at the end)
    qt = oracle.rotate(q[None, :], s)[0]
    sc = head_scale(qt)
    qh, ql = planes(qt * sc)
    ch, cl = planes(gamma)
    idx = oracle.unpack(codes, d, bits)  # [tokens, d]
    terms = (ch[idx] + cl[idx]) * (qh + ql)  # all four plane products, exact in fp64
    got = terms.sum(axis=1) / sc * n16.astype(np.float64) * scale / math.sqrt(d)
    err = np.abs(got - want)
    # about 2^-25 of A in practice: a hundredth of the tolerance still leaves room, while a dropped lo plane
    # (2^-11 relative) would not fit
    assert np.all(err <= 1e-2 * (parity.SCORE_ABS + parity.SCORE_REL * A))
