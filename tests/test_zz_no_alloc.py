"""axr_attend_decode_static: the decode step for callers that cannot allocate device memory (it keeps its split
partials in a fixed library-owned device array instead of a caller workspace).  Called through the C ABI with raw
pointers, twice in a row, it must give the same result as axr_attend_decode with a caller workspace.

This file is collected last so that a run stopping at the first failure has already run every other test."""

import math

import numpy as np
import pytest
import torch

from kv_cache_quantized_b200 import _abi, ops
from kv_cache_quantized_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("vq", [False, True])
def test_static_scratch_matches_workspace_path(vq):
    B, Hq, Hkv, T, Tcap, d, bits = 3, 16, 4, 3000, 3072, 128, 4
    k = W.lognormal_rows((B, Hkv, T, d), 31, dtype=np.float16)
    v = W.lognormal_rows((B, Hkv, T, d), 32, dtype=np.float16)
    q = _cuda(W.normal((B, Hq, d), 33, np.float32))
    s = _cuda(W.sign_vector(d, 34))
    kc = torch.zeros((B, Hkv, Tcap, d * bits // 8), dtype=torch.uint8, device="cuda")
    kn = torch.zeros((B, Hkv, Tcap), dtype=torch.float16, device="cuda")
    kc[:, :, :T], kn[:, :, :T] = ops.write_keys(_cuda(k), s, bits)
    lens = _cuda(np.array([T, 1234, 0], np.int32))
    scale = 1.0 / math.sqrt(d)
    if vq:
        vc = torch.zeros_like(kc)
        vn = torch.zeros_like(kn)
        vc[:, :, :T], vn[:, :, :T] = ops.write_keys(_cuda(v), s, bits)
        vkind, vptr, vnptr = _abi.V_QUANT, vc.data_ptr(), vn.data_ptr()
        want = ops.attend_decode(q, kc, kn, s, bits, vcodes=vc, vnorms=vn, seq_lens=lens, T=T, scale=scale)
    else:
        vv = torch.zeros((B, Hkv, Tcap, d), dtype=torch.float16, device="cuda")
        vv[:, :, :T] = _cuda(v)
        vkind, vptr, vnptr = _abi.V_F16, vv.data_ptr(), None
        want = ops.attend_decode(q, kc, kn, s, bits, v=vv, seq_lens=lens, T=T, scale=scale)
    assert _abi.lib().axr_attend_static_scratch_bytes() >= ops.attend_workspace_bytes(B, Hq, Hkv, T, d)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):  # two calls in a row: the shared array keeps the previous call's contents
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        st = _abi.lib().axr_attend_decode_static(q.data_ptr(), kc.data_ptr(), kn.data_ptr(), vkind, vptr, vnptr,
                                                 lens.data_ptr(), B, Hq, Hkv, T, Tcap, d, bits, s.data_ptr(),
                                                 scale, out.data_ptr(), stream)
        _abi.check(st, "axr_attend_decode_static")
        got = out.cpu().numpy()
        ref = want.cpu().numpy()
        rel = np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
        assert np.all(np.isfinite(got)) and np.all(rel <= 2e-3), rel.max()


def test_static_scratch_rejects_sizes_beyond_the_array():
    big_B, Hq, Hkv, T, d = 512, 32, 8, 131072, 128
    assert ops.attend_workspace_bytes(big_B, Hq, Hkv, T, d) > _abi.lib().axr_attend_static_scratch_bytes()
    F = 0x10000  # never dereferenced: the size check fails first
    st = _abi.lib().axr_attend_decode_static(F, F, F, _abi.V_F16, F, None, None, big_B, Hq, Hkv, T, T, d, 4, F,
                                             0.088, F, None)
    assert st == 4 and b"fixed" in _abi.lib().axr_last_error()
