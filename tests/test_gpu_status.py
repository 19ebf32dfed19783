"""The device status word: a kernel whose bounded wait gives up reports it to the host (axr_device_status), beside
the NaN it writes.  The give-up path is exercised by the library's self-test kernel, which waits with a short poll
limit on an mbarrier that nothing arrives on (no copy pending): it gives up, sets the word and returns, and the
context stays usable.  No GPU fault or hang is involved."""

import numpy as np
import pytest
import torch

from kv_cache_quantized_b200 import _abi, ops
from kv_cache_quantized_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_wait_timeout_sets_the_status_word_and_the_context_survives():
    ops.device_status(clear=True)
    assert ops.device_status() == 0
    _abi.check(_abi.lib().axr_selftest_wait_timeout(64, torch.cuda.current_stream().cuda_stream),
               "axr_selftest_wait_timeout")
    flags = ops.device_status()
    assert flags & _abi.STATUS_WAIT_TIMEOUT
    # the raw call reports the timeout as an error with a message
    import ctypes
    f = ctypes.c_uint(0)
    st = _abi.lib().axr_device_status(ctypes.byref(f), 1)
    assert st == 3 and f.value & 1 and b"gave up" in _abi.lib().axr_last_error()
    assert ops.device_status() == 0  # cleared
    # the context is still usable: a decode call afterwards runs and reports nothing
    d, bits = 128, 4
    k = torch.from_numpy(W.lognormal_rows((1, 2, 300, d), 5, dtype=np.float16)).cuda()
    st_ = torch.from_numpy(W.sign_vector(d, 6)).cuda()
    q = torch.from_numpy(W.normal((1, 8, d), 7, np.float32)).cuda()
    kc, kn = ops.write_keys(k, st_, bits)
    out = ops.attend_decode(q, kc, kn, st_, bits, vcodes=kc, vnorms=kn)
    assert torch.isfinite(out).all()
    assert ops.device_status() == 0
