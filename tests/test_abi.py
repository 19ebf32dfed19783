"""Host-side checks of the C ABI (no GPU): the library loads, exports every function include/axr.h declares, its
host codebook matches the oracle's, and bad arguments come back as error statuses before any CUDA call."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from kv_cache_quantized_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(_abi.LIB_PATH):
        from kv_cache_quantized_b200 import build
        build.build()
    return _abi.lib()


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"AXR_API\s+[\w\s\*]+?\b(axr_\w+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
        assert n in _abi.SIGNATURES, f"{n} has no ctypes signature"


def test_version(L):
    assert L.axr_version() == 100


@pytest.mark.parametrize("d", [8, 64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_host_codebook_matches_oracle(L, d, bits):
    n = 1 << bits
    c = np.zeros(n)
    t = np.zeros(n - 1 if n > 1 else 1)
    st = L.axr_codebook(d, bits, c.ctypes.data_as(ctypes.c_void_p), t.ctypes.data_as(ctypes.c_void_p))
    assert st == 0
    oc, ot = oracle.codebook(d, bits)
    assert np.max(np.abs(c - oc)) < 1e-13
    assert np.max(np.abs(t[: n - 1] - ot)) < 1e-13
    assert t[n // 2 - 1] == 0.0  # exact middle threshold


def test_codebook_errors(L):
    buf = np.zeros(16)
    p = buf.ctypes.data_as(ctypes.c_void_p)
    assert L.axr_codebook(100, 2, p, p) == 2
    assert L.axr_codebook(128, 5, p, p) == 2
    assert L.axr_codebook(128, 2, None, p) == 1
    assert b"null" in L.axr_last_error()


FAKE = 0x10000  # a 64 KiB-aligned non-null address; never dereferenced because every call below fails validation


def test_write_argument_errors(L):
    assert L.axr_write_keys(FAKE, 0, -1, 128, 4, FAKE, None, FAKE, FAKE, None) == 1
    assert L.axr_write_keys(FAKE, 0, 5, 96, 4, FAKE, None, FAKE, FAKE, None) == 2
    assert L.axr_write_keys(FAKE, 0, 5, 128, 5, FAKE, None, FAKE, FAKE, None) == 2
    assert L.axr_write_keys(FAKE, 7, 5, 128, 4, FAKE, None, FAKE, FAKE, None) == 1
    assert L.axr_write_keys(None, 0, 5, 128, 4, FAKE, None, FAKE, FAKE, None) == 1
    assert L.axr_write_keys(FAKE + 4, 0, 5, 128, 4, FAKE, None, FAKE, FAKE, None) == 1  # fp32 rows need 16 B
    assert L.axr_write_keys(None, 0, 0, 128, 4, None, None, None, None, None) == 0  # empty is a no-op


def test_write_tiled_argument_errors(L):
    W = L.axr_write_values_tiled
    assert W(FAKE, 0, -1, 128, 4, FAKE, None, 256, FAKE, FAKE, None) == 1     # n_vec < 0
    assert W(FAKE, 0, 128, 64, 4, FAKE, None, 256, FAKE, FAKE, None) == 2     # tiles are built for d = 128
    assert W(FAKE, 0, 128, 128, 0, FAKE, None, 256, FAKE, FAKE, None) == 2
    assert W(FAKE, 0, 128, 128, 4, FAKE, None, 200, FAKE, FAKE, None) == 1    # Tcap not a multiple of 128
    assert W(FAKE, 0, 128, 128, 4, FAKE, None, 0, FAKE, FAKE, None) == 1
    assert W(None, 0, 128, 128, 4, FAKE, None, 256, FAKE, FAKE, None) == 1
    assert W(FAKE, 0, 128, 128, 4, FAKE, None, 256, FAKE + 2, FAKE, None) == 1  # codes need 4-byte alignment
    assert W(None, 0, 0, 128, 4, None, None, 256, None, None, None) == 0       # empty is a no-op


def test_attend_tiled_argument_errors(L):
    call = lambda d=128, Tcap=256, vn=FAKE: L.axr_attend_decode(FAKE, FAKE, FAKE, 2, FAKE, vn, None, 2, 8, 2, 200,
                                                               Tcap, d, 4, FAKE, 0.1, FAKE, FAKE, 1 << 20, None)
    assert call(d=64, Tcap=256) == 2   # tiled values: d = 128 only
    assert call(Tcap=320) == 1         # Tcap a multiple of 128
    assert call(vn=None) == 1          # value norms required
    assert L.axr_attend_decode(FAKE, FAKE, FAKE, 3, FAKE, FAKE, None, 2, 8, 2, 200, 256, 128, 4, FAKE, 0.1, FAKE,
                               FAKE, 1 << 20, None) == 1  # unknown vkind


def test_decode_step_argument_errors(L):
    call = lambda kn=FAKE, vn_new=FAKE, vkind=1, d=128: L.axr_decode_step(
        FAKE, kn, vn_new, FAKE, FAKE, vkind, FAKE, FAKE, None, 2, 8, 2, 200, 256, d, 4, FAKE, 0.1, FAKE, FAKE,
        1 << 20, None)
    assert call(kn=None) == 1            # the new key is required
    assert call(vn_new=None) == 1        # and the new value
    assert call(kn=FAKE + 8) == 1        # 16-byte aligned
    assert call(vkind=2) == 1            # row value layouts only
    assert call(d=32) == 2
    assert L.axr_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, 1, FAKE, FAKE, None, 0, 8, 2, 200, 256, 128, 4, FAKE,
                             0.1, FAKE, FAKE, 1 << 20, None) == 0  # B = 0: nothing to do


def test_score_argument_errors(L):
    args = lambda **kw: dict(dict(q=FAKE, kc=FAKE, kn=FAKE, sl=None, B=2, Hq=8, Hkv=2, T=10, Tcap=16, d=128,
                                  bits=4, s=FAKE, scale=1.0, out=FAKE), **kw)
    call = lambda a: L.axr_score(a["q"], a["kc"], a["kn"], a["sl"], a["B"], a["Hq"], a["Hkv"], a["T"], a["Tcap"],
                                 a["d"], a["bits"], a["s"], a["scale"], a["out"], None)
    assert call(args(Hq=6, Hkv=4)) == 1          # Hq not a multiple of Hkv
    assert call(args(T=20)) == 1                 # T > Tcap
    assert call(args(d=32)) == 2
    assert call(args(Hq=6, Hkv=2)) == 2          # G = 3
    assert call(args(bits=0)) == 2
    assert call(args(q=None)) == 1
    assert call(args(kc=FAKE + 8)) == 1          # codes need 16-byte alignment
    assert call(args(scale=float("inf"))) == 1
    assert call(args(B=0)) == 0


def test_attend_workspace_rules(L):
    ws = L.axr_attend_workspace_bytes(8, 32, 8, 32768, 128)
    assert ws > 0 and ws % 256 == 0
    assert L.axr_attend_workspace_bytes(8, 32, 8, 32768, 128) == ws
    assert L.axr_attend_workspace_bytes(0, 32, 8, 32768, 128) == 0
    assert L.axr_attend_workspace_bytes(1, 32, 8, 100, 128) > 0
    call = lambda wsb, vk=0, vn=None: L.axr_attend_decode(FAKE, FAKE, FAKE, vk, FAKE, vn, None, 8, 32, 8, 32768,
                                                          32768, 128, 4, FAKE, 0.088, FAKE, FAKE, wsb, None)
    assert call(ws - 1) == 4
    assert L.axr_attend_decode(FAKE, FAKE, FAKE, 0, FAKE, None, None, 8, 32, 8, 32768, 32768, 128, 4, FAKE, 0.088,
                               FAKE, None, ws, None) == 4
    assert call(ws, vk=1, vn=None) == 1          # quantized V needs value norms
    assert call(ws, vk=3) == 1
    assert L.axr_dense_decode(FAKE, FAKE, FAKE, None, 8, 32, 8, 32768, 32768, 128, 0.088, FAKE, FAKE, ws - 1,
                              None) == 4


def test_select_argument_errors(L):
    ws = L.axr_select_workspace_bytes(2, 2, 64, 16, 2, 128, 8)
    assert ws > 0
    call = lambda **kw: L.axr_select_signs(FAKE, FAKE, FAKE, kw.get("Ly", 2), 2, 64, kw.get("Hq", 16), 2,
                                           kw.get("d", 128), kw.get("bits", 4), FAKE, 8, 1, FAKE, FAKE,
                                           kw.get("ws", FAKE), kw.get("wsb", ws), None)
    assert call(d=32) == 2
    assert call(bits=7) == 2
    assert call(Hq=15) == 1
    assert call(Ly=0) == 1
    assert call(wsb=ws - 1) == 4
    assert call(ws=None) == 4


def test_select_per_layer_argument_errors(L):
    ws = L.axr_select_workspace_bytes(2, 2, 64, 16, 2, 128, 8)
    # the per-(candidate, layer, sequence) sums are part of the workspace
    assert ws >= 8 * 2 * 2 * 8 and ws == L.axr_select_workspace_bytes(2, 2, 64, 16, 2, 128, 8)
    call = lambda **kw: L.axr_select_signs_per_layer(FAKE, FAKE, FAKE, kw.get("Ly", 2), 2, 64, kw.get("Hq", 16), 2,
                                                     kw.get("d", 128), kw.get("bits", 4), FAKE, 8, 1, FAKE, FAKE,
                                                     kw.get("parts", None), kw.get("ws", FAKE), kw.get("wsb", ws),
                                                     None)
    assert call(d=32) == 2
    assert call(bits=0) == 2
    assert call(Hq=15) == 1
    assert call(Ly=0) == 1
    assert call(parts=FAKE + 4) == 1  # f64 parts need 8-byte alignment
    assert call(wsb=ws - 1) == 4
    assert call(ws=None) == 4


def test_status_argument_errors(L):
    """Host-side rejections of the status entry points (no CUDA call is made)."""
    assert L.axr_device_status(None, 0) == 1 and b"null" in L.axr_last_error()
    for polls in (0, -1, (1 << 20) + 1):
        assert L.axr_selftest_wait_timeout(polls, None) == 1


def test_paged_argument_errors_host(L):
    """Rejections made on the host before any launch (block size, table reach, null table, tiled values)."""
    call = lambda **kw: L.axr_attend_decode_paged(FAKE, FAKE, FAKE, kw.get("vk", 1), FAKE, FAKE, kw.get("tab", FAKE),
                                                  kw.get("mb", 4), kw.get("bt", 64), None, 2, 8, 2, kw.get("T", 256),
                                                  128, 4, FAKE, 0.088, FAKE, FAKE, 1 << 20, None)
    assert call(bt=48) == 1 and b"power of two" in L.axr_last_error()
    assert call(bt=8) == 1
    assert call(T=257) == 1 and b"exceeds" in L.axr_last_error()
    assert call(tab=None) == 1
    assert call(tab=FAKE + 2) == 1
    assert call(vk=2) == 1
    step = L.axr_decode_step_paged(FAKE, None, FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, 4, 64, None, 2, 8, 2, 256, 128,
                                   4, FAKE, 0.088, FAKE, FAKE, 1 << 20, None)
    assert step == 1


def test_codec_argument_errors_host(L):
    """LOOKAT and PoT entry points reject bad sizes and formats on the host, before any CUDA call."""
    assert L.axr_pq_encode(FAKE, 1, 10, 96, 4, 256, FAKE, 1, 1, None, FAKE, None) == 2      # d
    assert L.axr_pq_encode(FAKE, 1, 10, 128, 3, 256, FAKE, 1, 1, None, FAKE, None) == 2     # m
    assert L.axr_pq_encode(FAKE, 1, 10, 128, 4, 257, FAKE, 1, 1, None, FAKE, None) == 2     # K
    assert L.axr_pq_encode(FAKE, 1, 0, 128, 4, 256, None, 1, 1, None, None, None) == 0      # empty
    assert L.axr_pq_train(FAKE, 1, 10, 128, 4, 256, 3, FAKE, None, 0, None) == 4            # workspace
    assert L.axr_pq_train_workspace_bytes(128, 4, 256) >= 128 * 256 * 8
    assert L.axr_pq_score(FAKE, FAKE, FAKE, None, 2, 6, 4, 100, 100, 128, 4, 256, 0.1, FAKE, None) == 1  # Hq % Hkv
    assert L.axr_pq_attend_decode(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 100, 100, 128, 4, 256, 0.1, FAKE, None, 0,
                                  None) == 4
    assert L.axr_pot_write(FAKE, 10, 128, 3, 1, None, FAKE, FAKE, None) == 2  # 5-bit format
    assert L.axr_pot_write(FAKE, 10, 128, 0, 0, None, FAKE, FAKE, None) == 2
    assert L.axr_pot_score(FAKE, FAKE, FAKE, None, 2, 8, 2, 100, 100, 128, 3, 0, 0.1, None, None, None) == 1
    assert L.axr_pot_score(FAKE, FAKE + 8, FAKE, None, 2, 8, 2, 100, 100, 128, 3, 0, 0.1, FAKE, None, None) == 1
    assert L.axr_pot_attend_decode(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 100, 100, 128, 2, 1, 0.1, FAKE, FAKE, 16,
                                   None) == 4


def _plan(B, Hkv, T, workers, tile, min_tiles, setup):
    """The split rule, restated: the split count minimising ceil(items / workers) x (tiles per split + setup), chunks
    of whole tiles, at least min_tiles long; the first minimum wins."""
    units, tt = B * Hkv, -(-T // tile)
    best, plan = None, (1, tile)
    for s in range(1, max(1, min(tt // min_tiles, 4096)) + 1):
        tiles = -(-tt // s)
        splits = -(-tt // tiles)
        cost = -(-(units * splits) // workers) * (tiles + setup)
        if best is None or cost < best - 1e-9:
            best, plan = cost, (splits, tiles * tile)
    return plan


@pytest.mark.parametrize("B,Hq,Hkv,T,d", [(8, 32, 8, 32768, 128), (1, 32, 8, 4096, 128), (64, 32, 8, 131072, 64),
                                         (3, 16, 4, 3000, 128), (8, 32, 8, 8192, 128)])
def test_attend_workspace_holds_every_kernels_split_plan(L, B, Hq, Hkv, T, d):
    """The workspace query covers the largest split plan of the kernels that may run: the row kernel (296 workers,
    128-token tiles) and the streaming kernels (one worker per warp: 592 dense, 1184 fp16 values, 2368 quantized
    values; 32-token tiles); the long-context step's plan is 37 splits of 896 tokens."""
    s = max([_plan(B, Hkv, T, 296, 128, 4, 0.5)[0]] + [_plan(B, Hkv, T, w, 32, 2, 2.0)[0] for w in (592, 1184, 2368)])
    parts = B * Hq * s
    assert L.axr_attend_workspace_bytes(B, Hq, Hkv, T, d) == -(-(parts * d * 4 + 2 * parts * 4) // 256) * 256
    assert _plan(8, 8, 32768, 2368, 32, 2, 2.0) == (37, 896)


def _prototypes():
    """name -> list of parameter declarations, from the AXR_API prototypes of include/*.h."""
    out = {}
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = re.sub(r"/\*.*?\*/", " ", open(os.path.join(ROOT, "include", f)).read(), flags=re.S)
            for m in re.finditer(r"AXR_API\s+([\w\s\*]+?)\b(axr_\w+)\s*\(([^)]*)\)", txt):
                params = [p.strip() for p in m.group(3).split(",")]
                out[m.group(2)] = (m.group(1).strip(), [] if params in ([""], ["void"]) else params)
    return out


def _ctype_of(decl):
    if "*" in decl:
        return "ptr"
    base = decl.rsplit(None, 1)[0].replace("const", "").strip()
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t, "int64_t": ctypes.c_int64,
            "axr_vkind": ctypes.c_int, "axr_gather": ctypes.c_int, "axr_dtype": ctypes.c_int,
            "uint32_t": ctypes.c_uint32}.get(base, base)


def test_binding_signatures_match_the_header():
    """Every ctypes signature of the binding has the header's return type and parameter count, and each parameter the
    header's kind: a pointer where the header has one, the matching integer or float type elsewhere."""
    protos = _prototypes()
    assert set(protos) == set(_abi.SIGNATURES)
    for name, (ret, params) in protos.items():
        res, args = _abi.SIGNATURES[name]
        want_res = {"axr_status": ctypes.c_int, "int": ctypes.c_int, "axr_gather": ctypes.c_int,
                    "size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p}[ret.replace(" *", "*")]
        assert res is want_res, f"{name}: returns {ret}, bound as {res}"
        assert len(args) == len(params), f"{name}: {len(args)} ctypes arguments, {len(params)} in the header"
        for decl, ct in zip(params, args):
            want = _ctype_of(decl)
            if want == "ptr":
                assert ct in (ctypes.c_void_p, ctypes.c_char_p), f"{name}: {decl!r} bound as {ct}"
            else:
                assert ct is want or ct == want, f"{name}: {decl!r} bound as {ct}, header wants {want}"
