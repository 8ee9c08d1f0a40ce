"""Host-side checks of the C ABI (no GPU work): the library loads, exports every
symbol the header declares, and rejects bad arguments before any launch."""

import ctypes
import os
import re

import pytest

from hybrid_sliding_window_sink_b200 import _lib
from hybrid_sliding_window_sink_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mimo_attn.h")


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mimo_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert set(names) == set(_lib.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    for code in range(8):
        s = L.mimo_status_string(code).decode()
        assert s and s != "unknown status"
    assert L.mimo_status_string(99).decode() == "unknown status"
    assert L.mimo_attn_version() >= 100


def _shape(**kw):
    base = dict(batch=1, seqlen=64, hq=8, hkv=1, dqk=192, dv=128, softmax_scale=0.0)
    base.update(kw)
    return _lib.make_shape(base["batch"], base["seqlen"], base["hq"], base["hkv"], base["dqk"],
                           base["dv"], base["softmax_scale"])


P = ctypes.c_void_p
GOOD = P(0x10000)   # never dereferenced: every case below fails validation first


def _prefill(L, shape, q=GOOD, k=GOOD, v=GOOD, out=GOOD, sink=None, lse=None, window=128,
             theta=1e4, rot=64):
    return L.mimo_attn_prefill(ctypes.byref(shape), q, k, v, sink, window, theta, rot, out, lse, None)


def test_prefill_rejects_before_launch(L):
    assert L.mimo_attn_prefill(None, GOOD, GOOD, GOOD, None, 128, 1e4, 64, GOOD, None, None) == 1
    assert _prefill(L, _shape(), q=None) == 1
    assert _prefill(L, _shape(), out=None) == 1
    assert _prefill(L, _shape(seqlen=0)) == 2
    assert _prefill(L, _shape(batch=0)) == 2
    assert _prefill(L, _shape(hq=6, hkv=4)) == 2
    assert _prefill(L, _shape(hq=64, hkv=2)) == 3          # group 32
    assert _prefill(L, _shape(hq=12, hkv=4)) == 3          # group 3
    assert _prefill(L, _shape(dqk=128)) == 3
    assert _prefill(L, _shape(dv=192)) == 3
    assert _prefill(L, _shape(softmax_scale=float("nan"))) == 2
    assert _prefill(L, _shape(), rot=-2) == 2
    assert _prefill(L, _shape(), rot=200) == 2
    assert _prefill(L, _shape(), rot=40) == 3
    assert _prefill(L, _shape(), theta=0.0) == 2
    assert _prefill(L, _shape(), theta=float("inf")) == 2
    assert _prefill(L, _shape(), q=P(0x10008)) == 4
    assert _prefill(L, _shape(), out=P(0x10004)) == 4
    assert _prefill(L, _shape(), sink=P(0x10002)) == 4


def _decode(L, shape, kind=0, cap=128, stride=128, lengths=GOOD, q=GOOD, ws=None, nbytes=0):
    return L.mimo_attn_decode(ctypes.byref(shape), q, GOOD, GOOD, kind, cap, stride, lengths, None,
                              GOOD, None, ws, nbytes, None)


def test_decode_rejects_before_launch(L):
    s = _shape(hq=64, hkv=8)
    assert _decode(L, s, kind=5) == 2
    assert _decode(L, s, lengths=None) == 1
    assert _decode(L, s, q=None) == 1
    assert _decode(L, s, cap=0) == 2
    assert _decode(L, s, cap=256, stride=128) == 2
    assert _decode(L, s, q=P(0x10001)) == 4
    assert _decode(L, s, lengths=P(0x10002)) == 4
    assert _decode(L, _shape(hq=64, hkv=8, dqk=64)) == 3


def test_sparse_rejects_before_launch(L):
    s = _shape(hq=64, hkv=4)
    f = L.mimo_attn_sparse
    assert f(ctypes.byref(s), GOOD, GOOD, GOOD, 4096, 4096, GOOD, 128, None, 16, None, GOOD, None,
             None, 0, None) == 1
    assert f(ctypes.byref(s), GOOD, GOOD, GOOD, 4096, 4096, GOOD, -1, GOOD, 16, None, GOOD, None,
             None, 0, None) == 2
    assert f(ctypes.byref(s), GOOD, GOOD, GOOD, 4096, 4096, GOOD, 128, GOOD, -3, None, GOOD, None,
             None, 0, None) == 2


def test_workspace_size_plans(L):
    # ring of 128 slots: one chunk per (b, g), finalised in place, no workspace
    assert _lib.workspace_size(64, 64, 8, op=_lib.MIMO_OP_DECODE, kind=_lib.MIMO_CACHE_RING,
                               capacity=128) == 0
    # long linear cache: split-KV partials (m, l) + o per chunk
    n = _lib.workspace_size(64, 64, 4, op=_lib.MIMO_OP_DECODE, kind=_lib.MIMO_CACHE_LINEAR,
                            capacity=131072)
    assert n > 0 and n % 4 == 0
    nsp = _lib.workspace_size(8, 64, 4, op=_lib.MIMO_OP_SPARSE, capacity=262144, recent=128,
                              n_sel=1024)
    assert nsp > 0
    assert _lib.workspace_size(8, 64, 4, op=7, capacity=10) == 0
    assert _lib.workspace_size(8, 64, 4, op=_lib.MIMO_OP_SPARSE, capacity=10, recent=-1) == 0


def _decode_mq(L, shape, kind=_lib.MIMO_CACHE_RING, cap=131, stride=131, q_len=4, window=128,
               q=GOOD, k=GOOD, v=GOOD, lengths=GOOD, out=GOOD):
    return L.mimo_attn_decode_mq(ctypes.byref(shape), q, k, v, kind, cap, stride, lengths, q_len,
                                 window, None, out, None, None, 0, None)


def test_decode_mq_rejects_before_launch(L):
    s16 = _shape(hq=64, hkv=4)                       # 16 query heads per KV head
    # ring must keep every draft token's window: capacity >= window + q_len - 1
    assert _decode_mq(L, s16, cap=130, stride=130) == 2
    assert _decode_mq(L, s16, window=0) == 2
    assert _decode_mq(L, s16, q_len=0) == 2
    assert _decode_mq(L, s16, kind=7) == 2
    assert _decode_mq(L, s16, q_len=5) == 3          # 5 * 16 rows > 64
    assert _decode_mq(L, s16, q=None) == 1
    assert _decode_mq(L, s16, stride=100) == 2       # stride below capacity
    assert _decode_mq(L, s16, q=P(0x10002)) == 4     # misaligned
    # linear cache ignores the window
    assert _decode_mq(L, s16, kind=_lib.MIMO_CACHE_LINEAR, window=0, cap=4096, stride=4096,
                      q=None) == 1


def test_decode_mq_workspace_plans(L):
    ring = _shape(batch=64, hq=64, hkv=8)
    # a ring of window + 3 slots fits one chunk: finalised in place
    assert L.mimo_attn_decode_mq_workspace_size(ctypes.byref(ring), _lib.MIMO_CACHE_RING, 131, 4,
                                                128) == 0
    lin = _shape(batch=64, hq=64, hkv=4)
    n = L.mimo_attn_decode_mq_workspace_size(ctypes.byref(lin), _lib.MIMO_CACHE_LINEAR, 131072, 4, 0)
    assert n > 0 and n % 4 == 0
    # invalid sizes: no plan
    assert L.mimo_attn_decode_mq_workspace_size(ctypes.byref(ring), _lib.MIMO_CACHE_RING, 128, 4,
                                                128) == 0
    assert L.mimo_attn_decode_mq_workspace_size(ctypes.byref(lin), _lib.MIMO_CACHE_LINEAR, 4096, 8,
                                                0) == 0


def test_prefill_chunk_and_append_reject_before_launch(L):
    s = _shape(hq=64, hkv=8, seqlen=100)
    chunk = lambda **kw: L.mimo_attn_prefill_chunk(  # noqa: E731
        ctypes.byref(s), kw.get("q", GOOD), GOOD, GOOD, kw.get("off", 10), 1, None, 128,
        kw.get("theta", 1e4), kw.get("rot", 64), GOOD, None, None)
    assert chunk(off=-1) == 2
    assert chunk(q=None) == 1
    assert chunk(rot=24) == 3
    assert chunk(theta=0.0) == 2
    assert chunk(q=P(0x10004)) == 4
    app = lambda **kw: L.mimo_attn_cache_append(  # noqa: E731
        ctypes.byref(s), GOOD, GOOD, kw.get("off", 0), 1e4, 64, kw.get("kind", _lib.MIMO_CACHE_LINEAR),
        kw.get("kc", GOOD), GOOD, kw.get("cap", 1000), kw.get("stride", 1000), None)
    assert app(off=950) == 2                          # linear cache too small for the chunk
    assert app(kind=5) == 2
    assert app(kc=None) == 1
    assert app(stride=999) == 2
    assert app(kc=P(0x10008)) == 4


def test_select_tokens_rejects_before_launch(L):
    s = _shape(hq=64, hkv=4)
    sel = lambda **kw: L.mimo_attn_select_tokens(  # noqa: E731
        ctypes.byref(s), kw.get("q", GOOD), GOOD, kw.get("cap", 4096), kw.get("stride", 4096), GOOD,
        kw.get("recent", 128), kw.get("n_sel", 1024), kw.get("out", GOOD), kw.get("ws", GOOD),
        kw.get("wsb", 1 << 30), None)
    assert sel(q=None) == 1
    assert sel(out=None) == 1
    assert sel(recent=-1) == 2
    assert sel(n_sel=-5) == 2
    assert sel(stride=100) == 2
    assert sel(ws=None) == 5
    assert sel(wsb=16) == 5
    assert sel(q=P(0x10002)) == 4
    assert sel(n_sel=0) == 0          # nothing to select: OK without a launch
    need = L.mimo_attn_select_workspace_size(ctypes.byref(s), 4096)
    assert need == 1 * 4 * 4096 * 4 + 1 * 4 * 4 * 256 * 2      # keys, then top-byte histograms
    # key rows padded to 16 bytes
    assert L.mimo_attn_select_workspace_size(ctypes.byref(s), 1027) == (4 * 1028 * 4 + 4 * 2 * 512 + 255) // 256 * 256
