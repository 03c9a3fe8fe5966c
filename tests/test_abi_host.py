"""Host-only checks of the C ABI: the library loads, exports every declared
symbol, sizes its buffers as documented and rejects bad arguments before it
touches a device. No compute call runs here."""
import ctypes
import os
import re

import pytest

from residual_binary_weight_b200 import _lib
from residual_binary_weight_b200._lib import GemvDesc, Layout

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rb_api.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*RB_API\s+(?:const\s+)?[a-z_0-9]+\s*\*?\s*(rb_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.EXPORTED, n


def test_library_hides_internal_symbols():
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {n for n in exported if n.startswith("rb_")}
    assert ours == set(_declared_functions())


def test_sizes():
    lib = _lib.load()
    assert lib.rb_planes_words(Layout(4096, 4096, 2, 0, 0, 0)) == 2 * 4096 * 128
    assert lib.rb_scales_count(Layout(4096, 4096, 2, 0, 0, 0)) == 2 * 4096
    assert lib.rb_scales_count(Layout(11008, 4096, 4, 128, 0, 0)) == 4 * 11008 * 32
    # invalid layouts size to zero
    assert lib.rb_planes_words(Layout(4096, 4000, 2, 0, 0, 0)) == 0
    assert lib.rb_planes_words(Layout(0, 4096, 2, 0, 0, 0)) == 0
    assert lib.rb_planes_words(Layout(16, 128, 9, 0, 0, 0)) == 0
    assert lib.rb_scales_count(Layout(16, 128, 2, 64, 0, 0)) == 0
    # the sliced order pads the last 512-column slice
    assert lib.rb_planes_words(Layout(4096, 11008, 2, 0, 1, 0)) == 2 * 4096 * 16 * 22
    assert lib.rb_planes_words(Layout(4096, 4096, 2, 0, 1, 0)) == 2 * 4096 * 128
    assert lib.rb_planes_words(Layout(16, 128, 2, 0, 2, 0)) == 0
    assert lib.rb_planes_words(Layout(16, 128, 2, 0, 0, 1)) == 0


def test_status_strings():
    lib = _lib.load()
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.rb_status_string(code).decode() == name


FAKE = 1 << 40          # a 16-byte aligned address that is never dereferenced


def _status(rc):
    return _lib.STATUS_NAMES[rc]


def test_pack_rejects_bad_arguments_before_launch():
    lib = _lib.load()
    L = Layout(64, 256, 2, 0, 0, 0)
    p = ctypes.c_void_p
    assert _status(lib.rb_pack(None, 0, 256, L, p(FAKE), p(FAKE), None, None)) == "RB_ERR_INVALID_ARG"
    assert _status(lib.rb_pack(p(FAKE), 0, 255, L, p(FAKE), p(FAKE), None, None)) == "RB_ERR_INVALID_ARG"
    assert _status(lib.rb_pack(p(FAKE), 7, 256, L, p(FAKE), p(FAKE), None, None)) == "RB_ERR_INVALID_ARG"
    assert _status(lib.rb_pack(p(FAKE + 4), 0, 256, L, p(FAKE), p(FAKE), None, None)) == "RB_ERR_ALIGNMENT"
    assert _status(lib.rb_pack(p(FAKE), 1, 260, L, p(FAKE), p(FAKE), None, None)) == "RB_ERR_ALIGNMENT"
    assert _status(lib.rb_pack(p(FAKE), 0, 256, L, p(FAKE + 8), p(FAKE), None, None)) == "RB_ERR_ALIGNMENT"
    assert _status(lib.rb_pack(p(FAKE), 0, 256, Layout(64, 200, 2, 0, 0, 0), p(FAKE), p(FAKE), None, None)) == \
        "RB_ERR_UNSUPPORTED"
    assert _status(lib.rb_pack(p(FAKE), 0, 256, Layout(64, 256, 0, 0, 0, 0), p(FAKE), p(FAKE), None, None)) == \
        "RB_ERR_UNSUPPORTED"
    assert _status(lib.rb_pack(p(FAKE), 0, 256, Layout(64, 256, 2, 32, 0, 0), p(FAKE), p(FAKE), None, None)) == \
        "RB_ERR_UNSUPPORTED"
    assert _status(lib.rb_pack(p(FAKE), 0, 1 << 17, Layout(4, 1 << 17, 2, 0, 0, 0), p(FAKE), p(FAKE), None, None)) == \
        "RB_ERR_UNSUPPORTED"
    lib.rb_pack(p(FAKE), 0, 256, Layout(64, 200, 2, 0, 0, 0), p(FAKE), p(FAKE), None, None)
    assert b"multiple of 128" in lib.rb_last_error()


def test_gemv_rejects_bad_arguments_before_launch():
    lib = _lib.load()
    L = Layout(64, 256, 2, 0, 0, 0)
    p = ctypes.c_void_p
    ok = (p(FAKE), p(FAKE), 0, L, p(FAKE), 256, 1, p(FAKE), 1, 64, p(FAKE), 1 << 20, None)

    def call(**kw):
        args = list(ok)
        names = ["planes", "alpha", "adt", "L", "x", "ldx", "T", "y", "ydt", "ldy", "ws", "wsb", "s"]
        for k, v in kw.items():
            args[names.index(k)] = v
        return _status(lib.rb_gemv(*args))

    assert call(planes=None) == "RB_ERR_INVALID_ARG"
    assert call(T=0) == "RB_ERR_UNSUPPORTED"
    assert call(T=65) == "RB_ERR_UNSUPPORTED"
    assert call(ldx=100) == "RB_ERR_INVALID_ARG"
    assert call(ldy=10) == "RB_ERR_INVALID_ARG"
    assert call(x=p(FAKE + 2)) == "RB_ERR_ALIGNMENT"
    assert call(ldx=260) == "RB_ERR_ALIGNMENT"
    assert call(ws=None) == "RB_ERR_WORKSPACE"
    assert call(wsb=8) == "RB_ERR_WORKSPACE"
    assert call(adt=5) == "RB_ERR_INVALID_ARG"
    assert call(L=Layout(64, 256, 9, 0, 0, 0)) == "RB_ERR_UNSUPPORTED"


def test_grouped_rejects_bad_descriptors():
    lib = _lib.load()
    p = ctypes.c_void_p
    d = (GemvDesc * 2)()
    d[0] = GemvDesc(FAKE, FAKE, FAKE, FAKE, 128, 256)
    d[1] = GemvDesc(FAKE, FAKE, FAKE, FAKE, 128, 200)
    host = ctypes.cast(d, p)
    rc = lib.rb_gemv_grouped(host, p(FAKE), 2, 2, 0, 0, 0, 1, 1, p(FAKE), 1 << 20, None)
    assert _status(rc) == "RB_ERR_UNSUPPORTED"
    assert b"descriptor 1" in lib.rb_last_error()
    d[1] = GemvDesc(FAKE, None, FAKE, FAKE, 128, 256)
    assert _status(lib.rb_gemv_grouped(host, p(FAKE), 2, 2, 0, 0, 0, 1, 1, p(FAKE), 1 << 20, None)) == \
        "RB_ERR_INVALID_ARG"
    d[1] = GemvDesc(FAKE, FAKE, FAKE, FAKE, 128, 256)
    assert _status(lib.rb_gemv_grouped(host, None, 2, 2, 0, 0, 0, 1, 1, p(FAKE), 1 << 20, None)) == \
        "RB_ERR_INVALID_ARG"
    assert _status(lib.rb_gemv_grouped(host, p(FAKE), 0, 2, 0, 0, 0, 1, 1, p(FAKE), 1 << 20, None)) == \
        "RB_ERR_UNSUPPORTED"
    assert lib.rb_gemv_grouped_workspace_bytes(host, 2, 2, 1) >= 256


def test_workspace_sizes_follow_the_split():
    lib = _lib.load()
    # one matrix with few rows is split along K, which needs counters and partial sums
    small = lib.rb_gemv_workspace_bytes(Layout(512, 8192, 2, 0, 0, 0), 1)
    assert small > 256 + 4 * 512
    # a layout that is rejected needs nothing
    assert lib.rb_gemv_workspace_bytes(Layout(512, 8000, 2, 0, 0, 0), 1) == 0


def test_missing_library_fails_loudly(monkeypatch):
    """Without librb.so the binding raises; there is no fallback path."""
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/librb.so")
    with pytest.raises(ImportError):
        _lib.load()


def test_grouped_checks_every_descriptor_alignment():
    """alpha and y of every descriptor, not only the first, must be aligned
    for their dtypes (a misaligned one would fault on the device)."""
    lib = _lib.load()
    p = ctypes.c_void_p
    d = (GemvDesc * 3)()
    for i in range(3):
        d[i] = GemvDesc(FAKE, FAKE, FAKE, FAKE, 128, 256)
    host = ctypes.cast(d, p)
    args = (host, p(FAKE), 3, 2, 0, 0, 0, 1, 1, p(FAKE), 1 << 20, None)   # fp32 alpha, fp16 y
    assert lib.rb_gemv_grouped_workspace_bytes(host, 3, 2, 1) <= 1 << 20
    d[2] = GemvDesc(FAKE, FAKE + 2, FAKE, FAKE, 128, 256)          # fp32 alpha at +2
    assert _status(lib.rb_gemv_grouped(*args)) == "RB_ERR_ALIGNMENT"
    assert b"descriptor 2" in lib.rb_last_error()
    d[2] = GemvDesc(FAKE, FAKE, FAKE, FAKE + 1, 128, 256)          # fp16 y at +1
    assert _status(lib.rb_gemv_grouped(*args)) == "RB_ERR_ALIGNMENT"
    assert b"descriptor 2" in lib.rb_last_error()
    d[1] = GemvDesc(FAKE, FAKE + 2, FAKE, FAKE, 128, 256)          # fp16 alpha at +2 is fine ...
    d[2] = GemvDesc(FAKE, FAKE, FAKE, FAKE, 128, 256)
    args16 = (host, p(FAKE), 3, 2, 0, 0, 1, 1, 1, p(FAKE), 8, None)  # ... but the workspace is too small
    assert _status(lib.rb_gemv_grouped(*args16)) == "RB_ERR_WORKSPACE"


def test_gemm_rejects_bad_arguments_before_launch():
    lib = _lib.load()
    p = ctypes.c_void_p
    L = Layout(256, 512, 2, 0, 0, 0)
    ok = [p(FAKE), p(FAKE), 0, L, p(FAKE), 512, 16, p(FAKE), 1, 256, p(FAKE), 1 << 30, None]
    names = ["planes", "alpha", "adt", "L", "X", "ldx", "T", "Y", "ydt", "ldy", "ws", "wsb", "s"]

    def call(**kw):
        args = list(ok)
        for k, v in kw.items():
            args[names.index(k)] = v
        return _status(lib.rb_gemm(*args))

    assert call(planes=None) == "RB_ERR_INVALID_ARG"
    assert call(T=0) == "RB_ERR_UNSUPPORTED"
    assert call(T=(1 << 22) + 1) == "RB_ERR_UNSUPPORTED"
    assert call(L=Layout(256, 512, 5, 0, 0, 0)) == "RB_ERR_UNSUPPORTED"
    # fp32 scales per 128 columns would be rounded to fp16 operands: refused
    assert call(L=Layout(256, 512, 2, 128, 0, 0), adt=0) == "RB_ERR_UNSUPPORTED"
    assert b"fp16 scales" in lib.rb_last_error()
    assert call(ldx=500) == "RB_ERR_INVALID_ARG"
    assert call(X=p(FAKE + 8)) == "RB_ERR_ALIGNMENT"
    assert call(alpha=p(FAKE + 2)) == "RB_ERR_ALIGNMENT"
    assert call(Y=p(FAKE + 1)) == "RB_ERR_ALIGNMENT"
    assert call(ws=None) == "RB_ERR_WORKSPACE"
    need = lib.rb_gemm_workspace_bytes(L, 16)
    assert call(wsb=need - 1) == "RB_ERR_WORKSPACE"
    assert call(ws=p(FAKE + 8)) == "RB_ERR_WORKSPACE"


def test_gemm_workspace_sizes():
    """Decode batches (T <= 64) need the header, one counter per 128-row tile,
    two partial-sum slots per CTA and a permuted copy of X; prefill blocks
    only the header."""
    lib = _lib.load()
    L = Layout(28672, 8192, 2, 0, 1, 0)
    for T in (1, 16, 64):
        b = lib.rb_gemm_workspace_bytes(L, T)
        bn = 16 if T <= 16 else 32 if T <= 32 else 64
        assert b >= 256 + 4 * 224 + T * 8192 * 2 + 2 * bn * 128 * 4
    assert lib.rb_gemm_workspace_bytes(L, 65) == 256
    assert lib.rb_gemm_workspace_bytes(L, 2048) == 256
    assert lib.rb_gemm_workspace_bytes(L, 0) == 0
    assert lib.rb_gemm_workspace_bytes(Layout(28672, 8000, 2, 0, 1, 0), 16) == 0


def test_dual_block_rejects_bad_arguments_before_launch():
    lib = _lib.load()
    p = ctypes.c_void_p
    L = Layout(64, 256, 2, 0, 0, 0)
    assert _status(lib.rb_pack_fixed(p(FAKE), 0, 256, Layout(64, 256, 2, 128, 0, 0), p(FAKE), None, p(FAKE),
                                     None)) == "RB_ERR_UNSUPPORTED"
    assert _status(lib.rb_pack_fixed(p(FAKE), 0, 256, L, None, None, p(FAKE), None)) == "RB_ERR_INVALID_ARG"
    assert _status(lib.rb_pack_fixed(p(FAKE), 0, 256, L, p(FAKE + 2), None, p(FAKE), None)) == "RB_ERR_ALIGNMENT"
    assert _status(lib.rb_pack_fixed(p(FAKE), 0, 256, L, p(FAKE), p(FAKE + 1), p(FAKE), None)) == "RB_ERR_ALIGNMENT"
    need = lib.rb_dual_gemv_workspace_bytes(L, 4)
    assert need > 256
    assert lib.rb_dual_gemv_workspace_bytes(Layout(64, 256, 2, 128, 0, 0), 4) == 0
    ok = [p(FAKE), L, p(FAKE), p(FAKE), p(FAKE), 256, 4, p(FAKE), 1, 64, p(FAKE), need, None]
    names = ["planes", "L", "h", "g", "x", "ldx", "T", "y", "ydt", "ldy", "ws", "wsb", "s"]

    def call(**kw):
        args = list(ok)
        for k, v in kw.items():
            args[names.index(k)] = v
        return _status(lib.rb_dual_gemv(*args))

    assert call(L=Layout(64, 256, 2, 128, 0, 0)) == "RB_ERR_UNSUPPORTED"
    assert call(T=65) == "RB_ERR_UNSUPPORTED"
    assert call(h=None) == "RB_ERR_INVALID_ARG"
    assert call(g=p(FAKE + 2)) == "RB_ERR_ALIGNMENT"
    assert call(x=p(FAKE + 2)) == "RB_ERR_ALIGNMENT"
    assert call(wsb=need - 1) == "RB_ERR_WORKSPACE"


def test_gemm_from_weight_rejections():
    """Refused before anything is enqueued (no GPU needed)."""
    lib = _lib.load()
    p = ctypes.c_void_p
    L = Layout(256, 1024, 2, 0, 1, 0)
    need = lib.rb_gemm_from_weight_workspace_bytes(L, 300)
    assert need >= 256 + 2 * 256 * 1024 // 8 + 2 * 256 * 4
    args = dict(W=p(FAKE), wd=1, ldw=1024, X=p(FAKE), ldx=1024, T=300, Y=p(FAKE), yd=1, ldy=256)

    def call(L=L, ws=need, **kw):
        a = dict(args, **kw)
        return _status(lib.rb_gemm_from_weight(a["W"], a["wd"], a["ldw"], L, a["X"], a["ldx"], a["T"], a["Y"],
                                               a["yd"], a["ldy"], p(FAKE), ws, None))
    assert call(W=None) == "RB_ERR_INVALID_ARG"
    assert call(L=Layout(256, 1024, 5, 0, 1, 0)) == "RB_ERR_UNSUPPORTED"
    assert call(ldw=1000) == "RB_ERR_INVALID_ARG"
    assert call(W=p(FAKE + 8)) == "RB_ERR_ALIGNMENT"
    assert call(T=0) == "RB_ERR_UNSUPPORTED"
    assert call(ldy=100) == "RB_ERR_INVALID_ARG"
    assert call(ws=need - 16) == "RB_ERR_WORKSPACE"
    assert lib.rb_gemm_from_weight_workspace_bytes(Layout(256, 1000, 2, 0, 1, 0), 300) == 0


def test_matvec_workspace_layout_and_counter_zone():
    """A K-split plan needs the 256-byte header, the fixed 64 KB counter zone
    and its fp32 partial sums; a plan that would need more counters than the
    zone holds does not split (header only); the SiLU-gated pair keeps two
    partial sums per row."""
    lib = _lib.load()
    L = Layout(512, 8192, 2, 0, 1, 0)
    b = lib.rb_gemv_workspace_bytes(L, 1)
    assert b > 256 + 65536 and (b - 256 - 65536) % (4 * 512) == 0   # partials: nch x T x M fp32
    nch = (b - 256 - 65536) // (4 * 512)
    assert nch >= 2
    # 257 row blocks of 512 rows x 64 tokens = 16448 counters > 16384: no split
    assert lib.rb_gemv_workspace_bytes(Layout(512 * 257, 8192, 2, 0, 1, 0), 64) == 256
    g = lib.rb_gemv_swiglu_workspace_bytes(Layout(512, 8192, 1, 0, 1, 0), 1)
    assert g > 256 + 65536 and (g - 256 - 65536) % (2 * 4 * 512) == 0   # two sums per row and chunk
    assert lib.rb_gemv_swiglu_workspace_bytes(Layout(512, 8192, 5, 0, 1, 0), 1) == 0   # > 4 paths per matrix


def test_swiglu_rejections():
    lib = _lib.load()
    p = ctypes.c_void_p
    L = Layout(256, 1024, 2, 0, 1, 0)
    ws = lib.rb_gemv_swiglu_workspace_bytes(L, 1)

    def call(L=L, **kw):
        a = dict(planes=p(FAKE), alpha=p(FAKE), x=p(FAKE), T=1, h=p(FAKE), ldh=256)
        a.update(kw)
        return _status(lib.rb_gemv_swiglu(a["planes"], a["alpha"], 0, L, a["x"], 1024, a["T"], a["h"], 1, a["ldh"],
                                          p(FAKE), max(ws, 256), None))
    assert call(planes=None) == "RB_ERR_INVALID_ARG"
    assert call(L=Layout(256, 1024, 5, 0, 1, 0)) == "RB_ERR_UNSUPPORTED"
    assert call(T=65) == "RB_ERR_UNSUPPORTED"
    assert call(ldh=100) == "RB_ERR_INVALID_ARG"
    assert call(h=p(FAKE + 1)) == "RB_ERR_ALIGNMENT"
