"""The C ABI on a machine without a GPU: the library loads, exports every
symbol its header declares, and rejects bad arguments on the host before any
CUDA call."""

import ctypes
import os
import re

import pytest

from prefill_eviction_scoring_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "waits.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(waits_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_bound_functions():
    assert _declared() == sorted(_lib.SIGNATURES)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_version_and_strerror(lib):
    assert lib.waits_abi_version() == 1
    for st in range(8):
        assert len(lib.waits_strerror(st)) >= 2
    assert b"unknown" in lib.waits_strerror(99)


FAKE = 0x100000   # never dereferenced: every call below fails validation


def _shape(**kw):
    d = dict(nseq=1, total_tokens=4096, max_seqlen=4096, num_q_heads=32,
             num_kv_heads=8, head_dim=128, cu_seqlens=FAKE)
    d.update(kw)
    return _lib.Shape(**d)


def _ws(lib, shape):
    n = ctypes.c_size_t(0)
    st = lib.waits_workspace_size(ctypes.byref(shape), ctypes.byref(n))
    return st, n.value


def test_workspace_size_host_only(lib):
    st, n = _ws(lib, _shape())
    assert st == 0 and n > 0
    st2, n2 = _ws(lib, _shape(total_tokens=8192, max_seqlen=8192))
    assert st2 == 0 and n2 > n
    assert lib.waits_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == 1
    assert lib.waits_workspace_size(ctypes.byref(_shape()), None) == 1


@pytest.mark.parametrize("kw,want", [
    (dict(nseq=0), 2), (dict(total_tokens=0), 2), (dict(num_q_heads=30), 2),
    (dict(head_dim=96), 3), (dict(head_dim=256), 3),
    (dict(num_q_heads=256, num_kv_heads=1), 3), (dict(max_seqlen=5000), 2),
    (dict(cu_seqlens=0), 1), (dict(nseq=5000), 2)])
def test_shape_errors(lib, kw, want):
    assert _ws(lib, _shape(**kw))[0] == want


def test_score_argument_errors(lib):
    sh = _shape()
    _, n = _ws(lib, sh)
    W = 0x200000
    call = lambda Q=FAKE, K=FAKE, a=1.0, b=16, s=FAKE, ws=W, nb=n: lib.waits_score(
        ctypes.byref(sh), Q, K, a, b, s, ws, nb, None)
    assert call(Q=None) == 1
    assert call(K=None) == 1
    assert call(s=None) == 1
    assert call(Q=FAKE + 8) == 1                    # 16-byte alignment
    assert call(a=-1.0) == 1
    assert call(a=float("nan")) == 1
    assert call(a=float("inf")) == 1
    assert call(b=-1) == 1
    assert call(ws=None) == 4
    assert call(nb=n - 1) == 4
    assert call(ws=W + 16) == 1                     # 256-byte alignment


def test_select_compact_compress_errors(lib):
    sh = _shape()
    _, n = _ws(lib, sh)
    assert lib.waits_select(ctypes.byref(sh), FAKE, 17, 16, FAKE, FAKE, None, 0, None) == 1
    assert lib.waits_select(ctypes.byref(sh), FAKE, -1, 16, FAKE, FAKE, None, 0, None) == 1
    assert lib.waits_select(ctypes.byref(sh), FAKE, 0, 0, FAKE, FAKE, None, 0, None) == 1
    assert lib.waits_select(ctypes.byref(sh), None, 1, 16, FAKE, FAKE, None, 0, None) == 1
    assert lib.waits_compact(ctypes.byref(sh), FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE,
                             None, 0, None) == 1
    assert lib.waits_compact(ctypes.byref(sh), FAKE, FAKE + 4, FAKE, FAKE, 16, FAKE, FAKE,
                             None, 0, None) == 1
    assert lib.waits_compress(ctypes.byref(sh), FAKE, FAKE, FAKE, 1.0, 16, 32, 16, FAKE,
                              FAKE, FAKE, FAKE, FAKE, 0x200000, n, None) == 1
    assert lib.waits_compress(ctypes.byref(sh), FAKE, FAKE, FAKE, 1.0, 16, 16, 128, FAKE,
                              FAKE, FAKE, FAKE, FAKE, 0x200000, 10, None) == 4


def test_select_compact_argument_errors(lib):
    """waits_select_compact validates like waits_select and waits_compact
    together, on the host, before any launch."""
    sh = _shape()
    call = lambda scores=FAKE, K=FAKE, V=FAKE, R=16, B=128, idx=FAKE, kept=FAKE, Ko=FAKE, \
        Vo=FAKE: lib.waits_select_compact(ctypes.byref(sh), scores, K, V, R, B, idx, kept, Ko,
                                          Vo, None, 0, None)
    assert call(scores=None) == 1
    assert call(R=17, B=16) == 1                    # R > B
    assert call(R=-1) == 1
    assert call(B=0) == 1
    assert call(idx=None) == 1
    assert call(kept=None) == 1
    assert call(K=None) == 1
    assert call(V=None) == 1
    assert call(Ko=None) == 1
    assert call(Vo=None) == 1
    assert call(V=FAKE + 4) == 1                    # K/V rows must be 16-byte aligned
    bad = _shape(nseq=0)
    assert lib.waits_select_compact(ctypes.byref(bad), FAKE, FAKE, FAKE, 16, 128, FAKE, FAKE,
                                    FAKE, FAKE, None, 0, None) == 2


def test_host_variant_validates_offsets(lib):
    sh = _shape(nseq=2, total_tokens=100, max_seqlen=60)
    _, n = _ws(lib, sh)
    cu_bad = (ctypes.c_int32 * 3)(0, 70, 100)       # 70 > max_seqlen
    cu_bad2 = (ctypes.c_int32 * 3)(0, 40, 90)       # does not end at T
    bufs = _lib.DeviceBuffers(*([FAKE] * 9))
    for cu in (cu_bad, cu_bad2):
        st = lib.waits_compress_host(ctypes.byref(sh), cu, FAKE, FAKE, FAKE, 1.0, 16, 16,
                                     128, FAKE, FAKE, FAKE, FAKE, ctypes.byref(bufs),
                                     0x200000, n, None, None, None)
        assert st == 2


def test_status_read_needs_out_pointer(lib):
    assert lib.waits_read_device_status(0x200000, 4096, None, None) == 1
    assert lib.waits_read_device_status(None, 4096, None,
                                        ctypes.byref(ctypes.c_uint32())) == 4


def test_python_binding_fails_loudly_without_library(tmp_path):
    saved = _lib._lib
    _lib._lib = None
    try:
        with pytest.raises(_lib.WaitsLibraryError):
            _lib.load(str(tmp_path / "missing.so"))
    finally:
        _lib._lib = saved


def _kernels(lib, shape, a, b):
    n = ctypes.c_int32(0)
    st = lib.waits_score_kernels(ctypes.byref(shape), a, b, ctypes.byref(n))
    return st, n.value


def test_score_kernel_count(lib, monkeypatch):
    """Small plans are rebuilt inside the scorer (2 kernels); large ones take
    the planner kernel first and merge the row biases between the passes (4;
    3 with the general kernel forced for both passes)."""
    monkeypatch.delenv("WAITS_SCORER", raising=False)
    llama8b = _shape(total_tokens=32768, max_seqlen=32768)
    assert _kernels(lib, llama8b, 1.0, 16) == (0, 2)     # ~105 active rows: 4 Q tiles
    assert _kernels(lib, llama8b, 10.0, 1) == (0, 2)
    assert _kernels(lib, llama8b, 0.0, 16) == (0, 4)     # every row active
    assert _kernels(lib, llama8b, 0.01, 128) == (0, 4)   # ~9000 active rows
    batch = _shape(nseq=40, total_tokens=40 * 512, max_seqlen=512, num_kv_heads=4,
                   num_q_heads=28)
    assert _kernels(lib, batch, 1.0, 16) == (0, 4)        # more than 32 sequences
    two = _shape(nseq=2, total_tokens=2 * 8192, max_seqlen=8192)
    assert _kernels(lib, two, 1.0, 16) == (0, 2)          # 8 heads x 2 x 2 = 32 pass-1 entries
    three = _shape(nseq=3, total_tokens=3 * 8192, max_seqlen=8192)
    assert _kernels(lib, three, 1.0, 16) == (0, 4)        # 48 pass-1 entries
    monkeypatch.setenv("WAITS_SCORER", "tc")
    assert _kernels(lib, three, 1.0, 16) == (0, 3)        # general kernel, no bias merge
    assert _kernels(lib, llama8b, -1.0, 16)[0] == 1
    assert _kernels(lib, llama8b, 1.0, -1)[0] == 1
    assert lib.waits_score_kernels(ctypes.byref(llama8b), 1.0, 16, None) == 1


def test_decode_argument_errors(lib):
    n = ctypes.c_size_t(0)
    assert lib.waits_decode_workspace_size(1, 32, 128, 2048, None) == 1
    assert lib.waits_decode_workspace_size(1, 32, 96, 2048, ctypes.byref(n)) == 3
    assert lib.waits_decode_workspace_size(1, 32, 128, 2048, ctypes.byref(n)) == 0
    assert n.value == 32 * 8 * 130 * 4
    F = 0x100000

    def call(nseq=1, Hq=32, Hkv=8, d=128, C=2048, q=F, k=F, v=F, ln=F, out=F, ws=F, wsb=10**7):
        return lib.waits_decode_attention(nseq, Hq, Hkv, d, C, q, k, v, ln, out, None, ws, wsb,
                                          None)

    assert call(Hq=30) == 2                 # Hq not a multiple of Hkv
    assert call(d=80) == 3                  # head dim
    assert call(Hq=32, Hkv=1) == 3          # G > 16
    assert call(q=0) == 1 and call(out=0) == 1
    assert call(q=F + 8) == 1               # 16-byte alignment
    assert call(wsb=16) == 4                # workspace too small
