"""Host-only checks of the C ABI: the libraries load, export every declared symbol, and reject bad
arguments before anything is launched (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

import oracle
from delta_rule_sequence_b200 import prism as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(prism_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from delta_rule_sequence_b200 import build

    build.build()
    return P.load_library()


def test_prism_h_symbols_exported(lib):
    names = _declared("prism.h")
    assert set(names) == set(P.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), n


def test_prism_ref_h_symbols_exported():
    lib = ctypes.CDLL(oracle.build())
    for n in _declared("prism_ref.h"):
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in enumerate(["PRISM_OK", "PRISM_ERR_INVALID_ARG", "PRISM_ERR_UNSUPPORTED",
                                 "PRISM_ERR_CUDA", "PRISM_ERR_TIMEOUT"]):
        assert P.status_string(code) == name
    assert P.status_string(99) == "PRISM_ERR_UNKNOWN"


def _shape(**kw):
    base = dict(B=1, H=2, T=256, dk=32, dv=32, L=1, chunk=64, io=P.PRISM_F32)
    base.update(kw)
    return P.PrismShape(**base)


FAKE = ctypes.c_void_p(0x10000)       # 16-byte aligned, never dereferenced: calls fail before launch
MISALIGNED = ctypes.c_void_p(0x10004)


def _fwd(lib, shape, q=FAKE, k=FAKE, v=FAKE, a=FAKE, b=FAKE, u=None, w=None, S0=None, o=FAKE,
         Sf=None, ws=ctypes.c_void_p(0x20000), ws_bytes=256):
    return lib.prism_scan_fwd(ctypes.byref(shape), q, k, v, a, b, u, w, S0, o, Sf, ws,
                              ctypes.c_size_t(ws_bytes), None)


@pytest.mark.parametrize("kw,expect", [
    (dict(dk=48), P.PRISM_ERR_UNSUPPORTED),
    (dict(dv=256), P.PRISM_ERR_UNSUPPORTED),
    (dict(L=0), P.PRISM_ERR_INVALID_ARG),
    (dict(L=9), P.PRISM_ERR_UNSUPPORTED),
    (dict(L=2), P.PRISM_ERR_INVALID_ARG),       # u, w NULL needs L == 1
    (dict(chunk=32), P.PRISM_ERR_INVALID_ARG),
    (dict(T=-1), P.PRISM_ERR_INVALID_ARG),
    (dict(io=7), P.PRISM_ERR_INVALID_ARG),
])
def test_scan_rejects_bad_shapes(lib, kw, expect):
    assert _fwd(lib, _shape(**kw)) == expect


def test_scan_rejects_bad_pointers(lib):
    s = _shape()
    assert _fwd(lib, s, q=None) == P.PRISM_ERR_INVALID_ARG
    assert _fwd(lib, s, v=None) == P.PRISM_ERR_INVALID_ARG          # GDN write needs v
    assert _fwd(lib, s, u=FAKE) == P.PRISM_ERR_INVALID_ARG          # u without w
    assert _fwd(lib, s, k=MISALIGNED) == P.PRISM_ERR_INVALID_ARG
    assert _fwd(lib, s, o=None) == P.PRISM_ERR_INVALID_ARG
    assert _fwd(lib, s, o=FAKE, q=FAKE) == P.PRISM_ERR_INVALID_ARG  # o aliases q
    assert _fwd(lib, s, ws=None) == P.PRISM_ERR_INVALID_ARG
    assert _fwd(lib, s, ws_bytes=8) == P.PRISM_ERR_INVALID_ARG
    assert _fwd(lib, s, ws=ctypes.c_void_p(0x20010)) == P.PRISM_ERR_INVALID_ARG  # not 256-aligned
    assert lib.prism_scan_fwd(None, *([None] * 10), None, 0, None) == P.PRISM_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(lib):
    s = _shape(T=2)
    args = [FAKE] * 5 + [None, None, FAKE, FAKE, None]
    assert lib.prism_step_decode(ctypes.byref(s), *args) == P.PRISM_ERR_INVALID_ARG  # T != 1
    s = _shape(T=1)
    bad = [FAKE] * 5 + [None, None, None, FAKE, None]
    assert lib.prism_step_decode(ctypes.byref(s), *bad) == P.PRISM_ERR_INVALID_ARG  # S NULL


def test_producer_rejects_bad_arguments(lib):
    def call(shape, x=FAKE, v=FAKE, conv=FAKE, Wk=FAKE, Wp=FAKE, beta=FAKE,
             u=ctypes.c_void_p(0x30000), w=ctypes.c_void_p(0x40000)):
        return lib.prism_write_producer(ctypes.byref(shape), x, v, conv, Wk, Wp, beta, u, w, None)

    ok = dict(dk=64, dv=64, L=3, io=P.PRISM_BF16)
    assert call(_shape(**dict(ok, T=0))) == P.PRISM_OK                       # nothing to do
    assert call(_shape(**dict(ok, dk=32, dv=32))) == P.PRISM_ERR_UNSUPPORTED
    assert call(_shape(**dict(ok, dv=128))) == P.PRISM_ERR_UNSUPPORTED      # dk != dv
    assert call(_shape(**dict(ok, io=P.PRISM_F32))) == P.PRISM_ERR_UNSUPPORTED
    assert call(_shape(**dict(ok, L=0))) == P.PRISM_ERR_INVALID_ARG
    assert call(_shape(**dict(ok, L=65))) == P.PRISM_ERR_UNSUPPORTED
    assert call(_shape(**ok), x=None) == P.PRISM_ERR_INVALID_ARG
    assert call(_shape(**ok), Wp=MISALIGNED) == P.PRISM_ERR_INVALID_ARG
    assert call(_shape(**ok), beta=ctypes.c_void_p(0x10002)) == P.PRISM_ERR_INVALID_ARG
    assert call(_shape(**ok), u=FAKE) == P.PRISM_ERR_INVALID_ARG             # u aliases the inputs
    assert call(_shape(**ok), w=ctypes.c_void_p(0x30000)) == P.PRISM_ERR_INVALID_ARG  # u == w
    assert lib.prism_write_producer(None, *([None] * 8), None) == P.PRISM_ERR_INVALID_ARG


def test_launch_probe_arguments(lib):
    assert lib.prism_debug_record_launch_events(None, -1) == P.PRISM_ERR_INVALID_ARG
    assert lib.prism_debug_record_launch_events(None, 2) == P.PRISM_ERR_INVALID_ARG
    null_handles = (ctypes.c_void_p * 2)(None, None)
    assert lib.prism_debug_record_launch_events(null_handles, 2) == P.PRISM_ERR_INVALID_ARG
    many = (ctypes.c_void_p * 65)(*([1] * 65))
    assert lib.prism_debug_record_launch_events(many, 65) == P.PRISM_ERR_UNSUPPORTED
    assert lib.prism_debug_record_launch_events(None, 0) == P.PRISM_OK  # disarm


def test_workspace_size(lib):
    n = ctypes.c_size_t(0)
    assert lib.prism_scan_fwd_workspace_size(ctypes.byref(_shape()), ctypes.byref(n)) == 0
    assert n.value >= 256
    assert lib.prism_scan_fwd_workspace_size(None, ctypes.byref(n)) == P.PRISM_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(P, "_lib", None)
    monkeypatch.setattr(P, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        P.load_library()


def test_binding_refuses_cpu_tensors():
    import torch

    x = torch.zeros((1, 4, 1, 32))
    with pytest.raises(TypeError, match="CUDA"):
        P.prism_scan_fwd(x, x, x, torch.ones(1, 4, 1), torch.zeros(1, 4, 1))


def _bwd(lib, shape, q=FAKE, k=FAKE, v=FAKE, a=FAKE, b=FAKE, u=None, w=None, S0=None,
         dO=ctypes.c_void_p(0x50000), dSf=None, dq=ctypes.c_void_p(0x60000),
         dk=ctypes.c_void_p(0x70000), dv=ctypes.c_void_p(0x80000), da=ctypes.c_void_p(0x90000),
         db=ctypes.c_void_p(0xA0000), du=None, dw=None, dS0=None, ws=ctypes.c_void_p(0x100000),
         ws_bytes=1 << 30):
    return lib.prism_scan_bwd(ctypes.byref(shape), q, k, v, a, b, u, w, S0, dO, dSf, dq, dk, dv,
                              da, db, du, dw, dS0, ws, ctypes.c_size_t(ws_bytes), None)


def test_backward_rejects_bad_arguments(lib):
    s = _shape()
    assert _bwd(lib, _shape(dk=48)) == P.PRISM_ERR_UNSUPPORTED
    assert _bwd(lib, _shape(L=0)) == P.PRISM_ERR_INVALID_ARG
    assert _bwd(lib, s, dO=None) == P.PRISM_ERR_INVALID_ARG
    assert _bwd(lib, s, dq=None) == P.PRISM_ERR_INVALID_ARG
    assert _bwd(lib, s, dv=None) == P.PRISM_ERR_INVALID_ARG                 # GDN write needs dv
    assert _bwd(lib, s, dk=ctypes.c_void_p(0x60000)) == P.PRISM_ERR_INVALID_ARG  # dk overlaps dq
    assert _bwd(lib, s, dq=FAKE) == P.PRISM_ERR_INVALID_ARG                 # dq overlaps q
    assert _bwd(lib, s, da=MISALIGNED) == P.PRISM_ERR_INVALID_ARG
    assert _bwd(lib, s, ws_bytes=8) == P.PRISM_ERR_INVALID_ARG
    rank = _shape(L=2)
    u, w = ctypes.c_void_p(0xB0000), ctypes.c_void_p(0xC0000)
    assert _bwd(lib, rank, u=u, w=w) == P.PRISM_ERR_INVALID_ARG              # rank L needs du, dw
    assert _bwd(lib, rank, u=u, w=w, du=ctypes.c_void_p(0xD0000)) == P.PRISM_ERR_INVALID_ARG
    assert lib.prism_scan_bwd(None, *([None] * 18), None, 0, None) == P.PRISM_ERR_INVALID_ARG
    n = ctypes.c_size_t(0)
    assert lib.prism_scan_bwd_workspace_size(ctypes.byref(s), ctypes.byref(n)) == P.PRISM_OK
    assert n.value >= 4 * 2 * 4 * 32 * 32  # at least the chunk-start states
    assert lib.prism_scan_bwd_workspace_size(None, ctypes.byref(n)) == P.PRISM_ERR_INVALID_ARG


def test_noalloc_rejects_like_the_workspace_entry(lib):
    """Checked before any sizing: the same status codes as prism_scan_fwd for malformed shapes."""
    for kw in (dict(B=-1, dk=64, dv=64, io=P.PRISM_BF16), dict(dk=48), dict(chunk=32), dict(L=0),
               dict(L=9), dict(io=7)):
        s = _shape(**kw)
        rc = lib.prism_scan_fwd_noalloc(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
                                        None, ctypes.c_void_p(0x20000), None, None)
        assert rc == _fwd(lib, s, o=ctypes.c_void_p(0x20000)), kw
        assert rc != P.PRISM_OK
