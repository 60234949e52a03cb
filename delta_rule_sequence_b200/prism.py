"""ctypes binding of libprism.so (C ABI in include/prism.h).

Argument marshalling only: shapes are read from torch tensors, outputs and workspace are
allocated with torch when the caller does not pass them, and every step of the computation runs
in the library's CUDA kernels on the current torch stream.  There is no CPU fallback: if the
library is missing or the tensors are not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libprism.so")

PRISM_OK, PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED, PRISM_ERR_CUDA, PRISM_ERR_TIMEOUT = range(5)
PRISM_BF16, PRISM_F32 = 0, 1

# Every symbol that include/prism.h declares.
EXPORTS = (
    "prism_scan_fwd_workspace_size",
    "prism_scan_fwd_launch_count",
    "prism_scan_fwd",
    "prism_scan_fwd_noalloc",
    "prism_scan_bwd_workspace_size",
    "prism_scan_bwd",
    "prism_scan_segment_element",
    "prism_state_fold",
    "prism_step_decode",
    "prism_write_producer",
    "prism_query_device_status",
    "prism_status_string",
    "prism_last_cuda_error",
    "prism_debug_set_flags",
    "prism_debug_record_launch_events",
)


class PrismError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == PRISM_ERR_CUDA:
            try:
                detail = load_library().prism_last_cuda_error().decode()
            except RuntimeError:
                pass
        super().__init__(f"{where}: {status_string(status)} ({status})" + (f": {detail}" if detail else ""))


class PrismShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("L", ctypes.c_int),
                ("chunk", ctypes.c_int), ("io", ctypes.c_int)]


_lib = None


def load_library():
    """Load libprism.so (built in-tree by delta_rule_sequence_b200.build); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libprism.so is not built ({LIB_PATH}); run `python -m delta_rule_sequence_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, ci = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    shp = ctypes.POINTER(PrismShape)
    lib.prism_scan_fwd_workspace_size.argtypes = [shp, ctypes.POINTER(sz)]
    lib.prism_scan_fwd_workspace_size.restype = ci
    lib.prism_scan_fwd_launch_count.argtypes = [shp, ctypes.POINTER(ci)]
    lib.prism_scan_fwd_launch_count.restype = ci
    lib.prism_scan_fwd.argtypes = [shp] + [vp] * 10 + [vp, sz, vp]
    lib.prism_scan_fwd.restype = ci
    lib.prism_scan_fwd_noalloc.argtypes = [shp] + [vp] * 10 + [vp]
    lib.prism_scan_fwd_noalloc.restype = ci
    lib.prism_scan_bwd_workspace_size.argtypes = [shp, ctypes.POINTER(sz)]
    lib.prism_scan_bwd_workspace_size.restype = ci
    lib.prism_scan_bwd.argtypes = [shp] + [vp] * 18 + [vp, sz, vp]
    lib.prism_scan_bwd.restype = ci
    lib.prism_scan_segment_element.argtypes = [shp] + [vp] * 9 + [vp, sz, vp]
    lib.prism_scan_segment_element.restype = ci
    lib.prism_state_fold.argtypes = [ci, ci, ci, vp, vp, vp, vp, vp]
    lib.prism_state_fold.restype = ci
    lib.prism_step_decode.argtypes = [shp] + [vp] * 9 + [vp]
    lib.prism_step_decode.restype = ci
    lib.prism_write_producer.argtypes = [shp] + [vp] * 8 + [vp]
    lib.prism_write_producer.restype = ci
    lib.prism_query_device_status.argtypes = [vp, vp]
    lib.prism_query_device_status.restype = ci
    lib.prism_status_string.argtypes = [ci]
    lib.prism_status_string.restype = ctypes.c_char_p
    lib.prism_last_cuda_error.argtypes = []
    lib.prism_last_cuda_error.restype = ctypes.c_char_p
    lib.prism_debug_set_flags.argtypes = [ci]
    lib.prism_debug_set_flags.restype = ci
    lib.prism_debug_record_launch_events.argtypes = [ctypes.POINTER(vp), ci]
    lib.prism_debug_record_launch_events.restype = ci
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load_library().prism_status_string(int(status)).decode()
    except RuntimeError:
        return f"status {status}"


def _ptr(x):
    return None if x is None else ctypes.c_void_p(x.data_ptr())


def _stream(stream, device):
    """The stream to launch on: the caller's (which must belong to `device`), else the current
    stream of `device` (not of whichever device happens to be current)."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors are on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _call(device, fn, *args):
    """Run a library entry point with `device` current (the library launches on the current
    device and looks up per-device state there)."""
    with torch.cuda.device(device):
        return fn(*args)


def _check_tensor(name, x, dtype, shape, device):
    if x is None:
        return
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (libprism has no CPU path)")
    if x.device != device:
        raise ValueError(f"{name} is on {x.device}, q is on {device}")
    if x.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {x.dtype}")
    if tuple(x.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(x.shape)}")
    if not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_shape(q, v=None, u=None, chunk=64, L=None) -> PrismShape:
    B, T, H, dk = q.shape
    if u is not None:
        Lr, dv = u.shape[3], u.shape[4]
    else:
        Lr, dv = 1, v.shape[3]
    io = PRISM_F32 if q.dtype == torch.float32 else PRISM_BF16
    return PrismShape(B, H, T, dk, dv, L or Lr, chunk, io)


_ws_cache = {}


def workspace_for(shape: PrismShape, device) -> torch.Tensor:
    """A cached device workspace of the size prism_scan_fwd needs (one per device/size)."""
    need = ctypes.c_size_t(0)
    rc = load_library().prism_scan_fwd_workspace_size(ctypes.byref(shape), ctypes.byref(need))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_fwd_workspace_size")
    key = (str(device), int(need.value))
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(max(256, int(need.value)), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def prism_scan_fwd(q, k, v, alpha, beta, u=None, w=None, S0=None, *, chunk=64, o=None,
                   S_final=None, want_state=True, workspace=None, stream=None):
    """Chunked scan forward.  q, k: [B,T,H,dk]; v: [B,T,H,dv] or None; alpha, beta: [B,T,H]
    fp32; u: [B,T,H,L,dv] / w: [B,T,H,L,dk] or None; S0: [B,H,dv,dk] fp32 or None.
    Returns (o [B,T,H,dv], S_final [B,H,dv,dk] fp32 or None)."""
    lib = load_library()
    if not isinstance(q, torch.Tensor) or not q.is_cuda:
        raise TypeError("q must be a CUDA tensor (libprism has no CPU path)")
    dev, io = q.device, q.dtype
    shape = make_shape(q, v, u, chunk)
    B, T, H, dk = q.shape
    dv, L = shape.dv, shape.L
    _check_tensor("q", q, io, (B, T, H, dk), dev)
    _check_tensor("k", k, io, (B, T, H, dk), dev)
    _check_tensor("v", v, io, (B, T, H, dv), dev)
    _check_tensor("alpha", alpha, torch.float32, (B, T, H), dev)
    _check_tensor("beta", beta, torch.float32, (B, T, H), dev)
    _check_tensor("u", u, io, (B, T, H, L, dv), dev)
    _check_tensor("w", w, io, (B, T, H, L, dk), dev)
    _check_tensor("S0", S0, torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=io, device=dev)
    _check_tensor("o", o, io, (B, T, H, dv), dev)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    _check_tensor("S_final", S_final, torch.float32, (B, H, dv, dk), dev)
    if workspace is None:
        workspace = workspace_for(shape, dev)
    _check_tensor("workspace", workspace, torch.uint8, (workspace.numel(),), dev)
    rc = _call(dev, lib.prism_scan_fwd, ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
               _ptr(beta), _ptr(u), _ptr(w), _ptr(S0), _ptr(o), _ptr(S_final),
               _ptr(workspace), ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_fwd")
    return o, S_final


def prism_scan_fwd_noalloc(q, k, v, alpha, beta, u=None, w=None, S0=None, *, chunk=64, o, S_final,
                           stream=None):
    """prism_scan_fwd without a workspace, for callers that cannot allocate device memory when
    they run the scan: the library uses its own fixed device scratch instead.  The caller passes
    every output (o, S_final or None) already allocated; this wrapper allocates nothing.  Calls
    whose kernels overlap on the GPU share that scratch and race: keep them on one stream."""
    lib = load_library()
    if not isinstance(q, torch.Tensor) or not q.is_cuda:
        raise TypeError("q must be a CUDA tensor (libprism has no CPU path)")
    dev, io = q.device, q.dtype
    shape = make_shape(q, v, u, chunk)
    B, T, H, dk = q.shape
    dv, L = shape.dv, shape.L
    for name, x, dt, shp in (("q", q, io, (B, T, H, dk)), ("k", k, io, (B, T, H, dk)),
                             ("v", v, io, (B, T, H, dv)), ("alpha", alpha, torch.float32, (B, T, H)),
                             ("beta", beta, torch.float32, (B, T, H)),
                             ("u", u, io, (B, T, H, L, dv)), ("w", w, io, (B, T, H, L, dk)),
                             ("S0", S0, torch.float32, (B, H, dv, dk)), ("o", o, io, (B, T, H, dv)),
                             ("S_final", S_final, torch.float32, (B, H, dv, dk))):
        _check_tensor(name, x, dt, shp, dev)
    rc = _call(dev, lib.prism_scan_fwd_noalloc, ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
               _ptr(alpha), _ptr(beta), _ptr(u), _ptr(w), _ptr(S0), _ptr(o), _ptr(S_final),
               _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_fwd_noalloc")
    return o, S_final


def bwd_workspace_for(shape: PrismShape, device) -> torch.Tensor:
    """A cached device workspace of the size prism_scan_bwd needs (one per device/size)."""
    need = ctypes.c_size_t(0)
    rc = load_library().prism_scan_bwd_workspace_size(ctypes.byref(shape), ctypes.byref(need))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_bwd_workspace_size")
    key = ("bwd", str(device), int(need.value))
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(max(256, int(need.value)), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def prism_scan_bwd(q, k, v, alpha, beta, u=None, w=None, S0=None, *, dO, dS_final=None,
                   want_dS0=True, workspace=None, stream=None):
    """Backward of prism_scan_fwd: gradients of every input, fp32.  Inputs as for prism_scan_fwd;
    dO: [B,T,H,dv] (io dtype); dS_final: [B,H,dv,dk] fp32 or None.  Returns a dict with dq, dk
    [B,T,H,dk], dalpha, dbeta [B,T,H], dv [B,T,H,dv] (GDN write) or du [B,T,H,L,dv] and dw
    [B,T,H,L,dk] (rank-L write), and dS0 [B,H,dv,dk] (or None)."""
    lib = load_library()
    if not isinstance(q, torch.Tensor) or not q.is_cuda:
        raise TypeError("q must be a CUDA tensor (libprism has no CPU path)")
    dev, io = q.device, q.dtype
    shape = make_shape(q, v, u)
    B, T, H, dk = q.shape
    dv, L = shape.dv, shape.L
    f32 = torch.float32
    _check_tensor("q", q, io, (B, T, H, dk), dev)
    _check_tensor("k", k, io, (B, T, H, dk), dev)
    _check_tensor("v", v, io, (B, T, H, dv), dev)
    _check_tensor("alpha", alpha, f32, (B, T, H), dev)
    _check_tensor("beta", beta, f32, (B, T, H), dev)
    _check_tensor("u", u, io, (B, T, H, L, dv), dev)
    _check_tensor("w", w, io, (B, T, H, L, dk), dev)
    _check_tensor("S0", S0, f32, (B, H, dv, dk), dev)
    _check_tensor("dO", dO, io, (B, T, H, dv), dev)
    _check_tensor("dS_final", dS_final, f32, (B, H, dv, dk), dev)
    gdn = u is None
    out = {"dq": torch.empty((B, T, H, dk), dtype=f32, device=dev),
           "dk": torch.empty((B, T, H, dk), dtype=f32, device=dev),
           "dv": torch.empty((B, T, H, dv), dtype=f32, device=dev) if gdn else None,
           "dalpha": torch.empty((B, T, H), dtype=f32, device=dev),
           "dbeta": torch.empty((B, T, H), dtype=f32, device=dev),
           "du": None if gdn else torch.empty((B, T, H, L, dv), dtype=f32, device=dev),
           "dw": None if gdn else torch.empty((B, T, H, L, dk), dtype=f32, device=dev),
           "dS0": torch.empty((B, H, dv, dk), dtype=f32, device=dev) if want_dS0 else None}
    if workspace is None:
        workspace = bwd_workspace_for(shape, dev)
    _check_tensor("workspace", workspace, torch.uint8, (workspace.numel(),), dev)
    rc = _call(dev, lib.prism_scan_bwd, ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
               _ptr(beta), _ptr(u), _ptr(w), _ptr(S0), _ptr(dO), _ptr(dS_final), _ptr(out["dq"]),
               _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dalpha"]), _ptr(out["dbeta"]),
               _ptr(out["du"]), _ptr(out["dw"]), _ptr(out["dS0"]), _ptr(workspace),
               ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_bwd")
    return out


def prism_step_decode(q, k, v, alpha, beta, u, w, S, *, o=None, stream=None):
    """One decode step, S updated in place.  q, k: [B,1,H,dk]; v: [B,1,H,dv] or None;
    alpha, beta: [B,1,H]; u: [B,1,H,L,dv] / w: [B,1,H,L,dk] or None; S: [B,H,dv,dk] fp32.
    Returns o [B,1,H,dv]."""
    lib = load_library()
    if not isinstance(q, torch.Tensor) or not q.is_cuda:
        raise TypeError("q must be a CUDA tensor (libprism has no CPU path)")
    dev, io = q.device, q.dtype
    shape = make_shape(q, v, u, 64)
    B, T, H, dk = q.shape
    dv, L = shape.dv, shape.L
    _check_tensor("q", q, io, (B, T, H, dk), dev)
    _check_tensor("k", k, io, (B, T, H, dk), dev)
    _check_tensor("v", v, io, (B, T, H, dv), dev)
    _check_tensor("alpha", alpha, torch.float32, (B, T, H), dev)
    _check_tensor("beta", beta, torch.float32, (B, T, H), dev)
    _check_tensor("u", u, io, (B, T, H, L, dv), dev)
    _check_tensor("w", w, io, (B, T, H, L, dk), dev)
    _check_tensor("S", S, torch.float32, (B, H, dv, dk), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=io, device=dev)
    _check_tensor("o", o, io, (B, T, H, dv), dev)
    rc = _call(dev, lib.prism_step_decode, ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
               _ptr(alpha), _ptr(beta), _ptr(u), _ptr(w), _ptr(S), _ptr(o), _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_step_decode")
    return o


def prism_write_producer(x, v, conv, Wk, Wp, beta, *, u=None, w=None, stream=None):
    """The input-anchored write terms (include/prism.h, prism_write_producer).  x, v: [B,T,H,d]
    bf16; conv: [H,4,d] fp32; Wk, Wp: [H,L,d,d] bf16; beta: [B,T,H,L] fp32.  Returns (u, w), each
    [B,T,H,L,d] bf16, ready for prism_scan_fwd."""
    lib = load_library()
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError("x must be a CUDA tensor (libprism has no CPU path)")
    dev = x.device
    B, T, H, d = x.shape
    L = Wk.shape[1]
    bf = torch.bfloat16
    _check_tensor("x", x, bf, (B, T, H, d), dev)
    _check_tensor("v", v, bf, (B, T, H, d), dev)
    _check_tensor("conv", conv, torch.float32, (H, 4, d), dev)
    _check_tensor("Wk", Wk, bf, (H, L, d, d), dev)
    _check_tensor("Wp", Wp, bf, (H, L, d, d), dev)
    _check_tensor("beta", beta, torch.float32, (B, T, H, L), dev)
    if u is None:
        u = torch.empty((B, T, H, L, d), dtype=bf, device=dev)
    if w is None:
        w = torch.empty((B, T, H, L, d), dtype=bf, device=dev)
    _check_tensor("u", u, bf, (B, T, H, L, d), dev)
    _check_tensor("w", w, bf, (B, T, H, L, d), dev)
    shape = PrismShape(B, H, T, d, d, L, 64, PRISM_BF16)
    rc = _call(dev, lib.prism_write_producer, ctypes.byref(shape), _ptr(x), _ptr(v), _ptr(conv),
               _ptr(Wk), _ptr(Wp), _ptr(beta), _ptr(u), _ptr(w), _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_write_producer")
    return u, w


def prism_scan_fwd_launch_count(shape: PrismShape) -> int:
    """Kernels one prism_scan_fwd call with `shape` enqueues."""
    n = ctypes.c_int(0)
    rc = load_library().prism_scan_fwd_launch_count(ctypes.byref(shape), ctypes.byref(n))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_fwd_launch_count")
    return n.value


def prism_query_device_status(workspace, stream=None, device=None) -> int:
    """Synchronise and return (and clear) the status words: the one kernels wrote into
    `workspace` (or None), and the library's own (decode, producer, no-alloc scratch) on the
    workspace's device (else `device`, else the current device)."""
    if workspace is not None:
        device = workspace.device
    elif device is None:
        device = stream.device if stream is not None else torch.device("cuda", torch.cuda.current_device())
    device = torch.device(device)
    return _call(device, load_library().prism_query_device_status, _ptr(workspace),
                 _stream(stream, device))


def record_launch_events(events) -> None:
    """Arm this thread's next prism_scan_fwd / prism_step_decode call to record events[j] (torch
    CUDA events, already recorded once so that their handles exist) before its launch j and the
    last one after its final launch."""
    handles = (ctypes.c_void_p * max(1, len(events)))(*[e.cuda_event for e in events])
    rc = load_library().prism_debug_record_launch_events(handles, len(events))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_debug_record_launch_events")


def prism_scan_segment_element(q, k, v, alpha, beta, u=None, w=None, *, chunk=64, E=None, f=None,
                               workspace=None, stream=None):
    """Affine map (E, f) of each (b, h) sequence over these T tokens: S -> S E + f.
    E: [B,H,dk,dk] fp32, f: [B,H,dv,dk] fp32 (allocated when not given).  Requires dk == dv."""
    lib = load_library()
    dev = q.device
    io = q.dtype
    B, T, H, dk = q.shape
    shape = make_shape(q, v, u, chunk)
    dv, L = shape.dv, shape.L
    _check_tensor("q", q, io, (B, T, H, dk), dev)
    _check_tensor("k", k, io, (B, T, H, dk), dev)
    _check_tensor("v", v, io, (B, T, H, dv), dev)
    _check_tensor("alpha", alpha, torch.float32, (B, T, H), dev)
    _check_tensor("beta", beta, torch.float32, (B, T, H), dev)
    _check_tensor("u", u, io, (B, T, H, L, dv), dev)
    _check_tensor("w", w, io, (B, T, H, L, dk), dev)
    if E is None:
        E = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    if f is None:
        f = torch.empty((B, H, dv, dk), dtype=torch.float32, device=dev)
    _check_tensor("E", E, torch.float32, (B, H, dk, dk), dev)
    _check_tensor("f", f, torch.float32, (B, H, dv, dk), dev)
    if workspace is None:
        workspace = workspace_for(shape, dev)
    _check_tensor("workspace", workspace, torch.uint8, (workspace.numel(),), dev)
    rc = _call(dev, lib.prism_scan_segment_element, ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
               _ptr(alpha), _ptr(beta), _ptr(u), _ptr(w), _ptr(E), _ptr(f), _ptr(workspace),
               ctypes.c_size_t(workspace.numel()), _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_scan_segment_element")
    return E, f


def prism_state_fold(S_in, E, f, S_out=None, stream=None):
    """S_out = S_in E + f per state; S_in None means zero.  S_in, f, S_out: [..., dv, dk] fp32,
    E: [..., dk, dk] fp32 with the same leading dims."""
    lib = load_library()
    dv, dk = f.shape[-2], f.shape[-1]
    lead = tuple(f.shape[:-2])
    BH = 1
    for n in lead:
        BH *= n
    dev = f.device
    _check_tensor("E", E, torch.float32, lead + (dk, dk), dev)
    _check_tensor("f", f, torch.float32, lead + (dv, dk), dev)
    _check_tensor("S_in", S_in, torch.float32, lead + (dv, dk), dev)
    if S_out is None:
        S_out = torch.empty_like(f)
    _check_tensor("S_out", S_out, torch.float32, lead + (dv, dk), dev)
    rc = _call(dev, lib.prism_state_fold, BH, dk, dv, _ptr(S_in), _ptr(E), _ptr(f), _ptr(S_out),
               _stream(stream, dev))
    if rc != PRISM_OK:
        raise PrismError(rc, "prism_state_fold")
    return S_out
