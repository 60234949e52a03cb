"""fp64 CPU oracle for the gated delta-rule scan with a rank-L write.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import this package.  It shares no code with the CUDA library
(``delta_rule_sequence_b200``) and imports nothing from it.

The oracle is the plain token-by-token definition (``oracle/prism_ref.c``), in double precision:

    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + sum_l u_{t,l} w_{t,l}^T,    o_t = S_t q_t

after "PRISM: Parallel Residual Iterative Sequence Model" (gist.science explainer), technical
summary sections 2.1 and 2.2, and the banbantang.com PRISM article, section 1(4).

Pins (all in ``tests/test_oracle_pins.py``): brute-force Blelloch scan over explicit affine
elements, causal linear attention and gated linear attention closed forms, the delta-rule
overwrite identity, superposition, row independence, resumability, and the GDN route equal to
the general route with u = beta v, w = k.  Planted mistakes (``scan_ref_mutant``) are each caught
by at least one pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "prism_ref.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_prism.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``prism_ref.c`` into ``liboracle_prism.so`` next to it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        cmd = [
            "gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared", "-pthread",
            _SRC, "-o", _LIB_PATH,
        ]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        vp, fp, dp, ci = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int
        common = [ci] * 7 + [vp, vp, vp, fp, fp, vp, vp, dp, dp, dp, ci]
        lib.prism_scan_ref.argtypes = common
        lib.prism_scan_ref.restype = ci
        lib.prism_scan_ref_mutant.argtypes = common + [ci]
        lib.prism_scan_ref_mutant.restype = ci
        _lib = lib
    return _lib


def _host_array(x, want_dtype=None):
    """Return a C-contiguous numpy array sharing the bytes the GPU gets (bf16 kept as uint16)."""
    if x is None:
        return None
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16)
            return x.numpy()
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    x = np.ascontiguousarray(x)
    if want_dtype is not None:
        x = np.ascontiguousarray(x, dtype=want_dtype)
    return x


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def scan_ref(q, k, v, alpha, beta, u=None, w=None, S0=None, *, L=None, n_threads=None,
             mutation=0):
    """Run the oracle.

    q, k: [B,T,H,dk]; v: [B,T,H,dv] (read only when u is None); alpha, beta: [B,T,H] fp32;
    u: [B,T,H,L,dv]; w: [B,T,H,L,dk]; S0: [B,H,dv,dk] (any float type, widened to double) or
    None.  q/k/v/u/w may be torch bf16/fp32 tensors or numpy float32/uint16(bf16 bits) arrays;
    all must share one I/O type.  Returns (o [B,T,H,dv] float64, S_final [B,H,dv,dk] float64).
    """
    qa, ka = _host_array(q), _host_array(k)
    io_f32 = 1 if qa.dtype == np.float32 else 0
    if qa.dtype not in (np.float32, np.uint16):
        raise TypeError(f"oracle: q must be fp32 or bf16, got {qa.dtype}")
    B, T, H, dk = qa.shape
    va = _host_array(v)
    ua, wa = _host_array(u), _host_array(w)
    if ua is not None:
        Lr = ua.shape[3]
        dv = ua.shape[4]
    else:
        Lr = 1
        dv = va.shape[3]
    if L is not None and L != Lr:
        raise ValueError("oracle: L disagrees with u's shape")
    for name, arr in (("k", ka), ("v", va), ("u", ua), ("w", wa)):
        if arr is not None and arr.dtype != qa.dtype:
            raise TypeError(f"oracle: {name} has dtype {arr.dtype}, q has {qa.dtype}")
    al = _host_array(alpha, np.float32).astype(np.float32, copy=False)
    be = _host_array(beta, np.float32).astype(np.float32, copy=False)
    S0a = None
    if S0 is not None:
        S0a = np.ascontiguousarray(_host_array(S0), dtype=np.float64)
    o = np.zeros((B, T, H, dv), dtype=np.float64)
    Sf = np.zeros((B, H, dv, dk), dtype=np.float64)
    nt = n_threads or default_threads()
    lib = _load()
    args = [B, H, T, dk, dv, Lr, io_f32, _ptr(qa), _ptr(ka), _ptr(va), _ptr(al), _ptr(be),
            _ptr(ua), _ptr(wa), _ptr(S0a), _ptr(o), _ptr(Sf), nt]
    if mutation:
        rc = lib.prism_scan_ref_mutant(*args, mutation)
    else:
        rc = lib.prism_scan_ref(*args)
    if rc != 0:
        raise ValueError(f"oracle: prism_scan_ref rejected the arguments (status {rc})")
    return o, Sf
