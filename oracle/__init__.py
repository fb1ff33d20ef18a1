"""CPU oracle for the SSD forward and backward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline and
reference legs of ``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it, and this package never
imports the product path.  The only module both sides use is ``ssd_inputs``,
which draws random tensors and holds none of the method's arithmetic.

Contents:
  * ``ssd_fwd``            -- the plain fp64 sequential recurrence (C + OpenMP,
                              ``ssd_oracle.c``); this is the oracle proper.
  * ``matrix_form.ssd_matrix_form`` -- y = M x with the semiseparable matrix M
                              written out (tiny inputs; a pin for the oracle).
  * ``block.conv1d_silu``, ``block.gate`` -- the Mamba-2 block pieces around the SSD
                              (causal depthwise conv1d + SiLU; the SiLU gate).
  * ``block.conv1d_silu_bwd`` -- their backward (du, dweight, dbias).
  * ``backward.ssd_bwd``     -- the backward pass: the adjoint of the recurrence
                              (derived; the pages give no formulas), fp64 numpy.
  * ``backward.ssd_bwd_gated`` -- the backward through the gate y * SiLU(z).
  * ``ssd_bwd``              -- the same adjoint in C + OpenMP (``ssd_oracle.c``),
                              states recomputed from 64-token checkpoints, for
                              larger inputs; also the magnitude sums of the terms
                              of dA and dD (the scale of their rounding).
  * ``chunked.ssd_chunked``  -- the four chunked steps written out literally in
                              fp64 numpy (a pin for the decomposition the CUDA
                              kernels use).

Every function upcasts its inputs to fp64 after widening bf16 values to fp32
(exact), so both sides see identical numbers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_ssd.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the C oracle with gcc (fp64, OpenMP).  Returns the .so path."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-o", tmp, src, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def load_library(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    f = lib.oracle_ssd_fwd
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    f.argtypes = [i64] * 6 + [vp] * 8 + [i64, vp, vp, vp, i64, ctypes.c_int]
    f.restype = ctypes.c_int
    g = lib.oracle_ssd_bwd
    g.argtypes = [i64] * 6 + [vp] * 17 + [ctypes.c_int, vp, vp]
    g.restype = ctypes.c_int
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _get_lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(build())
        return _lib


def as_f32(a) -> Optional[np.ndarray]:
    """Widen a torch tensor / array to a contiguous fp32 numpy array (exact for
    bf16 and fp32 values)."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch
        if a.dtype != torch.float32:
            a = a.float()
        a = a.numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def as_f64(a) -> Optional[np.ndarray]:
    f = as_f32(a)
    return None if f is None else f.astype(np.float64)


def as_i32(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def max_threads() -> int:
    return int(_get_lib().oracle_max_threads())


def ssd_fwd(x, dt, A, B, C, D=None, initial_states=None, seq_idx=None, num_seqs=None,
            units: Optional[Sequence[int]] = None, nthreads: int = 0, lib: Optional[ctypes.CDLL] = None):
    """fp64 sequential SSD recurrence.

    x (b,L,H,P), dt (b,L,H), A (H), B/C (b,L,G,N), D (H) or None,
    initial_states (b,H,P,N) or None, seq_idx (b,L) int32 or None.
    Returns (y (b,L,H,P) float64, final_states float64): final_states is
    (b,H,P,N), or (num_seqs,H,P,N) when seq_idx is given (rows of ids that do
    not occur stay zero).  ``units`` restricts the work to the listed
    flattened (b*H + h) units; other outputs stay zero.
    """
    x32, dt32, A32, B32, C32 = (as_f32(v) for v in (x, dt, A, B, C))
    D32, h032, si = as_f32(D), as_f32(initial_states), as_i32(seq_idx)
    b, L, H, P = x32.shape
    G, N = B32.shape[2], B32.shape[3]
    assert dt32.shape == (b, L, H) and A32.shape == (H,)
    assert B32.shape == (b, L, G, N) and C32.shape == (b, L, G, N)
    if D32 is not None:
        assert D32.shape == (H,)
    if h032 is not None:
        assert h032.shape == (b, H, P, N)
    y = np.zeros((b, L, H, P), dtype=np.float64)
    if si is not None:
        assert si.shape == (b, L)
        if num_seqs is None:
            num_seqs = int(si.max()) + 1
        final = np.zeros((num_seqs, H, P, N), dtype=np.float64)
    else:
        num_seqs = 0
        final = np.zeros((b, H, P, N), dtype=np.float64)
    u = None if units is None else np.ascontiguousarray(np.asarray(units, dtype=np.int64))

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    lib = lib or _get_lib()
    rc = lib.oracle_ssd_fwd(b, L, H, P, N, G, ptr(x32), ptr(dt32), ptr(A32), ptr(B32), ptr(C32),
                            ptr(D32), ptr(h032), ptr(si), int(num_seqs), ptr(y), ptr(final),
                            ptr(u), 0 if u is None else len(u), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_ssd_fwd failed with code {rc}")
    return y, final


def ssd_bwd(x, dt, A, B, C, D=None, initial_states=None, dy=None, dfinal=None, seq_idx=None,
            nthreads: int = 0) -> dict:
    """The backward pass in C (fp64, OpenMP over (b, h)): gradients of
    sum(dy * y) + sum(dfinal * final) as a dict like ``backward.ssd_bwd``,
    plus dA_abs and dD_abs (H): the sums of the magnitudes of the terms
    that dA and dD add up."""
    x32, dt32, A32, B32, C32 = (as_f32(v) for v in (x, dt, A, B, C))
    D32, h032, si = as_f32(D), as_f32(initial_states), as_i32(seq_idx)
    dy32, df32 = as_f32(dy), as_f32(dfinal)
    b, L, H, P = x32.shape
    G, N = B32.shape[2], B32.shape[3]
    assert dy32.shape == (b, L, H, P)
    dx = np.zeros((b, L, H, P))
    ddt = np.zeros((b, L, H))
    dBh = np.zeros((b, L, H, N))
    dCh = np.zeros((b, L, H, N))
    dA_u = np.zeros(b * H)
    dD_u = np.zeros(b * H)
    dA_abs = np.zeros(b * H)
    dD_abs = np.zeros(b * H)
    dh0 = np.zeros((b, H, P, N)) if h032 is not None else None

    def ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    rc = _get_lib().oracle_ssd_bwd(b, L, H, P, N, G, ptr(x32), ptr(dt32), ptr(A32), ptr(B32), ptr(C32),
                                   ptr(D32), ptr(h032), ptr(si), ptr(dy32), ptr(df32), ptr(dx), ptr(ddt),
                                   ptr(dBh), ptr(dCh), ptr(dA_u), ptr(dD_u), ptr(dh0), int(nthreads), ptr(dA_abs),
                                   ptr(dD_abs))
    if rc != 0:
        raise RuntimeError(f"oracle_ssd_bwd failed with code {rc}")
    grp = np.arange(H) // (H // G)
    dB = np.zeros((b, L, G, N))
    dC = np.zeros((b, L, G, N))
    for h in range(H):
        dB[:, :, grp[h]] += dBh[:, :, h]
        dC[:, :, grp[h]] += dCh[:, :, h]
    return {"dx": dx, "ddt": ddt, "dA": dA_u.reshape(b, H).sum(axis=0), "dB": dB, "dC": dC,
            "dD": None if D32 is None else dD_u.reshape(b, H).sum(axis=0), "dh0": dh0,
            "dA_abs": dA_abs.reshape(b, H).sum(axis=0), "dD_abs": dD_abs.reshape(b, H).sum(axis=0)}
