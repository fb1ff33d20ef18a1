"""Chunked SSD (Mamba-2 structured state space duality) forward and backward on B200.

Thin Python binding over the C ABI in ``include/ssd.h`` (``libssd.so``, built
in-tree by ``mamba_ssd_chunked_03_b200/build.py``).  This module only marshals
arguments: it checks tensor placement, dtypes and shapes, allocates outputs
and the workspace with PyTorch on the current stream, and calls the library
(``ssd_fwd``, ``ssd_bwd``, ``ssd_step``, ``ssd_conv1d_silu`` and the rest).
Every step runs in the library's CUDA kernels; there is no Python or CPU
fallback, and importing fails loudly if the library is missing.

    y, final_states = fwd(x, dt, A, B, C, D, chunk_size=64,
                          initial_states=None, seq_idx=None, num_seqs=None)
    y_t = step(x_t, dt_t, A, B_t, C_t, D, state)   # one decode step, state in place
    grads = bwd(x, dt, A, B, C, D, dy)              # the backward (fp32 gradients)
    y, final_states = ssd_chunked(x, dt, A, B, C, D)  # differentiable: fwd, then bwd
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = ["fwd", "fwd_host", "bwd", "BwdArgs", "bwd_workspace_size", "bwd_chunk_size", "bwd_path", "ssd_chunked", "make_args",
           "make_bwd_args", "main_kernel", "device_status",
           "conv1d_silu_bwd", "ConvBwdArgs", "causal_conv1d_silu", "step", "StepArgs", "total_decay", "state_fold", "conv1d_silu", "ConvArgs", "workspace_size", "launch_count", "kernel_path", "SSDError", "lib", "LIB_PATH", "Args",
           "SSD_OK", "SSD_ERR_INVALID_ARG", "SSD_ERR_UNSUPPORTED", "SSD_ERR_WORKSPACE", "SSD_ERR_CUDA",
           "SSD_ERR_TIMEOUT", "SSD_F32", "SSD_BF16", "SSD_FLAG_GENERIC", "SSD_FLAG_CHECK_SEQ", "SSD_FLAG_TEST_STALL"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssd.so")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_WORKSPACE, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = range(6)
SSD_F32, SSD_BF16 = 0, 1
SSD_FLAG_GENERIC = 1
SSD_FLAG_CHECK_SEQ = 2
SSD_FLAG_TEST_STALL = 4  # failure-path tests only: the two-head kernel's hand-over wait runs out
SSD_BWD_DINITIAL_ONLY = 1


class Args(ctypes.Structure):
    """Mirror of ``ssd_fwd_args``."""
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "chunk_size")] + [
        ("dtype", ctypes.c_int),
        ("flags", ctypes.c_uint32),
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p), ("C", ctypes.c_void_p), ("D", ctypes.c_void_p),
        ("initial_states", ctypes.c_void_p), ("seq_idx", ctypes.c_void_p),
        ("num_seqs", ctypes.c_int64),
        ("y", ctypes.c_void_p), ("final_states", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("timing_events", ctypes.c_void_p * 2),
        ("z", ctypes.c_void_p),
    ]


class StepArgs(ctypes.Structure):
    """Mirror of ``ssd_step_args``."""
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "nheads", "headdim", "dstate", "ngroups")] + [
        ("dtype", ctypes.c_int),
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p), ("C", ctypes.c_void_p), ("D", ctypes.c_void_p),
        ("state", ctypes.c_void_p), ("y", ctypes.c_void_p),
    ]


class ConvArgs(ctypes.Structure):
    """Mirror of ``ssd_conv_args``."""
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seqlen", "channels", "width")] + [
        ("dtype", ctypes.c_int),
        ("u", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("seq_idx", ctypes.c_void_p), ("out", ctypes.c_void_p),
    ]


class BwdArgs(ctypes.Structure):
    """Mirror of ``ssd_bwd_args``."""
    _fields_ = [(n, ctypes.c_int64) for n in
                ("batch", "seqlen", "nheads", "headdim", "dstate", "ngroups", "chunk_size")] + [
        ("dtype", ctypes.c_int),
        ("x", ctypes.c_void_p), ("dt", ctypes.c_void_p), ("A", ctypes.c_void_p),
        ("B", ctypes.c_void_p), ("C", ctypes.c_void_p), ("D", ctypes.c_void_p),
        ("initial_states", ctypes.c_void_p), ("seq_idx", ctypes.c_void_p),
        ("dy", ctypes.c_void_p), ("dfinal_states", ctypes.c_void_p),
        ("dx", ctypes.c_void_p), ("ddt", ctypes.c_void_p), ("dA", ctypes.c_void_p),
        ("dB", ctypes.c_void_p), ("dC", ctypes.c_void_p), ("dD", ctypes.c_void_p),
        ("dinitial_states", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("timing_events", ctypes.c_void_p * 2),
        ("z", ctypes.c_void_p), ("dz", ctypes.c_void_p),
        ("flags", ctypes.c_uint32),
    ]


class ConvBwdArgs(ctypes.Structure):
    """Mirror of ``ssd_conv_bwd_args``."""
    _fields_ = [(n, ctypes.c_int64) for n in ("batch", "seqlen", "channels", "width")] + [
        ("dtype", ctypes.c_int),
        ("u", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p),
        ("seq_idx", ctypes.c_void_p), ("dout", ctypes.c_void_p),
        ("du", ctypes.c_void_p), ("dweight", ctypes.c_void_p), ("dbias", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python mamba_ssd_chunked_03_b200/build.py` "
            "(there is no fallback implementation)")
    L = ctypes.CDLL(LIB_PATH)
    L.ssd_fwd.argtypes = [ctypes.POINTER(Args), ctypes.c_void_p]
    L.ssd_fwd.restype = ctypes.c_int
    L.ssd_fwd_workspace_size.argtypes = [ctypes.POINTER(Args)]
    L.ssd_fwd_workspace_size.restype = ctypes.c_size_t
    L.ssd_fwd_host_workspace_size.argtypes = [ctypes.POINTER(Args), ctypes.c_int64]
    L.ssd_fwd_host_workspace_size.restype = ctypes.c_size_t
    L.ssd_fwd_host.argtypes = [ctypes.POINTER(Args), ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                               ctypes.c_void_p, ctypes.c_void_p]
    L.ssd_fwd_host.restype = ctypes.c_int
    L.ssd_fwd_launch_count.argtypes = [ctypes.POINTER(Args)]
    L.ssd_fwd_launch_count.restype = ctypes.c_int
    L.ssd_fwd_device_status.argtypes = [ctypes.POINTER(Args), ctypes.c_void_p]
    L.ssd_fwd_device_status.restype = ctypes.c_int
    L.ssd_fwd_path.argtypes = [ctypes.POINTER(Args)]
    L.ssd_fwd_path.restype = ctypes.c_char_p
    L.ssd_fwd_main_kernel.argtypes = [ctypes.POINTER(Args)]
    L.ssd_fwd_main_kernel.restype = ctypes.c_char_p
    L.ssd_step.argtypes = [ctypes.POINTER(StepArgs), ctypes.c_void_p]
    L.ssd_step.restype = ctypes.c_int
    L.ssd_bwd.argtypes = [ctypes.POINTER(BwdArgs), ctypes.c_void_p]
    L.ssd_bwd.restype = ctypes.c_int
    L.ssd_bwd_workspace_size.argtypes = [ctypes.POINTER(BwdArgs)]
    L.ssd_bwd_workspace_size.restype = ctypes.c_size_t
    L.ssd_bwd_chunk_size.argtypes = [ctypes.POINTER(BwdArgs)]
    L.ssd_bwd_chunk_size.restype = ctypes.c_int64
    L.ssd_bwd_path.argtypes = [ctypes.POINTER(BwdArgs)]
    L.ssd_bwd_path.restype = ctypes.c_char_p
    L.ssd_conv1d_silu_bwd.argtypes = [ctypes.POINTER(ConvBwdArgs), ctypes.c_void_p]
    L.ssd_conv1d_silu_bwd.restype = ctypes.c_int
    L.ssd_conv1d_silu_bwd_workspace_size.argtypes = [ctypes.POINTER(ConvBwdArgs)]
    L.ssd_conv1d_silu_bwd_workspace_size.restype = ctypes.c_size_t
    L.ssd_conv1d_silu.argtypes = [ctypes.POINTER(ConvArgs), ctypes.c_void_p]
    L.ssd_conv1d_silu.restype = ctypes.c_int
    L.ssd_total_decay.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p] + [ctypes.c_int64] * 3 + [
        ctypes.c_void_p]
    L.ssd_total_decay.restype = ctypes.c_int
    L.ssd_state_fold.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 5 + [ctypes.c_void_p]
    L.ssd_state_fold.restype = ctypes.c_int
    L.ssd_check_seq_idx.argtypes = [ctypes.c_void_p] + [ctypes.c_int64] * 3
    L.ssd_check_seq_idx.restype = ctypes.c_int
    L.ssd_status_string.argtypes = [ctypes.c_int]
    L.ssd_status_string.restype = ctypes.c_char_p
    L.ssd_version.restype = ctypes.c_int
    return L


lib = _load()


class SSDError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(f"ssd_fwd failed: {lib.ssd_status_string(status).decode()} (status {status})")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def make_args(x, dt, A, B, C, D=None, chunk_size: int = 64, initial_states=None, seq_idx=None,
              num_seqs: Optional[int] = None, y=None, final_states=None, workspace=None,
              workspace_bytes: int = 0, generic: bool = False, z=None) -> Args:
    """Fill an ``ssd_fwd_args`` from tensors (shapes read from x and B)."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    a = Args()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk_size = b, L, H, P, N, G, int(chunk_size)
    a.dtype = SSD_BF16 if x.dtype == torch.bfloat16 else SSD_F32
    a.flags = SSD_FLAG_GENERIC if generic else 0
    a.x, a.dt, a.A, a.B, a.C, a.D = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D)
    a.initial_states, a.seq_idx = _ptr(initial_states), _ptr(seq_idx)
    a.num_seqs = int(num_seqs) if seq_idx is not None else 0
    a.y, a.final_states = _ptr(y), _ptr(final_states)
    a.workspace, a.workspace_bytes = _ptr(workspace), int(workspace_bytes)
    a.z = _ptr(z)
    return a


def _check(x, dt, A, B, C, D, initial_states, seq_idx):
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    if x.dim() != 4 or B.dim() != 4 or C.dim() != 4 or dt.dim() != 3 or A.dim() != 1:
        raise ValueError("expected x (b,L,H,P), dt (b,L,H), A (H), B and C (b,L,G,N)")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if tuple(B.shape) != (b, L, G, N) or tuple(C.shape) != (b, L, G, N):
        raise ValueError("B and C must be (b, L, G, N)")
    if tuple(dt.shape) != (b, L, H) or tuple(A.shape) != (H,):
        raise ValueError("dt must be (b, L, H) and A (H,)")
    if B.dtype != x.dtype or C.dtype != x.dtype:
        raise TypeError("B and C must have x's dtype")
    if dt.dtype != torch.float32 or A.dtype != torch.float32:
        raise TypeError("dt and A must be float32")
    if D is not None and (D.dtype != torch.float32 or tuple(D.shape) != (H,)):
        raise ValueError("D must be float32 (H,)")
    if initial_states is not None and (initial_states.dtype != torch.float32
                                       or tuple(initial_states.shape) != (b, H, P, N)):
        raise ValueError("initial_states must be float32 (b, H, P, N)")
    if seq_idx is not None and (seq_idx.dtype != torch.int32 or tuple(seq_idx.shape) != (b, L)):
        raise ValueError("seq_idx must be int32 (b, L)")
    dev = x.device
    for name, t in (("x", x), ("dt", dt), ("A", A), ("B", B), ("C", C), ("D", D),
                    ("initial_states", initial_states), ("seq_idx", seq_idx)):
        if t is None:
            continue
        if t.device != dev or dev.type != "cuda":
            raise ValueError(f"{name} must be a CUDA tensor on {dev}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def workspace_size(x, B, chunk_size: int, seq_idx=None, num_seqs=None, final_states: bool = True,
                   generic: bool = False) -> int:
    """Workspace bytes for these shapes (tensors only supply shapes/dtype)."""
    a = make_args(x, None, None, B, None, chunk_size=chunk_size, seq_idx=seq_idx, num_seqs=num_seqs,
                  generic=generic)
    if final_states:
        a.final_states = 1 << 8  # presence only; the size query does not dereference
    return int(lib.ssd_fwd_workspace_size(ctypes.byref(a)))


def device_status(x, B, chunk_size: int, workspace: torch.Tensor, generic: bool = False) -> int:
    """Synchronise the current stream and report whether the last call that
    used ``workspace`` had a device-side wait give up (``SSD_ERR_TIMEOUT``)
    or not (``SSD_OK``)."""
    a = make_args(x, None, None, B, None, chunk_size=chunk_size, generic=generic)
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    return int(lib.ssd_fwd_device_status(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)))


def launch_count(x, B, chunk_size: int, seq_idx=None, num_seqs=None, final_states: bool = True,
                 generic: bool = False, z=None) -> int:
    """Kernels one ``fwd`` call enqueues for these shapes (``z``: the gate, if any)."""
    a = make_args(x, None, None, B, None, chunk_size=chunk_size, seq_idx=seq_idx, num_seqs=num_seqs,
                  generic=generic, z=z)
    if final_states:
        a.final_states = 1 << 8  # presence only; the query does not dereference
    return int(lib.ssd_fwd_launch_count(ctypes.byref(a)))


def kernel_path(x, B, chunk_size: int, generic: bool = False, seq_idx=None, num_seqs=None) -> str:
    a = make_args(x, None, None, B, None, chunk_size=chunk_size, seq_idx=seq_idx, num_seqs=num_seqs,
                  generic=generic)
    return lib.ssd_fwd_path(ctypes.byref(a)).decode()


def main_kernel(x, dt, B, chunk_size: int, generic: bool = False, seq_idx=None, num_seqs=None, z=None) -> str:
    """Name of the fused kernel a call with these tensors is dominated by
    (the one ``timing_events`` bracket; ``z``: the gate, if any)."""
    a = make_args(x, dt, None, B, None, chunk_size=chunk_size, seq_idx=seq_idx, num_seqs=num_seqs,
                  generic=generic, z=z)
    return lib.ssd_fwd_main_kernel(ctypes.byref(a)).decode()


def fwd(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
        D: Optional[torch.Tensor] = None, chunk_size: int = 64,
        initial_states: Optional[torch.Tensor] = None, seq_idx: Optional[torch.Tensor] = None,
        num_seqs: Optional[int] = None, return_final_states: bool = True,
        y: Optional[torch.Tensor] = None, final_states: Optional[torch.Tensor] = None,
        workspace: Optional[torch.Tensor] = None, generic: bool = False,
        timing_events: Optional[tuple] = None, z: Optional[torch.Tensor] = None, check_seq: bool = False,
        check_status: bool = False, flags: int = 0):
    """SSD forward.  Returns (y, final_states or None).

    x (b,L,H,P) fp32|bf16, dt (b,L,H) fp32, A (H) fp32, B/C (b,L,G,N) x.dtype,
    D (H) fp32 or None, initial_states (b,H,P,N) fp32 or None,
    seq_idx (b,L) int32 (non-decreasing per row) or None; with seq_idx,
    final_states is (num_seqs,H,P,N), else (b,H,P,N).
    ``y``, ``final_states`` and ``workspace`` may be passed preallocated.
    ``timing_events``: optional (start, end) torch.cuda.Event pair recorded on
    the current stream around the call's main kernel.
    ``z`` (b,L,H,P) x.dtype or None: the block's gate, y is returned as
    y * SiLU(z).
    ``check_seq``: check the seq_idx precondition on a host copy first
    (synchronous; raises SSDError on a violation).
    ``check_status``: wait for the call and raise SSDError(SSD_ERR_TIMEOUT)
    if a bounded device-side wait gave up (y is then incomplete); without it
    the call is asynchronous and such a failure is seen only through
    ``device_status``.
    ``flags``: further SSD_FLAG_* bits passed through to ssd_fwd.
    """
    _check(x, dt, A, B, C, D, initial_states, seq_idx)
    if z is not None and (z.dtype != x.dtype or tuple(z.shape) != tuple(x.shape) or z.device != x.device
                          or not z.is_contiguous()):
        raise ValueError("z must be a contiguous tensor like x")
    b, L, H, P = x.shape
    N = B.shape[3]
    if seq_idx is not None and num_seqs is None:
        num_seqs = int(seq_idx.max().item()) + 1
    if y is None:
        y = torch.empty_like(x)
    if return_final_states and final_states is None:
        rows = num_seqs if seq_idx is not None else b
        final_states = torch.empty(rows, H, P, N, device=x.device, dtype=torch.float32)
    if not return_final_states:
        final_states = None
    a = make_args(x, dt, A, B, C, D, chunk_size, initial_states, seq_idx, num_seqs, y, final_states,
                  generic=generic, z=z)
    if check_seq:
        a.flags |= SSD_FLAG_CHECK_SEQ
    a.flags |= int(flags)
    need = int(lib.ssd_fwd_workspace_size(ctypes.byref(a)))
    if need > 0:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    if timing_events is not None:
        h0_, h1_ = timing_events[0].cuda_event, timing_events[1].cuda_event
        if not h0_ or not h1_:
            raise ValueError("timing events must have been recorded once (torch creates them lazily)")
        a.timing_events[0], a.timing_events[1] = h0_, h1_
    stream = torch.cuda.current_stream(x.device).cuda_stream
    st = lib.ssd_fwd(ctypes.byref(a), ctypes.c_void_p(stream))
    if st != SSD_OK:
        raise SSDError(st)
    if check_status:
        st = int(lib.ssd_fwd_device_status(ctypes.byref(a), ctypes.c_void_p(stream)))
        if st != SSD_OK:
            raise SSDError(st)
    return y, final_states


_second_streams = {}


def fwd_host(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
             D: Optional[torch.Tensor] = None, chunk_size: int = 64,
             initial_states: Optional[torch.Tensor] = None, seq_idx: Optional[torch.Tensor] = None,
             num_seqs: Optional[int] = None, return_final_states: bool = True,
             y: Optional[torch.Tensor] = None, final_states: Optional[torch.Tensor] = None,
             z: Optional[torch.Tensor] = None, rows_per_piece: int = 0, workspace: Optional[torch.Tensor] = None,
             device=None, stream2=None, check_seq: bool = False, flags: int = 0):
    """SSD forward from and to HOST tensors via ``ssd_fwd_host``.  Inputs as
    for ``fwd`` but CPU tensors (pinned, for the copies to overlap); y and
    final_states come back as CPU tensors (pinned when allocated here).  The
    work runs in pieces of ``rows_per_piece`` rows, or (negative) of
    ``-rows_per_piece`` tokens of every row, each piece starting from the
    state the previous one ends in (0: the library chooses eight pieces, of
    rows for a batch of 8 or more, else of 64-token chunks), alternating
    between the current stream of ``device`` and ``stream2`` (a
    torch.cuda.Stream; one per device is kept here if None), so that a
    piece's copies in overlap the previous piece's compute and copies out.
    ``workspace``: a uint8 CUDA tensor of at least the size the library asks
    for, or None.  ``flags``: further SSD_FLAG_* bits (SSD_FLAG_GENERIC).
    Asynchronous on the current stream like ``fwd``: synchronize it before
    reading y."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("x must be float32 or bfloat16")
    if x.dim() != 4 or B.dim() != 4 or C.dim() != 4 or dt.dim() != 3 or A.dim() != 1:
        raise ValueError("expected x (b,L,H,P), dt (b,L,H), A (H), B and C (b,L,G,N)")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    for name, t in (("x", x), ("dt", dt), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
                    ("initial_states", initial_states), ("seq_idx", seq_idx)):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CPU tensor")
    if tuple(B.shape) != (b, L, G, N) or tuple(C.shape) != (b, L, G, N) or B.dtype != x.dtype or C.dtype != x.dtype:
        raise ValueError("B and C must be (b, L, G, N) in x's dtype")
    if tuple(dt.shape) != (b, L, H) or tuple(A.shape) != (H,) or dt.dtype != torch.float32 or A.dtype != torch.float32:
        raise ValueError("dt must be float32 (b, L, H) and A float32 (H,)")
    if D is not None and (D.dtype != torch.float32 or tuple(D.shape) != (H,)):
        raise ValueError("D must be float32 (H,)")
    if z is not None and (z.dtype != x.dtype or tuple(z.shape) != tuple(x.shape)):
        raise ValueError("z must be like x")
    if initial_states is not None and (initial_states.dtype != torch.float32
                                       or tuple(initial_states.shape) != (b, H, P, N)):
        raise ValueError("initial_states must be float32 (b, H, P, N)")
    if seq_idx is not None and (seq_idx.dtype != torch.int32 or tuple(seq_idx.shape) != (b, L)):
        raise ValueError("seq_idx must be int32 (b, L)")
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if seq_idx is not None and num_seqs is None:
        num_seqs = int(seq_idx.max().item()) + 1
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    if return_final_states and final_states is None:
        rows = num_seqs if seq_idx is not None else b
        final_states = torch.empty(rows, H, P, N, dtype=torch.float32, pin_memory=True)
    if not return_final_states:
        final_states = None
    a = make_args(x, dt, A, B, C, D, chunk_size, initial_states, seq_idx, num_seqs, y, final_states, z=z)
    if check_seq:
        a.flags |= SSD_FLAG_CHECK_SEQ
    a.flags |= int(flags)
    need = int(lib.ssd_fwd_host_workspace_size(ctypes.byref(a), int(rows_per_piece)))
    if need == 0:
        raise SSDError(SSD_ERR_INVALID_ARG)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if stream2 is None:
        stream2 = _second_streams.get(dev.index)
        if stream2 is None:
            stream2 = _second_streams[dev.index] = torch.cuda.Stream(dev)
    st = lib.ssd_fwd_host(ctypes.byref(a), int(rows_per_piece), ctypes.c_void_p(workspace.data_ptr()),
                          workspace.numel() * workspace.element_size(),
                          ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream),
                          ctypes.c_void_p(stream2.cuda_stream))
    if st != SSD_OK:
        raise SSDError(st)
    return y, final_states


def fwd_host_workspace_size(x, B, chunk_size: int = 64, rows_per_piece: int = 0, seq_idx=None, num_seqs=None,
                            final_states: bool = True, has_D: bool = True, z: bool = False,
                            initial_states: bool = False, flags: int = 0) -> int:
    """Device workspace bytes ``fwd_host`` needs for these shapes (tensors
    only supply shapes and dtype)."""
    a = make_args(x, None, None, B, None, chunk_size=chunk_size, seq_idx=seq_idx, num_seqs=num_seqs)
    a.flags |= int(flags)
    flag_ptr = 1 << 8  # presence only; the size query does not dereference
    a.final_states = flag_ptr if final_states else None
    a.D = flag_ptr if has_D else None
    a.z = flag_ptr if z else None
    a.initial_states = flag_ptr if initial_states else None
    return int(lib.ssd_fwd_host_workspace_size(ctypes.byref(a), int(rows_per_piece)))


def step(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
         D: Optional[torch.Tensor], state: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One recurrent (decode) step via ``ssd_step``: x (b,H,P), dt (b,H), A (H),
    B and C (b,G,N), D (H) or None, state (b,H,P,N) fp32, updated in place.
    Returns y (b,H,P) in x's dtype."""
    if x.dim() != 3 or dt.dim() != 2 or B.dim() != 3 or C.dim() != 3 or state.dim() != 4:
        raise ValueError("expected x (b,H,P), dt (b,H), B and C (b,G,N), state (b,H,P,N)")
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    if tuple(dt.shape) != (b, H) or tuple(A.shape) != (H,) or tuple(C.shape) != (b, G, N) \
            or tuple(B.shape) != (b, G, N) or tuple(state.shape) != (b, H, P, N):
        raise ValueError("shapes do not match x (b,H,P) and B (b,G,N)")
    if x.dtype not in (torch.float32, torch.bfloat16) or B.dtype != x.dtype or C.dtype != x.dtype:
        raise TypeError("x, B and C must all be float32 or all bfloat16")
    if dt.dtype != torch.float32 or A.dtype != torch.float32 or state.dtype != torch.float32 \
            or (D is not None and (D.dtype != torch.float32 or tuple(D.shape) != (H,))):
        raise TypeError("dt, A, D and state must be float32 (D of shape (H,))")
    for name, t in (("x", x), ("dt", dt), ("A", A), ("B", B), ("C", C), ("D", D), ("state", state)):
        if t is not None and (t.device != x.device or x.device.type != "cuda" or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor on {x.device}")
    if y is None:
        y = torch.empty_like(x)
    a = StepArgs()
    a.batch, a.nheads, a.headdim, a.dstate, a.ngroups = b, H, P, N, G
    a.dtype = SSD_BF16 if x.dtype == torch.bfloat16 else SSD_F32
    a.x, a.dt, a.A, a.B, a.C, a.D = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D)
    a.state, a.y = _ptr(state), _ptr(y)
    st = lib.ssd_step(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream(x.device).cuda_stream))
    if st != SSD_OK:
        raise SSDError(st)
    return y


def _stream(t: torch.Tensor) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def total_decay(dt: torch.Tensor, A: torch.Tensor) -> torch.Tensor:
    """``ssd_total_decay``: exp(A_h * sum_t dt[b,t,h]) as a (b,H) fp32 tensor."""
    if dt.dim() != 3 or dt.dtype != torch.float32 or A.dtype != torch.float32 or tuple(A.shape) != (dt.shape[2],):
        raise ValueError("dt must be float32 (b,L,H) and A float32 (H,)")
    if not (dt.is_cuda and A.is_cuda and dt.is_contiguous() and A.is_contiguous()):
        raise ValueError("dt and A must be contiguous CUDA tensors")
    b, L, H = dt.shape
    out = torch.empty(b, H, device=dt.device, dtype=torch.float32)
    st = lib.ssd_total_decay(dt.data_ptr(), A.data_ptr(), out.data_ptr(), b, L, H, _stream(dt))
    if st != SSD_OK:
        raise SSDError(st)
    return out


def state_fold(states: Optional[torch.Tensor], decays: Optional[torch.Tensor],
               initial_states: Optional[torch.Tensor], rank: int, shape) -> torch.Tensor:
    """``ssd_state_fold``: initial_states (or 0) carried through ranks
    0..rank-1 of states (R,b,H,P,N) and decays (R,b,H); shape = (b,H,P,N)."""
    b, H, P, N = shape
    dev = next(t.device for t in (states, initial_states, decays) if t is not None) if (
        states is not None or initial_states is not None) else torch.device("cuda")
    for name, t, want in (("states", states, None), ("decays", decays, None),
                          ("initial_states", initial_states, (b, H, P, N))):
        if t is None:
            continue
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
        if want is not None and tuple(t.shape) != want:
            raise ValueError(f"{name} must be {want}")
    if rank > 0 and (states is None or decays is None or states.shape[0] < rank or decays.shape[0] < rank
                     or tuple(states.shape[1:]) != (b, H, P, N) or tuple(decays.shape[1:]) != (b, H)):
        raise ValueError("states (R,b,H,P,N) and decays (R,b,H) with R >= rank are needed for rank > 0")
    out = torch.empty(b, H, P, N, device=dev, dtype=torch.float32)
    st = lib.ssd_state_fold(_ptr(states), _ptr(decays), _ptr(initial_states), out.data_ptr(), int(rank), b, H, P, N,
                            _stream(out))
    if st != SSD_OK:
        raise SSDError(st)
    return out


def conv1d_silu(u: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
                seq_idx: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``ssd_conv1d_silu``: SiLU of the causal depthwise convolution of u
    (b,L,C) with weight (C,K) fp32 and bias (C) fp32 or None; seq_idx (b,L)
    int32 keeps taps inside each packed sequence.  Returns (b,L,C) in u's dtype."""
    if u.dim() != 3 or weight.dim() != 2 or weight.shape[0] != u.shape[2]:
        raise ValueError("expected u (b,L,C) and weight (C,K)")
    if u.dtype not in (torch.float32, torch.bfloat16) or weight.dtype != torch.float32 \
            or (bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (u.shape[2],))):
        raise TypeError("u float32 or bfloat16; weight and bias float32 (bias of shape (C,))")
    if seq_idx is not None and (seq_idx.dtype != torch.int32 or tuple(seq_idx.shape) != tuple(u.shape[:2])):
        raise ValueError("seq_idx must be int32 (b,L)")
    for name, t in (("u", u), ("weight", weight), ("bias", bias), ("seq_idx", seq_idx)):
        if t is not None and (t.device != u.device or u.device.type != "cuda" or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor on {u.device}")
    if out is None:
        out = torch.empty_like(u)
    a = ConvArgs()
    a.batch, a.seqlen, a.channels = u.shape
    a.width = weight.shape[1]
    a.dtype = SSD_BF16 if u.dtype == torch.bfloat16 else SSD_F32
    a.u, a.weight, a.bias, a.seq_idx, a.out = _ptr(u), _ptr(weight), _ptr(bias), _ptr(seq_idx), _ptr(out)
    st = lib.ssd_conv1d_silu(ctypes.byref(a), _stream(u))
    if st != SSD_OK:
        raise SSDError(st)
    return out


def make_bwd_args(x, dt, A, B, C, D=None, dy=None, initial_states=None, seq_idx=None, dfinal_states=None,
                  chunk_size: int = 0) -> BwdArgs:
    """Fill an ``ssd_bwd_args`` from tensors (shapes read from x and B); the
    gradient and workspace pointers are left NULL."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    a = BwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk_size = b, L, H, P, N, G, int(chunk_size)
    a.dtype = SSD_BF16 if x.dtype == torch.bfloat16 else SSD_F32
    a.x, a.dt, a.A, a.B, a.C, a.D = _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D)
    a.initial_states, a.seq_idx = _ptr(initial_states), _ptr(seq_idx)
    a.dy, a.dfinal_states = _ptr(dy), _ptr(dfinal_states)
    return a


def bwd_workspace_size(x, B, chunk_size: int = 0, z=None) -> int:
    """Workspace bytes ``ssd_bwd`` needs for these shapes (0: not supported);
    ``z``: the gate, if the call has one."""
    a = make_bwd_args(x, None, None, B, None, chunk_size=chunk_size)
    a.z = _ptr(z)
    return int(lib.ssd_bwd_workspace_size(ctypes.byref(a)))


def bwd_chunk_size(x, B, chunk_size: int = 0) -> int:
    """The chunk length ``ssd_bwd`` uses for these shapes (0: not supported)."""
    a = make_bwd_args(x, None, None, B, None, chunk_size=chunk_size)
    return int(lib.ssd_bwd_chunk_size(ctypes.byref(a)))


def bwd_path(x, dy, B, C, z=None, chunk_size: int = 0, dx: Optional[torch.Tensor] = None) -> str:
    """Kernels ``bwd`` runs for these tensors: "tcgen05" (the chunk states and
    per-chunk gradients on the tensor cores) or "generic" (CUDA cores)."""
    a = make_bwd_args(x, None, None, B, C, dy=dy, chunk_size=chunk_size)
    a.z = _ptr(z)
    a.dx = _ptr(dx)
    return lib.ssd_bwd_path(ctypes.byref(a)).decode()


def bwd(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
        D: Optional[torch.Tensor], dy: torch.Tensor, initial_states: Optional[torch.Tensor] = None,
        seq_idx: Optional[torch.Tensor] = None, dfinal_states: Optional[torch.Tensor] = None,
        chunk_size: int = 0, want_dD: bool = True, want_dinitial_states: Optional[bool] = None,
        workspace: Optional[torch.Tensor] = None, timing_events: Optional[tuple] = None,
        z: Optional[torch.Tensor] = None, dinitial_only: bool = False) -> dict:
    """The SSD backward via ``ssd_bwd``: gradients of a loss given
    dy = dLoss/dy (like x) and dfinal_states = dLoss/dfinal_states
    ((b,H,P,N) fp32 or None; not with seq_idx).  Inputs as for ``fwd``.
    Returns a dict of fp32 tensors dx, ddt, dA, dB, dC, dD (None unless
    ``want_dD``) and dinitial_states (by default only when initial_states
    is given).  ``chunk_size`` is the backward's own chunk length (0: the
    library chooses).  ``timing_events``: optional (start, end)
    torch.cuda.Event pair recorded around the dominant kernel.  ``z``: the
    forward's gate (like x); dy is then the gradient of y * SiLU(z), and the
    dict also holds dz (fp32).  ``dinitial_only``: compute dinitial_states
    alone (two of the six kernels); the other entries are None."""
    _check(x, dt, A, B, C, D, initial_states, seq_idx)
    if dy.dtype != x.dtype or tuple(dy.shape) != tuple(x.shape) or dy.device != x.device or not dy.is_contiguous():
        raise ValueError("dy must be a contiguous tensor like x")
    if z is not None and (z.dtype != x.dtype or tuple(z.shape) != tuple(x.shape) or z.device != x.device
                          or not z.is_contiguous()):
        raise ValueError("z must be a contiguous tensor like x")
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if dfinal_states is not None and (dfinal_states.dtype != torch.float32 or tuple(dfinal_states.shape) != (b, H, P, N)
                                      or dfinal_states.device != x.device or not dfinal_states.is_contiguous()):
        raise ValueError("dfinal_states must be a contiguous float32 (b, H, P, N) tensor on x's device")
    if want_dinitial_states is None:
        want_dinitial_states = initial_states is not None
    f32 = dict(device=x.device, dtype=torch.float32)
    if dinitial_only:
        g = {k: None for k in ("dx", "ddt", "dA", "dB", "dC", "dD", "dz")}
        g["dinitial_states"] = torch.empty(b, H, P, N, **f32)
    else:
        g = {"dx": torch.empty(b, L, H, P, **f32), "ddt": torch.empty(b, L, H, **f32),
             "dA": torch.empty(H, **f32), "dB": torch.empty(b, L, G, N, **f32), "dC": torch.empty(b, L, G, N, **f32),
             "dD": torch.empty(H, **f32) if want_dD else None,
             "dinitial_states": torch.empty(b, H, P, N, **f32) if want_dinitial_states else None,
             "dz": torch.empty(b, L, H, P, **f32) if z is not None else None}
    a = make_bwd_args(x, dt, A, B, C, D, dy, initial_states, seq_idx, dfinal_states, chunk_size)
    a.dx, a.ddt, a.dA, a.dB, a.dC = (_ptr(g[k]) for k in ("dx", "ddt", "dA", "dB", "dC"))
    a.dD, a.dinitial_states = _ptr(g["dD"]), _ptr(g["dinitial_states"])
    a.z, a.dz = _ptr(z), _ptr(g["dz"])
    a.flags = SSD_BWD_DINITIAL_ONLY if dinitial_only else 0
    need = int(lib.ssd_bwd_workspace_size(ctypes.byref(a)))
    if need == 0:  # sizes the library rejects: let it say why (nothing is enqueued)
        raise SSDError(lib.ssd_bwd(ctypes.byref(a), _stream(x)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    if timing_events is not None:
        h0_, h1_ = timing_events[0].cuda_event, timing_events[1].cuda_event
        if not h0_ or not h1_:
            raise ValueError("timing events must have been recorded once (torch creates them lazily)")
        a.timing_events[0], a.timing_events[1] = h0_, h1_
    st = lib.ssd_bwd(ctypes.byref(a), _stream(x))
    if st != SSD_OK:
        raise SSDError(st)
    return g


class _SSDChunked(torch.autograd.Function):
    """``fwd`` forward, ``bwd`` backward; gradients returned in each input's dtype."""

    @staticmethod
    def forward(ctx, x, dt, A, B, C, D, initial_states, seq_idx, num_seqs, chunk_size, z):
        ctx.set_materialize_grads(False)
        y, fin = fwd(x, dt, A, B, C, D, chunk_size=chunk_size, initial_states=initial_states, seq_idx=seq_idx,
                     num_seqs=num_seqs, z=z)
        ctx.save_for_backward(x, dt, A, B, C, D, initial_states, seq_idx, z)
        return y, fin

    @staticmethod
    def backward(ctx, dy, dfin):
        x, dt, A, B, C, D, h0, seq, z = ctx.saved_tensors
        if seq is not None and dfin is not None:
            raise NotImplementedError("the gradient through per-sequence final states is not supported")
        dy = torch.zeros_like(x) if dy is None else dy.to(x.dtype).contiguous()
        dfin = None if dfin is None else dfin.to(torch.float32).contiguous()
        need = ctx.needs_input_grad
        g = bwd(x, dt, A, B, C, D, dy, initial_states=h0, seq_idx=seq, dfinal_states=dfin,
                want_dD=D is not None and need[5], want_dinitial_states=h0 is not None and need[6], z=z)
        return (g["dx"].to(x.dtype), g["ddt"], g["dA"], g["dB"].to(B.dtype), g["dC"].to(C.dtype), g["dD"],
                g["dinitial_states"], None, None, None, None if z is None else g["dz"].to(z.dtype))


def ssd_chunked(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                D: Optional[torch.Tensor] = None, chunk_size: int = 64,
                initial_states: Optional[torch.Tensor] = None, seq_idx: Optional[torch.Tensor] = None,
                num_seqs: Optional[int] = None, z: Optional[torch.Tensor] = None):
    """Differentiable SSD forward: returns (y, final_states) like ``fwd``
    (y * SiLU(z) with a gate z), and its backward runs ``ssd_bwd`` (the
    states and y are recomputed, nothing but the inputs is kept).  With
    seq_idx the final states carry no gradient."""
    if seq_idx is not None and num_seqs is None:
        num_seqs = int(seq_idx.max().item()) + 1
    return _SSDChunked.apply(x, dt, A, B, C, D, initial_states, seq_idx, num_seqs, chunk_size, z)


def conv1d_silu_bwd(u: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor], dout: torch.Tensor,
                    seq_idx: Optional[torch.Tensor] = None, want_dbias: bool = True) -> tuple:
    """``ssd_conv1d_silu_bwd``: (du (b,L,C), dweight (C,K), dbias (C) or None),
    all fp32, for dout = dLoss/d(conv1d_silu(u, weight, bias, seq_idx))."""
    if u.dim() != 3 or weight.dim() != 2 or weight.shape[0] != u.shape[2]:
        raise ValueError("expected u (b,L,C) and weight (C,K)")
    if dout.dtype != u.dtype or tuple(dout.shape) != tuple(u.shape):
        raise ValueError("dout must be like u")
    if u.dtype not in (torch.float32, torch.bfloat16) or weight.dtype != torch.float32 \
            or (bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (u.shape[2],))):
        raise TypeError("u float32 or bfloat16; weight and bias float32 (bias of shape (C,))")
    if seq_idx is not None and (seq_idx.dtype != torch.int32 or tuple(seq_idx.shape) != tuple(u.shape[:2])):
        raise ValueError("seq_idx must be int32 (b,L)")
    for name, t in (("u", u), ("weight", weight), ("bias", bias), ("seq_idx", seq_idx), ("dout", dout)):
        if t is not None and (t.device != u.device or u.device.type != "cuda" or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor on {u.device}")
    b, L, C = u.shape
    f32 = dict(device=u.device, dtype=torch.float32)
    du, dw = torch.empty(b, L, C, **f32), torch.empty(weight.shape, **f32)
    db = torch.empty(C, **f32) if want_dbias else None
    a = ConvBwdArgs()
    a.batch, a.seqlen, a.channels, a.width = b, L, C, weight.shape[1]
    a.dtype = SSD_BF16 if u.dtype == torch.bfloat16 else SSD_F32
    a.u, a.weight, a.bias, a.seq_idx, a.dout = _ptr(u), _ptr(weight), _ptr(bias), _ptr(seq_idx), _ptr(dout)
    a.du, a.dweight, a.dbias = _ptr(du), _ptr(dw), _ptr(db)
    need = int(lib.ssd_conv1d_silu_bwd_workspace_size(ctypes.byref(a)))
    if need == 0:
        raise SSDError(lib.ssd_conv1d_silu_bwd(ctypes.byref(a), _stream(u)))
    ws = torch.empty(need, dtype=torch.uint8, device=u.device)
    a.workspace, a.workspace_bytes = ws.data_ptr(), need
    st = lib.ssd_conv1d_silu_bwd(ctypes.byref(a), _stream(u))
    if st != SSD_OK:
        raise SSDError(st)
    return du, dw, db


class _CausalConv1dSilu(torch.autograd.Function):
    """``conv1d_silu`` forward, ``conv1d_silu_bwd`` backward."""

    @staticmethod
    def forward(ctx, u, weight, bias, seq_idx):
        ctx.save_for_backward(u, weight, bias, seq_idx)
        return conv1d_silu(u, weight, bias, seq_idx)

    @staticmethod
    def backward(ctx, dout):
        u, weight, bias, seq_idx = ctx.saved_tensors
        du, dw, db = conv1d_silu_bwd(u, weight, bias, dout.to(u.dtype).contiguous(), seq_idx,
                                     want_dbias=bias is not None and ctx.needs_input_grad[2])
        return du.to(u.dtype), dw, db, None


def causal_conv1d_silu(u: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None,
                       seq_idx: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Differentiable ``conv1d_silu``: the backward runs ``ssd_conv1d_silu_bwd``
    (the pre-activation is recomputed, nothing but the inputs is kept)."""
    return _CausalConv1dSilu.apply(u, weight, bias, seq_idx)
