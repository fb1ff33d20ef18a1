"""The C-ABI library: loads, exports every declared symbol, validates on the
host.  CPU only: no call here reaches a kernel launch."""
import ctypes
import os
import re

import pytest

import mamba_ssd_chunked_03_b200 as ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"SSD_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert "ssd_fwd" in names and "ssd_fwd_workspace_size" in names
    raw = ctypes.CDLL(ssd.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/ but not exported"


def test_status_strings_and_version():
    for s in range(6):
        assert ssd.lib.ssd_status_string(s)
    assert ssd.lib.ssd_status_string(99) == b"unknown status"
    assert ssd.lib.ssd_version() >= 100


def base_args(**kw):
    a = ssd.Args()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk_size = 2, 100, 4, 64, 128, 2, 64
    a.dtype = ssd.SSD_BF16
    fake = 1 << 20  # never dereferenced: every case below is rejected on the host
    a.x = a.dt = a.A = a.B = a.C = a.y = fake
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def call(a):
    return ssd.lib.ssd_fwd(ctypes.byref(a), None)


@pytest.mark.parametrize("field,value,status", [
    ("batch", 0, ssd.SSD_ERR_INVALID_ARG),
    ("seqlen", -1, ssd.SSD_ERR_INVALID_ARG),
    ("nheads", 0, ssd.SSD_ERR_INVALID_ARG),
    ("ngroups", 3, ssd.SSD_ERR_INVALID_ARG),       # H % G != 0
    ("chunk_size", 48, ssd.SSD_ERR_INVALID_ARG),   # not a power of two
    ("chunk_size", 8, ssd.SSD_ERR_INVALID_ARG),    # below 16
    ("chunk_size", 512, ssd.SSD_ERR_INVALID_ARG),  # above 256
    ("dtype", 7, ssd.SSD_ERR_INVALID_ARG),
    ("flags", 8, ssd.SSD_ERR_INVALID_ARG),
    ("headdim", 12, ssd.SSD_ERR_UNSUPPORTED),
    ("dstate", 512, ssd.SSD_ERR_UNSUPPORTED),
    ("x", None, ssd.SSD_ERR_INVALID_ARG),
    ("dt", None, ssd.SSD_ERR_INVALID_ARG),
    ("A", None, ssd.SSD_ERR_INVALID_ARG),
    ("B", None, ssd.SSD_ERR_INVALID_ARG),
    ("C", None, ssd.SSD_ERR_INVALID_ARG),
    ("y", None, ssd.SSD_ERR_INVALID_ARG),
    ("x", (1 << 20) + 8, ssd.SSD_ERR_INVALID_ARG),  # misaligned
    ("final_states", (1 << 20) + 4, ssd.SSD_ERR_INVALID_ARG),
])
def test_bad_argument_rejected(field, value, status):
    assert call(base_args(**{field: value})) == status


def test_seq_idx_needs_num_seqs():
    assert call(base_args(seq_idx=1 << 20, num_seqs=0)) == ssd.SSD_ERR_INVALID_ARG


def test_null_args_pointer():
    assert ssd.lib.ssd_fwd(None, None) == ssd.SSD_ERR_INVALID_ARG
    assert ssd.lib.ssd_fwd_workspace_size(None) == 0


def test_workspace_checked_before_launch():
    a = base_args()
    need = ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a))
    assert need > 0
    assert call(a) == ssd.SSD_ERR_WORKSPACE                 # none given
    a.workspace, a.workspace_bytes = 1 << 24, need - 1
    assert call(a) == ssd.SSD_ERR_WORKSPACE                 # one byte short
    a.workspace, a.workspace_bytes = (1 << 24) + 16, need
    assert call(a) == ssd.SSD_ERR_INVALID_ARG               # not 256-byte aligned


def test_workspace_size_is_pure_and_monotone():
    a = base_args(flags=ssd.SSD_FLAG_GENERIC)
    w1 = ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a))
    a.seqlen = 1000
    w2 = ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a))
    assert w2 > w1
    a.chunk_size = 48
    assert ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a)) == 0


def test_kernel_path_query():
    a = base_args()
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) in (b"generic", b"tcgen05")
    a.flags = ssd.SSD_FLAG_GENERIC
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"generic"
    a.chunk_size = 3
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"invalid"


def test_struct_layout_matches_header():
    # 7 int64 sizes, dtype + flags, 8 pointers, num_seqs, 2 outputs, workspace + bytes, events, z
    assert ctypes.sizeof(ssd.Args) == 7 * 8 + 4 + 4 + 8 * 8 + 8 + 2 * 8 + 8 + 8 + 2 * 8 + 8
    assert ssd.Args.x.offset == 64 and ssd.Args.num_seqs.offset == 128
    assert ssd.Args.timing_events.offset == 168


def test_timing_events_both_or_neither():
    a = base_args()
    a.timing_events[0] = 1 << 12
    assert call(a) == ssd.SSD_ERR_INVALID_ARG


def test_launch_count_query():
    a = base_args()
    n = ssd.lib.ssd_fwd_launch_count(ctypes.byref(a))
    assert n >= 1
    a.chunk_size = 3
    assert ssd.lib.ssd_fwd_launch_count(ctypes.byref(a)) == 0


def _c_layout(fields, struct):
    """offsetof/sizeof of a header struct, from a C program compiled here."""
    import subprocess
    import tempfile
    body = "\n".join(f'printf("%zu\\n", offsetof({struct}, {f}));' for f in fields)
    src = (f'#include <stddef.h>\n#include <stdio.h>\n#include "ssd.h"\n'
           f'int main(void) {{ {body} printf("%zu\\n", sizeof({struct})); return 0; }}\n')
    with tempfile.TemporaryDirectory() as tmp:
        c, exe = os.path.join(tmp, "l.c"), os.path.join(tmp, "l")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    return [int(v) for v in out]


def test_step_struct_layout_matches_the_compiled_header():
    names = [f[0] for f in ssd.StepArgs._fields_]
    got = _c_layout(names, "ssd_step_args")
    assert got[:-1] == [getattr(ssd.StepArgs, n).offset for n in names]
    assert got[-1] == ctypes.sizeof(ssd.StepArgs)


def test_fwd_struct_layout_matches_the_compiled_header():
    names = [f[0] for f in ssd.Args._fields_]
    got = _c_layout(names, "ssd_fwd_args")
    assert got[:-1] == [getattr(ssd.Args, n).offset for n in names]
    assert got[-1] == ctypes.sizeof(ssd.Args)


def _step_args(**kw):
    a = ssd.StepArgs()
    a.batch, a.nheads, a.headdim, a.dstate, a.ngroups = 2, 4, 64, 128, 2
    a.dtype = ssd.SSD_BF16
    # placeholders that are never dereferenced: every case below is rejected on the host
    for i, n in enumerate(("x", "dt", "A", "B", "C", "D", "state", "y")):
        setattr(a, n, 4096 * (i + 1))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    ({"batch": 0}, ssd.SSD_ERR_INVALID_ARG),
    ({"nheads": 6, "ngroups": 4}, ssd.SSD_ERR_INVALID_ARG),
    ({"dtype": 7}, ssd.SSD_ERR_INVALID_ARG),
    ({"x": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"state": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"state": 4096 + 8}, ssd.SSD_ERR_INVALID_ARG),   # not 16-byte aligned
    ({"B": 4096 + 4}, ssd.SSD_ERR_INVALID_ARG),       # not aligned to 4 bf16
    ({"dstate": 130}, ssd.SSD_ERR_UNSUPPORTED),
    ({"dstate": 512}, ssd.SSD_ERR_UNSUPPORTED),
])
def test_step_rejects_bad_arguments(kw, status):
    assert ssd.lib.ssd_step(ctypes.byref(_step_args(**kw)), None) == status


def test_step_null_args_pointer():
    assert ssd.lib.ssd_step(None, None) == ssd.SSD_ERR_INVALID_ARG


def _conv_args(**kw):
    a = ssd.ConvArgs()
    a.batch, a.seqlen, a.channels, a.width = 2, 64, 64, 4
    a.dtype = ssd.SSD_BF16
    for i, n in enumerate(("u", "weight", "bias", "seq_idx", "out")):  # never dereferenced: all rejected
        setattr(a, n, 4096 * (i + 1))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    ({"batch": 0}, ssd.SSD_ERR_INVALID_ARG),
    ({"width": 0}, ssd.SSD_ERR_INVALID_ARG),
    ({"u": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"out": 4096 + 8}, ssd.SSD_ERR_INVALID_ARG),
    ({"width": 5}, ssd.SSD_ERR_UNSUPPORTED),
    ({"channels": 62}, ssd.SSD_ERR_UNSUPPORTED),   # not a multiple of 4
])
def test_conv_rejects_bad_arguments(kw, status):
    assert ssd.lib.ssd_conv1d_silu(ctypes.byref(_conv_args(**kw)), None) == status


def test_conv_struct_layout_matches_the_compiled_header():
    names = [f[0] for f in ssd.ConvArgs._fields_]
    got = _c_layout(names, "ssd_conv_args")
    assert got[:-1] == [getattr(ssd.ConvArgs, n).offset for n in names]
    assert got[-1] == ctypes.sizeof(ssd.ConvArgs)


def test_packed_dispatch_queries():
    """Packed sequences take the per-sequence fast path: run list, C B^T per
    run chunk, the single-head kernel per (run, head), the exact kernel; with
    final states, the zeroing of ids that never occur after the run list."""
    a = base_args(seq_idx=1 << 21, num_seqs=8)
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"tcgen05"
    assert ssd.lib.ssd_fwd_main_kernel(ctypes.byref(a)) == b"k_ssd_fwd_fast"
    assert ssd.lib.ssd_fwd_launch_count(ctypes.byref(a)) == 4
    a.final_states = 1 << 22
    assert ssd.lib.ssd_fwd_launch_count(ctypes.byref(a)) == 5


def test_gated_dispatch_queries():
    """A gated call keeps the ungated call's fused kernel: the two-head kernel
    takes the gate in a pass of its own (one more launch), the single-head
    kernel in its epilogue.  An unaligned gate leaves the tensor-core path
    (z is read in 16-byte vectors)."""
    for dt in (1 << 20, (1 << 20) + 4):  # the pair kernel also needs dt 16-byte aligned
        a = base_args(nheads=8, ngroups=1, dt=dt)
        fused = ssd.lib.ssd_fwd_main_kernel(ctypes.byref(a))
        n0 = ssd.lib.ssd_fwd_launch_count(ctypes.byref(a))
        a.z = 1 << 22
        assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"tcgen05"
        assert ssd.lib.ssd_fwd_main_kernel(ctypes.byref(a)) == fused
        assert ssd.lib.ssd_fwd_launch_count(ctypes.byref(a)) == n0 + (1 if fused == b"k_ssd_fwd_pair" else 0)
        a.z = (1 << 22) + 8
        assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"generic"
    assert fused == b"k_ssd_fwd_fast"  # dt not 16-byte aligned


def test_workspace_grows_with_packed_sequences():
    a = base_args()
    plain = ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a))
    a.seq_idx, a.num_seqs = 1 << 21, 50
    assert ssd.lib.ssd_fwd_workspace_size(ctypes.byref(a)) > plain


def _check_seq(rows, num_seqs):
    import numpy as np
    arr = np.ascontiguousarray(np.array(rows, dtype=np.int32))
    return ssd.lib.ssd_check_seq_idx(arr.ctypes.data, arr.shape[0], arr.shape[1], num_seqs)


@pytest.mark.parametrize("rows,num_seqs,status", [
    ([[0, 0, 1, 1, 2]], 3, ssd.SSD_OK),
    ([[0, 0, 1], [2, 2, 3]], 4, ssd.SSD_OK),
    ([[0, 0, 2]], 5, ssd.SSD_OK),                      # ids that never occur are allowed
    ([[0, 1, 0]], 2, ssd.SSD_ERR_INVALID_ARG),         # decreasing along a row
    ([[0, 0, 3]], 3, ssd.SSD_ERR_INVALID_ARG),         # id outside [0, num_seqs)
    ([[-1, 0, 0]], 3, ssd.SSD_ERR_INVALID_ARG),
    ([[0, 0, 1], [1, 1, 2]], 3, ssd.SSD_ERR_INVALID_ARG),  # id 1 in two rows
])
def test_seq_idx_precondition_check(rows, num_seqs, status):
    assert _check_seq(rows, num_seqs) == status


def test_seq_idx_check_rejects_null_and_bad_sizes():
    assert ssd.lib.ssd_check_seq_idx(None, 1, 1, 1) == ssd.SSD_ERR_INVALID_ARG
    assert _check_seq([[0]], 0) == ssd.SSD_ERR_INVALID_ARG


def test_check_flag_is_accepted_and_unknown_flags_rejected():
    a = base_args()
    a.flags = ssd.SSD_FLAG_CHECK_SEQ
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"tcgen05"
    a.flags = ssd.SSD_FLAG_TEST_STALL
    assert ssd.lib.ssd_fwd_path(ctypes.byref(a)) == b"tcgen05"
    a.flags = 8
    assert call(a) == ssd.SSD_ERR_INVALID_ARG


def test_bwd_struct_layout_matches_the_compiled_header():
    names = [f[0] for f in ssd.BwdArgs._fields_]
    got = _c_layout(names, "ssd_bwd_args")
    assert got[:-1] == [getattr(ssd.BwdArgs, n).offset for n in names]
    assert got[-1] == ctypes.sizeof(ssd.BwdArgs)


def _bwd_args(**kw):
    a = ssd.BwdArgs()
    a.batch, a.seqlen, a.nheads, a.headdim, a.dstate, a.ngroups, a.chunk_size = 2, 100, 4, 64, 128, 2, 0
    a.dtype = ssd.SSD_BF16
    # placeholders that are never dereferenced: every case below is rejected on the host
    for i, n in enumerate(("x", "dt", "A", "B", "C", "dy", "dx", "ddt", "dA", "dB", "dC")):
        setattr(a, n, 4096 * (i + 1))
    a.workspace = 1 << 30
    a.workspace_bytes = ssd.lib.ssd_bwd_workspace_size(ctypes.byref(a))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    ({"batch": 0}, ssd.SSD_ERR_INVALID_ARG),
    ({"nheads": 6, "ngroups": 4}, ssd.SSD_ERR_INVALID_ARG),
    ({"dtype": 7}, ssd.SSD_ERR_INVALID_ARG),
    ({"chunk_size": -1}, ssd.SSD_ERR_INVALID_ARG),
    ({"x": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"dy": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"dC": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"workspace": None}, ssd.SSD_ERR_WORKSPACE),
    ({"workspace_bytes": 1024}, ssd.SSD_ERR_WORKSPACE),
    ({"workspace": (1 << 30) + 64}, ssd.SSD_ERR_INVALID_ARG),  # not 256-byte aligned
    ({"seq_idx": 1 << 24, "dfinal_states": 1 << 25}, ssd.SSD_ERR_UNSUPPORTED),
    ({"headdim": 257}, ssd.SSD_ERR_UNSUPPORTED),
    ({"chunk_size": 65}, ssd.SSD_ERR_UNSUPPORTED),
    ({"timing_events": (ctypes.c_void_p * 2)(1 << 12, None)}, ssd.SSD_ERR_INVALID_ARG),  # one event only
    ({"z": 1 << 26}, ssd.SSD_ERR_INVALID_ARG),                                           # a gate without dz
    ({"dz": 1 << 26}, ssd.SSD_ERR_INVALID_ARG),                                          # dz without a gate
])
def test_bwd_rejects_bad_arguments(kw, status):
    assert ssd.lib.ssd_bwd(ctypes.byref(_bwd_args(**kw)), None) == status


def test_bwd_null_args_pointer():
    assert ssd.lib.ssd_bwd(None, None) == ssd.SSD_ERR_INVALID_ARG
    assert ssd.lib.ssd_bwd_workspace_size(None) == 0


def test_bwd_workspace_size():
    size = lambda **kw: ssd.lib.ssd_bwd_workspace_size(ctypes.byref(_bwd_args(**kw)))
    assert size() > 0 and size() % 256 == 0
    assert size(seqlen=200) > size()
    assert size(batch=0) == 0 and size(headdim=300) == 0
    # states per chunk dominate: b*H*ceil(L/Q)*P*N*4 bytes twice, plus dB and dC per head
    b, L, H, P, N = 2, 100, 4, 64, 128
    assert size(chunk_size=64) >= 2 * b * H * 2 * P * N * 4 + 2 * b * L * H * N * 4
    assert size(chunk_size=16) > size(chunk_size=64)
    # dstate 256 does not fit a 64-token chunk: the library halves it
    assert size(dstate=256) == size(dstate=256, chunk_size=32)
    assert size(dstate=256, chunk_size=64) == 0


def test_bwd_chunk_size_query():
    q = lambda **kw: ssd.lib.ssd_bwd_chunk_size(ctypes.byref(_bwd_args(**kw)))
    assert q() == 64
    assert q(chunk_size=16) == 16
    assert q(dstate=256) == 32          # 64 would not fit one CTA's shared memory
    assert q(dstate=256, headdim=128) == 16
    assert q(dstate=256, headdim=256) == 0  # one 256 x 256 state alone exceeds a CTA's shared memory
    assert q(chunk_size=65) == 0 and q(batch=0) == 0
    assert ssd.lib.ssd_bwd_chunk_size(None) == 0


def test_conv_bwd_struct_layout_matches_the_compiled_header():
    names = [f[0] for f in ssd.ConvBwdArgs._fields_]
    got = _c_layout(names, "ssd_conv_bwd_args")
    assert got[:-1] == [getattr(ssd.ConvBwdArgs, n).offset for n in names]
    assert got[-1] == ctypes.sizeof(ssd.ConvBwdArgs)


def _conv_bwd_args(**kw):
    a = ssd.ConvBwdArgs()
    a.batch, a.seqlen, a.channels, a.width = 2, 64, 64, 4
    a.dtype = ssd.SSD_BF16
    for i, n in enumerate(("u", "weight", "dout", "du", "dweight")):
        setattr(a, n, 4096 * (i + 1))  # never dereferenced: every case below is rejected on the host
    a.workspace = 1 << 30
    a.workspace_bytes = ssd.lib.ssd_conv1d_silu_bwd_workspace_size(ctypes.byref(a))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    ({"batch": 0}, ssd.SSD_ERR_INVALID_ARG),
    ({"dtype": 5}, ssd.SSD_ERR_INVALID_ARG),
    ({"u": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"dout": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"dweight": None}, ssd.SSD_ERR_INVALID_ARG),
    ({"workspace": None}, ssd.SSD_ERR_WORKSPACE),
    ({"workspace_bytes": 16}, ssd.SSD_ERR_WORKSPACE),
    ({"workspace": (1 << 30) + 32}, ssd.SSD_ERR_INVALID_ARG),
    ({"width": 5}, ssd.SSD_ERR_UNSUPPORTED),
])
def test_conv_bwd_rejects_bad_arguments(kw, status):
    assert ssd.lib.ssd_conv1d_silu_bwd(ctypes.byref(_conv_bwd_args(**kw)), None) == status


def test_conv_bwd_workspace_size():
    size = lambda **kw: ssd.lib.ssd_conv1d_silu_bwd_workspace_size(ctypes.byref(_conv_bwd_args(**kw)))
    # per (row, strip) and channel: K dweight partials and one dbias partial, fp32;
    # a strip is 64 tokens of bf16 inputs and 32 of fp32 ones
    assert size() == 2 * 1 * 64 * 5 * 4
    assert size(seqlen=65) == 2 * 2 * 64 * 5 * 4
    assert size(dtype=ssd.SSD_F32) == 2 * 2 * 64 * 5 * 4
    assert size(dtype=ssd.SSD_F32, seqlen=65) == 2 * 3 * 64 * 5 * 4
    assert size(batch=0) == 0 and size(width=5) == 0
    assert ssd.lib.ssd_conv1d_silu_bwd(None, None) == ssd.SSD_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    ({"flags": 2}, ssd.SSD_ERR_INVALID_ARG),                               # unknown flag
    ({"flags": 1}, ssd.SSD_ERR_INVALID_ARG),                               # dinitial_states missing
    ({"flags": 1, "dinitial_states": 1 << 27, "dz": 1 << 26}, ssd.SSD_ERR_INVALID_ARG),  # dz without a gate
])
def test_bwd_dinitial_only_rejections(kw, status):
    assert ssd.lib.ssd_bwd(ctypes.byref(_bwd_args(**kw)), None) == status


def _host_call(a, rows=0, ws=None, nbytes=0):
    return ssd.lib.ssd_fwd_host(ctypes.byref(a), rows, ws, nbytes, None, None)


def test_host_workspace_size_by_pieces():
    """ssd_fwd_host's device workspace for one-row and whole-batch pieces, the
    library's default piece size, and 0 for invalid sizes."""
    a = base_args(batch=8)
    one = ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 8)
    per_row = ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 1)
    assert one > 0 and per_row > 0
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 0) == per_row  # b >= 8: b / 8 rows a piece
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 99) == one      # capped at the batch
    # token pieces (rows_per_piece < 0: that many tokens of every row)
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), -64) > 0
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), -100) == one  # one piece: the whole call
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), -1000) == one
    a.seq_idx, a.num_seqs = 1 << 20, 5
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), -64) == 0  # would split sequences
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 1) > one  # one piece with sequence ids
    a.chunk_size = 48
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 1) == 0
    assert ssd.lib.ssd_fwd_host_workspace_size(None, 1) == 0


def test_host_default_pieces_for_a_small_batch():
    """Under eight rows and without sequence ids the library cuts every row
    into eight token pieces of whole 64-token chunks; rows too short for two
    chunks stay one piece.  With sequence ids a single row is cut at sequence
    starts found at call time, so its two buffer sets are sized for the whole
    row; more rows with sequence ids stay one piece."""
    a = base_args(batch=1, seqlen=2000)  # ceil(2000 / 8) = 250 -> 256 tokens a piece
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 0) == \
        ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), -256)
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 0) != \
        ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 1)  # two buffer sets, not one
    short = base_args(batch=1, seqlen=100)
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(short), 0) == \
        ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(short), 1)
    a.seq_idx, a.num_seqs = 1 << 20, 3
    one = ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 1)
    assert 2 * one - 4096 < ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 0) < 2 * one
    two_rows = base_args(batch=2, seqlen=2000, seq_idx=1 << 20, num_seqs=3)
    assert ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(two_rows), 0) == \
        ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(two_rows), 1)


def test_host_call_checked_before_anything_is_enqueued():
    a = base_args(batch=4)
    need = ssd.lib.ssd_fwd_host_workspace_size(ctypes.byref(a), 1)
    assert _host_call(a, 1) == ssd.SSD_ERR_WORKSPACE                     # none given
    assert _host_call(a, 1, 1 << 24, need - 1) == ssd.SSD_ERR_WORKSPACE  # one byte short
    assert _host_call(a, 1, (1 << 24) + 16, need) == ssd.SSD_ERR_INVALID_ARG  # not 256-byte aligned
    assert _host_call(base_args(batch=4, x=None), 1, 1 << 24, need) == ssd.SSD_ERR_INVALID_ARG
    assert _host_call(base_args(batch=4, chunk_size=48), 1, 1 << 24, need) == ssd.SSD_ERR_INVALID_ARG
    assert ssd.lib.ssd_fwd_host(None, 1, None, 0, None, None) == ssd.SSD_ERR_INVALID_ARG
