"""Build and run the test-only host emulation of the backward kernels
(``tests/emu/bwd_emu.cpp`` for ``csrc/ssd_bwd.cuh``, ``tests/emu/conv_bwd_emu.cpp``
for ``csrc/ssd_conv_bwd.cuh``): the kernels and the host plan that launches
them, compiled by g++ with a sanitizer and run on small inputs on the CPU.  Used by the CPU tests only, to check indexing,
barriers and arithmetic before the code runs on a GPU; the GPU tests are the
parity claim."""
from __future__ import annotations

import os
import shutil
import subprocess
import tempfile

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "emu", "bwd_emu.cpp")
SHIM = os.path.join(HERE, "emu", "cuda_emu.h")
LAUNCH = os.path.join(HERE, "emu", "emu_launch.h")
KERNELS = os.path.join(ROOT, "mamba_ssd_chunked_03_b200", "csrc", "ssd_bwd.cuh")
HEADER = os.path.join(ROOT, "include", "ssd.h")
OUT = os.path.join(HERE, "emu", "_build")

# asan: fibers under AddressSanitizer + UBSan; tsan: host threads under ThreadSanitizer
SANITIZERS = {"asan": ["-fsanitize=address,undefined", "-fno-sanitize-recover=all"],
              "tsan": ["-fsanitize=thread", "-DSSD_EMU_THREADS"]}


def available() -> bool:
    return shutil.which("g++") is not None


CONV_SRC = os.path.join(HERE, "emu", "conv_bwd_emu.cpp")
CONV_KERNELS = os.path.join(ROOT, "mamba_ssd_chunked_03_b200", "csrc", "ssd_conv_bwd.cuh")


def build(kind: str = "asan", which: str = "ssd") -> str:
    os.makedirs(OUT, exist_ok=True)
    src, kernels = (SRC, KERNELS) if which == "ssd" else (CONV_SRC, CONV_KERNELS)
    exe = os.path.join(OUT, f"{'bwd' if which == 'ssd' else 'conv_bwd'}_emu_{kind}")
    deps = [src, SHIM, LAUNCH, kernels, HEADER, os.path.abspath(__file__)]
    if os.path.exists(exe) and os.path.getmtime(exe) >= max(os.path.getmtime(d) for d in deps):
        return exe
    tmp = exe + f".tmp{os.getpid()}"
    cmd = ["g++", "-std=c++20", "-O1", "-g", "-fno-omit-frame-pointer", *SANITIZERS[kind], "-pthread",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.dirname(kernels), "-I", os.path.dirname(SHIM),
           src, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, exe)
    return exe


def _raw(t) -> bytes:
    if isinstance(t, torch.Tensor):
        t = t.contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().tobytes()
        return t.numpy().tobytes()
    return np.ascontiguousarray(t).tobytes()


def run(inp: dict, dy, dfinal=None, chunk_size: int = 0, want_dD: bool = True, want_dh0: bool = True,
        kind: str = "asan", reverse: bool = False, timeout: int = 600, z=None, flags: int = 0) -> dict:
    """Run the emulated backward on ``inp`` (``ssd_inputs.make_inputs`` form)
    with upstream gradient ``dy`` (x's dtype) and ``dfinal`` (fp32 or None).
    ``reverse`` runs each block's threads in reverse order (fiber builds).
    ``z``: the forward's gate (x's dtype), dy then being the gradient of the
    gated output.
    Returns {"status", "chunk", and the fp32 gradients as numpy arrays}."""
    exe = build(kind)
    x = inp["x"]
    b, L, H, P = x.shape
    G, N = inp["B"].shape[2], inp["B"].shape[3]
    with tempfile.TemporaryDirectory() as d:
        arrays = {"x": x, "dt": inp["dt"], "A": inp["A"], "B": inp["B"], "C": inp["C"], "D": inp.get("D"),
                  "h0": inp.get("initial_states"), "seq": inp.get("seq_idx"), "dy": dy, "dfinal": dfinal,
                  "z": z}
        for k, v in arrays.items():
            if v is not None:
                with open(os.path.join(d, k + ".bin"), "wb") as f:
                    f.write(_raw(v))
        kv = dict(batch=b, seqlen=L, nheads=H, headdim=P, dstate=N, ngroups=G, chunk_size=chunk_size,
                  dtype=1 if x.dtype == torch.bfloat16 else 0, has_D=int(arrays["D"] is not None),
                  has_h0=int(arrays["h0"] is not None), has_seq=int(arrays["seq"] is not None),
                  has_dfinal=int(dfinal is not None), want_dD=int(want_dD), want_dh0=int(want_dh0),
                  reverse=int(reverse), has_z=int(z is not None), flags=int(flags))
        with open(os.path.join(d, "args.txt"), "w") as f:
            f.write("".join(f"{k} {v}\n" for k, v in kv.items()))
        env = dict(os.environ)
        env.setdefault("ASAN_OPTIONS", "detect_leaks=0")
        env.setdefault("TSAN_OPTIONS", "halt_on_error=1")
        r = subprocess.run([exe, d], capture_output=True, text=True, timeout=timeout, env=env)
        words = r.stdout.split()
        if r.returncode not in (0, 1) or len(words) < 6 or words[0] != "status":
            raise RuntimeError(f"emulator failed (rc {r.returncode}):\n{r.stdout}\n{r.stderr[-4000:]}")
        out = {"status": int(words[1]), "launches": int(words[3]), "chunk": int(words[5]), "stderr": r.stderr}
        if out["status"] != 0:
            return out
        shapes = {"dx": (b, L, H, P), "ddt": (b, L, H), "dA": (H,), "dB": (b, L, G, N), "dC": (b, L, G, N),
                  "dD": (H,), "dh0": (b, H, P, N), "dz": (b, L, H, P)}
        for k, shp in shapes.items():
            path = os.path.join(d, k + ".bin")
            out[k] = np.fromfile(path, dtype=np.float32).reshape(shp) if os.path.exists(path) else None
        return out


def run_conv(u, weight, bias, dout, seq_idx=None, want_dbias: bool = True, kind: str = "asan",
             reverse: bool = False, timeout: int = 600) -> dict:
    """Run the emulated conv1d + SiLU backward.  Returns {"status",
    "launches", and du (b,L,C), dw (C,K), dbias (C) as fp32 numpy arrays}."""
    exe = build(kind, which="conv")
    b, L, C = u.shape
    K = weight.shape[1]
    with tempfile.TemporaryDirectory() as d:
        for name, v in (("u", u), ("w", weight), ("bias", bias), ("seq", seq_idx), ("dout", dout)):
            if v is not None:
                with open(os.path.join(d, name + ".bin"), "wb") as f:
                    f.write(_raw(v))
        kv = dict(batch=b, seqlen=L, channels=C, width=K, dtype=1 if u.dtype == torch.bfloat16 else 0,
                  has_bias=int(bias is not None), has_seq=int(seq_idx is not None), want_dbias=int(want_dbias),
                  reverse=int(reverse))
        with open(os.path.join(d, "args.txt"), "w") as f:
            f.write("".join(f"{k} {v}\n" for k, v in kv.items()))
        env = dict(os.environ)
        env.setdefault("ASAN_OPTIONS", "detect_leaks=0")
        r = subprocess.run([exe, d], capture_output=True, text=True, timeout=timeout, env=env)
        words = r.stdout.split()
        if r.returncode not in (0, 1) or len(words) < 4 or words[0] != "status":
            raise RuntimeError(f"emulator failed (rc {r.returncode}):\n{r.stdout}\n{r.stderr[-4000:]}")
        out = {"status": int(words[1]), "launches": int(words[3])}
        if out["status"] != 0:
            return out
        out["du"] = np.fromfile(os.path.join(d, "du.bin"), dtype=np.float32).reshape(b, L, C)
        out["dw"] = np.fromfile(os.path.join(d, "dw.bin"), dtype=np.float32).reshape(C, K)
        p = os.path.join(d, "dbias.bin")
        out["dbias"] = np.fromfile(p, dtype=np.float32) if os.path.exists(p) else None
        return out
