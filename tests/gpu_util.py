"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library and the oracle on the same numbers, and measure the error the way
the tolerances are stated (relative L2 over y; max-abs over final states
scaled by max(1, max|ref|))."""
from __future__ import annotations

import numpy as np
import torch

import mamba_ssd_chunked_03_b200 as ssd
import oracle

KEYS = ("x", "dt", "A", "B", "C", "D", "initial_states")
TOL = {"f32": 1e-5, "bf16": 1e-2}


def to_dev(d, device="cuda"):
    out = {}
    for k, v in d.items():
        out[k] = v.to(device) if isinstance(v, torch.Tensor) else v
    return out


def run_gpu(d, chunk_size, generic=False):
    g = to_dev(d)
    y, f = ssd.fwd(g["x"], g["dt"], g["A"], g["B"], g["C"], g["D"], chunk_size=chunk_size,
                   initial_states=g["initial_states"], seq_idx=g.get("seq_idx"), num_seqs=d.get("num_seqs"),
                   generic=generic)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64), f.cpu().numpy().astype(np.float64)


def run_oracle(d, units=None):
    return oracle.ssd_fwd(*[d[k] for k in KEYS], seq_idx=d.get("seq_idx"), num_seqs=d.get("num_seqs"),
                          units=units)


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))


def state_err(a, b):
    return float(np.abs(a - b).max() / max(1.0, float(np.abs(b).max()))) if b.size else 0.0


def units_view(y, f, units, H, packed_rows=None):
    """Stack the (b, h) slices of y (and of f when not packed) for the units."""
    ys = np.stack([y[u // H, :, u % H] for u in units])
    fs = None if packed_rows is not None else np.stack([f[u // H, u % H] for u in units])
    return ys, fs
