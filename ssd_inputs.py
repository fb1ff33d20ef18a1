"""Seeded synthetic inputs for the chunked SSD forward.

This module only draws random tensors: it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle may take their inputs
from it without sharing any computation.

Distributions follow the workloads on the pages' subject (Mamba-2 SSD layer
shapes): x, B, C ~ N(0, 1); A_h = -exp(U(ln 1, ln 16)); dt = exp(U(ln 1e-3,
ln 1e-1)); D ~ N(0, 1); initial states zero unless a config draws them.
Packed variable-length inputs concatenate sequences whose lengths are drawn
uniformly from an integer range and truncate the last one to hit the token
total exactly.

Every tensor is created on the CPU with its own ``torch.Generator``; values
meant for a bf16 path are drawn in fp32 and then rounded to bf16 once, so the
oracle (which upcasts) and the GPU see identical numbers.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional

import torch

_SLICE = 1 << 22  # elements per independently seeded slice of a large draw


def _randn(shape, gen: torch.Generator) -> torch.Tensor:
    """N(0,1) fp32 draw of ``shape``.  Large draws are cut into fixed slices,
    each with a generator seeded from ``gen``, and filled on a thread pool;
    the values depend only on the seed, never on the thread count."""
    n = 1
    for d in shape:
        n *= d
    if n <= _SLICE:
        return torch.randn(*shape, generator=gen)
    nslices = -(-n // _SLICE)
    seeds = torch.randint(0, 2**62, (nslices,), generator=gen, dtype=torch.int64).tolist()
    out = torch.empty(n)

    def fill(i):
        g = torch.Generator().manual_seed(int(seeds[i]))
        lo = i * _SLICE
        hi = min(n, lo + _SLICE)
        out[lo:hi] = torch.randn(hi - lo, generator=g)

    from concurrent.futures import ThreadPoolExecutor
    import os
    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(nslices)))
    return out.view(*shape)


@dataclass(frozen=True)
class SSDShape:
    """One SSD forward workload: shapes, dtype and the random recipe."""

    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk_size: int
    dtype: str = "bf16"  # dtype of x, B, C and y: "bf16" or "f32"
    h0_std: float = 0.0  # > 0: initial_states ~ N(0, h0_std^2)
    packed: Optional[tuple] = None  # (min_len, max_len) of packed sequences
    seed: int = 1000
    has_D: bool = True

    def with_(self, **kw) -> "SSDShape":
        return replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


def _c2(n: int, q: int) -> SSDShape:
    return SSDShape(f"c2_N{n}_Q{q}", 8, 2048, 80, 64, n, 1, q, "bf16", seed=1002)


# The five workload families of the benchmark (c2 is a 3x3 sweep).
CONFIGS = {
    "c0": SSDShape("c0", 1, 256, 2, 16, 16, 1, 64, "f32", seed=1000),
    "c1": SSDShape("c1", 8, 2048, 80, 64, 128, 1, 64, "bf16", seed=1001),
    **{f"c2_N{n}_Q{q}": _c2(n, q) for n in (64, 128, 256) for q in (64, 128, 256)},
    "c3": SSDShape("c3", 1, 16384, 80, 64, 128, 1, 128, "bf16", h0_std=0.1, seed=1003),
    "c4": SSDShape("c4", 1, 32768, 64, 64, 256, 8, 256, "bf16", packed=(128, 4096), seed=1004),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def packed_lengths(total: int, lo: int, hi: int, gen: torch.Generator) -> list:
    """Integer lengths ~ U[lo, hi] drawn until their sum reaches ``total``;
    the last one is truncated so the lengths sum to ``total`` exactly."""
    lens = []
    acc = 0
    while acc < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return lens


def make_inputs(shape: SSDShape, seed: Optional[int] = None) -> dict:
    """Draw one seeded input set on the CPU.

    Returns a dict with x (b,L,H,P), dt (b,L,H), A (H), B and C (b,L,G,N),
    D (H) or None, initial_states (b,H,P,N) or None, seq_idx (b,L) int32 or
    None and num_seqs (int or None).  x, B, C carry the path dtype; the rest
    are fp32 (seq_idx int32).
    """
    s = shape
    gen = torch.Generator().manual_seed(s.seed if seed is None else seed)
    dt_path = torch_dtype(s.dtype)
    b, L, H, P, N, G = s.batch, s.seqlen, s.nheads, s.headdim, s.dstate, s.ngroups

    x = _randn((b, L, H, P), gen).to(dt_path)
    B = _randn((b, L, G, N), gen).to(dt_path)
    C = _randn((b, L, G, N), gen).to(dt_path)
    A = -torch.exp(torch.empty(H).uniform_(math.log(1.0), math.log(16.0), generator=gen))
    dt = torch.exp(torch.empty(b, L, H).uniform_(math.log(1e-3), math.log(1e-1), generator=gen))
    D = torch.randn(H, generator=gen) if s.has_D else None
    h0 = None
    if s.h0_std > 0:
        h0 = _randn((b, H, P, N), gen) * s.h0_std
    seq_idx = None
    num_seqs = None
    if s.packed is not None:
        lo, hi = s.packed
        rows = []
        base = 0
        for _ in range(b):
            lens = packed_lengths(L, lo, hi, gen)
            ids = torch.repeat_interleave(torch.arange(base, base + len(lens), dtype=torch.int32),
                                          torch.tensor(lens))
            rows.append(ids)
            base += len(lens)
        seq_idx = torch.stack(rows).to(torch.int32).contiguous()
        num_seqs = base
    return dict(x=x.contiguous(), dt=dt.contiguous(), A=A.contiguous(), B=B.contiguous(),
                C=C.contiguous(), D=D, initial_states=h0, seq_idx=seq_idx, num_seqs=num_seqs)


def seq_idx_from_lengths(rows_lengths: list) -> tuple:
    """seq_idx (b, L) int32 from per-row length lists (ids numbered across rows)."""
    rows = []
    base = 0
    for lens in rows_lengths:
        ids = torch.repeat_interleave(torch.arange(base, base + len(lens), dtype=torch.int32),
                                      torch.tensor(lens))
        rows.append(ids)
        base += len(lens)
    return torch.stack(rows).to(torch.int32).contiguous(), base
