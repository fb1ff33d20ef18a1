"""Sequence parallelism for the SSD forward over ``torch.distributed`` ranks.

Each of R ranks holds a contiguous range of the tokens of every row
(x (b, L_r, H, P), dt, B, C alike).  The recurrence is affine in the state,
so over rank k's range it is h_out = D_k h_in + S_k:

1. every rank runs its range from a zero state: S_k = its end state, and
   D_k = exp(A_h * sum of its dt) (``ssd_total_decay``);
2. the ranks all-gather (S_k, D_k) -- the one exchange step;
3. rank r starts from h0 carried through ranks 0..r-1 (``ssd_state_fold``)
   and runs its range again from that state, which gives its y and the state
   at its range's end (rank R-1's is the sequence's final state).

That is the state passing of "SSM 家族全景图（下）：Mamba-2 与 Jamba" section
三.4 with a rank's range as one chunk.  All arithmetic runs in the library's
kernels; this module only calls them and moves the states between ranks.
Packed sequences (seq_idx) are not split this way.

The backward (``bwd_seqpar``) is the same exchange run the other way.  The
gradient with respect to the state entering rank k's range is
D_k Lam_k + T_k, where Lam_k is the gradient with respect to the state
leaving it and T_k comes from the range's own outputs alone (the backward's
dinitial_states when no state gradient comes in).  So:

1. every rank recovers h_in as in the forward, and computes T_k: the
   backward's dinitial_states with no incoming state gradient (which does not
   depend on h_in; ``ssd_bwd`` with ``SSD_BWD_DINITIAL_ONLY`` runs two of its
   six kernels for it);
2. the ranks all-gather (T_k, D_k);
3. rank r folds Lam_r from the sequence's dfinal through ranks R-1..r+1
   (``ssd_state_fold`` over the reversed lists) and runs its backward again
   with h_in and Lam_r, which gives its tokens' gradients;
4. dA and dD, which sum over all tokens, are all-reduced.

With the block's gate z (out = y * SiLU(z)) only the outputs change: the
exchanged states do not depend on z, so the forward passes z to its final
local pass, and the backward to its adjoint summary and final pass.

The per-rank operations are taken from ``ops`` (default: the library), so the
exchange logic can be exercised on CPU ranks with another implementation of
them.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import bwd, fwd, state_fold, total_decay


class LibraryOps:
    """The per-rank operations, on the library's kernels."""

    @staticmethod
    def local_forward(x, dt, A, B, C, D, chunk_size, initial_states, z=None):
        return fwd(x, dt, A, B, C, D, chunk_size=chunk_size, initial_states=initial_states, z=z)

    @staticmethod
    def total_decay(dt, A):
        return total_decay(dt, A)

    @staticmethod
    def state_fold(states, decays, initial_states, rank, shape):
        return state_fold(states, decays, initial_states, rank, shape)

    @staticmethod
    def local_backward(x, dt, A, B, C, D, dy, initial_states, dfinal_states, z=None):
        return bwd(x, dt, A, B, C, D, dy, initial_states=initial_states, dfinal_states=dfinal_states,
                   want_dD=D is not None, want_dinitial_states=True, z=z)

    @staticmethod
    def adjoint_summary(x, dt, A, B, C, D, dy, z=None):
        """T: dLoss/d(the state entering the range) from the range's own
        outputs (no state gradient coming in), without the other gradients."""
        return bwd(x, dt, A, B, C, D, dy, dinitial_only=True, z=z)["dinitial_states"]


def local_summary(x, dt, A, B, C, D, chunk_size: int = 64, ops=LibraryOps):
    """(S, D_total) of this rank's range: its end state from a zero state and
    its total decay, (b,H,P,N) and (b,H) fp32."""
    _, S = ops.local_forward(x, dt, A, B, C, D, chunk_size, None)
    return S, ops.total_decay(dt, A)


def carry_in(states, decays, initial_states, rank: int, shape, ops=LibraryOps):
    """The state before rank ``rank``'s first token, from the gathered
    summaries of ranks 0..rank-1 (states (R,b,H,P,N), decays (R,b,H))."""
    return ops.state_fold(states, decays, initial_states, rank, shape)


def _state_in(x, dt, A, B, C, D, chunk_size, initial_states, group, ops):
    """(h_in of this rank, the gathered total decays (R,b,H), the state shape)."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    S, dec = local_summary(x, dt, A, B, C, D, chunk_size, ops)
    all_S = [torch.empty_like(S) for _ in range(R)]
    all_d = [torch.empty_like(dec) for _ in range(R)]
    dist.all_gather(all_S, S.contiguous(), group=group)
    dist.all_gather(all_d, dec.contiguous(), group=group)
    decays = torch.stack(all_d)
    return carry_in(torch.stack(all_S), decays, initial_states, r, tuple(S.shape), ops), decays, tuple(S.shape)


def fwd_seqpar(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
               D: Optional[torch.Tensor], chunk_size: int = 64, initial_states: Optional[torch.Tensor] = None,
               group=None, ops=LibraryOps, z: Optional[torch.Tensor] = None):
    """The forward of this rank's token range of a sequence split over the
    ranks of ``group``, in rank order.  ``initial_states`` (the state before
    the sequence's first token, or None) must be the same on every rank;
    ``z``, this rank's gate (like x), or None.  Returns (y of this rank's
    tokens, y * SiLU(z) with a gate, and the state at the end of its range)."""
    h_in, _, _ = _state_in(x, dt, A, B, C, D, chunk_size, initial_states, group, ops)
    if z is None:
        return ops.local_forward(x, dt, A, B, C, D, chunk_size, h_in)
    return ops.local_forward(x, dt, A, B, C, D, chunk_size, h_in, z=z)


def bwd_seqpar(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
               D: Optional[torch.Tensor], dy: torch.Tensor, chunk_size: int = 64,
               initial_states: Optional[torch.Tensor] = None, dfinal_states: Optional[torch.Tensor] = None,
               group=None, ops=LibraryOps, z: Optional[torch.Tensor] = None) -> dict:
    """The backward of ``fwd_seqpar`` for this rank's token range.  ``dy`` is
    dLoss/dy of this rank's tokens (of y * SiLU(z) with this rank's gate z);
    ``initial_states`` and ``dfinal_states`` (dLoss/d(the sequence's final
    state)), each None or the same on every rank.  Returns a dict: dx, ddt,
    dB, dC (and dz) of this rank's tokens; dA and dD summed over all ranks;
    dinitial_states on rank 0 (None elsewhere)."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    r = dist.get_rank(group)
    h_in, decays, shape = _state_in(x, dt, A, B, C, D, chunk_size, initial_states, group, ops)
    gate = {} if z is None else {"z": z}
    if hasattr(ops, "adjoint_summary"):
        T = ops.adjoint_summary(x, dt, A, B, C, D, dy, **gate)
    else:
        T = ops.local_backward(x, dt, A, B, C, D, dy, h_in, None, **gate)["dinitial_states"]
    all_T = [torch.empty_like(T) for _ in range(R)]
    dist.all_gather(all_T, T.contiguous(), group=group)
    after = list(range(R - 1, r, -1))  # the ranks after this one, last first
    lam = ops.state_fold(torch.stack([all_T[k] for k in after]) if after else None,
                         torch.stack([decays[k] for k in after]) if after else None,
                         dfinal_states, len(after), shape)
    g = ops.local_backward(x, dt, A, B, C, D, dy, h_in, lam, **gate)
    dist.all_reduce(g["dA"], group=group)
    if g.get("dD") is not None:
        dist.all_reduce(g["dD"], group=group)
    if r != 0:
        g["dinitial_states"] = None
    return g
