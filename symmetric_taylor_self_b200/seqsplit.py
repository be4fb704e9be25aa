"""A causal prefill split by sequence across ranks (one GPU each).

[CC-TAYLOR] "Feature maps and linear attention": the states S and Z are sums
over tokens, so the recurrence may be evaluated as a parallel prefix scan.  With
G ranks, rank r holds tokens [r n, (r + 1) n) of every head (q, k, v on its own
GPU) and:

  1. segment state: prefills its tokens from a zero state and keeps the state
     it ends with (dS_r, dZ_r); the outputs of this pass are not used;
  2. exchange: all-gathers (dS, dZ) over the group (NCCL over NVLink on GPUs);
  3. exclusive prefix: adds the states of the ranks before it, in rank order
     (sata_state_accumulate), so every rank sums in the same fixed order;
  4. prefills its tokens again from that prefix state: these are its outputs,
     and the last rank ends with the state of the whole sequence.

The exchange moves G x (d_V + 1) F fp32 values per head to every rank (12.5 MB
per head and rank at d = 64, P = 4).  Every step of the attention runs in
libsata's kernels; torch.distributed carries the states.  Each rank runs two
prefills of its segment, so the step takes about 2/G of a single-GPU prefill
plus the exchange.

The per-rank steps go through an ``impl`` object (``LibraryImpl``, the product
path, by default) so that the exchange logic can also be exercised by tests on
CPU ranks with a reference implementation of the same four methods.
"""
from __future__ import annotations

import torch

from . import binding as _b


class LibraryImpl:
    """The four per-rank steps on libsata (device tensors, the current stream)."""

    def zero_state(self, B, H, d_K, d_V, P, device):
        return _b.State(B, H, d_K, d_V, P, device=device)

    def segment_state(self, q, k, v, P):
        B, H, n, d_K = q.shape
        st = self.zero_state(B, H, d_K, v.shape[-1], P, q.device)
        _b.prefill(q, k, v, P=P, state=st)
        return st

    def accumulate(self, st, S, Z, tokens):
        _b.sata_state_accumulate(st.st, S, Z, tokens)

    def prefill(self, q, k, v, P, st):
        return _b.prefill(q, k, v, P=P, state=st)

    @staticmethod
    def tensors(st):
        return st.S, st.Z


def exclusive_prefix(impl, shapes, gathered, rank, tokens_per_rank, device):
    """State of all tokens before ``rank``'s segment: the sum, in rank order, of
    the gathered segment states of ranks 0 .. rank - 1."""
    B, H, d_K, d_V, P = shapes
    st = impl.zero_state(B, H, d_K, d_V, P, device)
    for r in range(rank):
        S, Z = gathered[r]
        impl.accumulate(st, S, Z, tokens_per_rank[r])
    return st


def prefill_sequence_split(q, k, v, P: int = 4, group=None, impl=None):
    """Causal prefill of a sequence split across the ranks of ``group``.

    q, k: [B, H, n_r, d_K], v: [B, H, n_r, d_V]: this rank's tokens (rank r holds
    the r-th segment; segments may differ in length).  Returns (y, state): the
    outputs for this rank's tokens and the state after them (on the last rank:
    the state of the whole sequence, ready for decode).
    """
    import torch.distributed as dist

    impl = impl or LibraryImpl()
    if dist.is_available() and dist.is_initialized():
        rank, world = dist.get_rank(group), dist.get_world_size(group)
    else:   # one rank: no exchange, the prefix is empty
        rank, world = 0, 1
    B, H, n, d_K = q.shape
    d_V = v.shape[-1]
    # 1. this segment's state from zero
    seg = impl.segment_state(q, k, v, P)
    S, Z = impl.tensors(seg)
    # 2. every rank's segment state and length
    if world > 1:
        n_all = [torch.zeros(1, dtype=torch.int64, device=S.device) for _ in range(world)]
        dist.all_gather(n_all, torch.tensor([n], dtype=torch.int64, device=S.device), group=group)
        S_all = [torch.empty_like(S) for _ in range(world)]
        Z_all = [torch.empty_like(Z) for _ in range(world)]
        dist.all_gather(S_all, S.contiguous(), group=group)
        dist.all_gather(Z_all, Z.contiguous(), group=group)
        lens = [int(x.item()) for x in n_all]
    else:
        S_all, Z_all, lens = [S], [Z], [n]
    # 3. the state before this segment
    st = exclusive_prefix(impl, (B, H, d_K, d_V, P), list(zip(S_all, Z_all)), rank, lens, q.device)
    # 4. this segment's outputs from that state
    y = impl.prefill(q, k, v, P, st)
    return y, st
