"""Decode with each sequence's context split over ranks (one process per GPU).

Host-side orchestration of the four hs2_decode_cp_* calls: every rank holds
a contiguous slice of each sequence's FP8 cache and runs the same four calls;
between them the ranks all-gather small records (a softmax state per query
head, then each rank's exact top k, then a softmax state per sparse layer and
query head).  No K/V row moves between ranks and no kernel reads another
GPU's memory.  The arithmetic runs in the library's kernels; this module only
allocates the record buffers and exchanges them.

``all_gather(t)`` must return the R ranks' tensors of t's shape stacked in
rank order along a new leading dimension; ``dist_all_gather(group)`` builds it
from torch.distributed.  A test on one device runs the steps of virtual
ranks in lockstep and stacks their records instead.
"""
from __future__ import annotations

import torch

from . import (DECODE_REC_FLOATS, OP_BLOCK_DECODE, Shape, hs2_decode_cp_attn,
               hs2_decode_cp_finish, hs2_decode_cp_select, hs2_decode_cp_sparse,
               workspace_size)


def slice_bounds(seq_len, n_ranks: int, rank: int):
    """Rank `rank`'s slice [lo, hi) of each sequence: contiguous, as equal as
    integer division makes them, tiling [0, seq_len[b]) in rank order."""
    lo = [(int(n) * rank) // n_ranks for n in seq_len]
    hi = [(int(n) * (rank + 1)) // n_ranks for n in seq_len]
    return lo, hi


def local_capacity(seq_len, n_ranks: int) -> int:
    """Cache rows per sequence that every rank's slice fits in."""
    return max(max(h - l for l, h in zip(*slice_bounds(seq_len, n_ranks, r)))
               for r in range(n_ranks))


def dist_all_gather(group=None):
    """all_gather over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for CPU ones): the ranks' tensors stacked in rank order."""
    import torch.distributed as dist

    def gather(t: torch.Tensor) -> torch.Tensor:
        world = dist.get_world_size(group)
        t = t.contiguous()
        out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        if t.is_cuda:
            dist.all_gather_into_tensor(out, t, group=group)
        else:
            dist.all_gather(list(out.unbind(0)), t, group=group)
        return out
    return gather


class DecodeCP:
    """One rank's part of a context-parallel decode step: the record buffers
    and the four steps (attn, select, sparse, finish) for a fixed batch, local
    cache capacity (shape.T) and shape."""

    def __init__(self, batch: int, shape: Shape, n_ranks: int, n_sparse: int, device):
        self.B, self.shape, self.R, self.L = batch, shape, n_ranks, n_sparse
        Hq, Hkv, k = shape.n_q_heads, shape.n_kv_heads, shape.k_global
        f32 = dict(dtype=torch.float32, device=device)
        self.attn_rec = torch.empty(batch, Hq, DECODE_REC_FLOATS, **f32)
        self.sel_rec = torch.empty(batch, Hkv, k, 2, dtype=torch.int32, device=device)
        self.sparse_rec = torch.empty(max(1, n_sparse), batch, Hq, DECODE_REC_FLOATS, **f32)
        self.ws = torch.empty(workspace_size(OP_BLOCK_DECODE, shape, batch), dtype=torch.uint8,
                              device=device)

    def attn(self, seq_len, lo, hi, q_full, Kc, Vc, k_scale, v_scale, stream=None):
        hs2_decode_cp_attn(seq_len, lo, hi, q_full, Kc, Vc, k_scale, v_scale, self.attn_rec,
                           self.shape, self.ws, stream)
        return self.attn_rec

    def select(self, seq_len, lo, hi, attn_recs, o_full, lse, stream=None):
        hs2_decode_cp_select(seq_len, lo, hi, self.R, attn_recs, o_full, lse, self.sel_rec,
                             self.shape, self.ws, stream)
        return self.sel_rec

    def sparse(self, seq_len, lo, hi, sel_recs, idx, Kc, Vc, k_scale, v_scale, q_sparse,
               stream=None):
        hs2_decode_cp_sparse(seq_len, lo, hi, self.R, sel_recs, idx, Kc, Vc, k_scale, v_scale,
                             q_sparse, self.sparse_rec if self.L else None, self.shape, stream)
        return self.sparse_rec[:self.L]

    def finish(self, sparse_recs, o_sparse, stream=None):
        hs2_decode_cp_finish(self.R, sparse_recs, o_sparse, self.shape, stream)

    def run(self, all_gather, seq_len, lo, hi, q_full, Kc, Vc, k_scale, v_scale, q_sparse,
            o_full, lse, idx, o_sparse, stream=None):
        """The four steps with the three exchanges; writes o_full, lse, idx and
        o_sparse (identical on every rank)."""
        attn_recs = all_gather(self.attn(seq_len, lo, hi, q_full, Kc, Vc, k_scale, v_scale,
                                         stream))
        sel_recs = all_gather(self.select(seq_len, lo, hi, attn_recs, o_full, lse, stream))
        recs = self.sparse(seq_len, lo, hi, sel_recs, idx, Kc, Vc, k_scale, v_scale, q_sparse,
                           stream)
        if self.L:
            self.finish(all_gather(recs), o_sparse, stream)
