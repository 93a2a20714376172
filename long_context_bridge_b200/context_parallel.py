"""The block split over ranks, one process per GPU: decode with each
sequence's context split over ranks, and prefill with the prompt's rows split
over ranks.

Decode.
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

Prefill.  The prompt's T rows are cut into 2R equal chunks and rank r owns
chunks r and 2R-1-r, so every rank gets the same causal work.  Each rank
bridges the K/V of its own rows, the ranks all-gather them (one exchange of
T * n_kv_heads * 128 * 2 bf16 values), and each rank runs the block on its
chunks with hs2_block_prefill_rows, which computes every row exactly as the
single-device hs2_block_prefill does.
"""
from __future__ import annotations

import torch

from . import (DECODE_REC_FLOATS, OP_BLOCK_DECODE, OP_BLOCK_PREFILL, Shape, hs2_block_prefill_rows,
               hs2_bridge_kv, hs2_decode_cp_attn, hs2_decode_cp_finish, hs2_decode_cp_select,
               hs2_decode_cp_sparse, workspace_size)


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


def zigzag_chunks(T: int, n_ranks: int, rank: int, align: int = 128):
    """Rank `rank`'s two row ranges [begin, end) of a T-row prompt cut into
    2R equal chunks: chunk r and chunk 2R-1-r.  The chunk size must be a
    multiple of `align` (the kernels' row tile)."""
    n = 2 * n_ranks
    if T % n != 0 or (T // n) % align != 0:
        raise ValueError(f"T = {T} does not split into {n} chunks of a multiple of {align} rows")
    c = T // n
    return [(rank * c, (rank + 1) * c), ((n - 1 - rank) * c, (n - rank) * c)]


class PrefillRows:
    """One rank's part of a row-sharded prefill of a T-row prompt."""

    def __init__(self, shape: Shape, n_ranks: int, rank: int, device):
        self.shape, self.R, self.rank = shape, n_ranks, rank
        self.chunks = zigzag_chunks(shape.T, n_ranks, rank)
        c = self.chunks[0][1] - self.chunks[0][0]
        self.c = c
        self.chunk_shape = Shape.make(c, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                                      shape.scale, shape.k_global, shape.window)
        self.ws = torch.empty(workspace_size(OP_BLOCK_PREFILL, self.chunk_shape),
                              dtype=torch.uint8, device=device)

    def rows(self):
        """This rank's rows (positions) in the order of its row buffers."""
        return torch.cat([torch.arange(b, e) for b, e in self.chunks])

    def bridge(self, H_rows, W_k, W_v):
        """K/V of this rank's rows (H_rows [2c, d_model], its chunks in order)."""
        sh = self.shape
        K = torch.empty(H_rows.shape[0], sh.n_kv_heads, sh.head_dim, dtype=torch.bfloat16,
                        device=H_rows.device)
        V = torch.empty_like(K)
        hs2_bridge_kv(H_rows, W_k, W_v, K, V, Shape.make(H_rows.shape[0], sh.n_kv_heads,
                                                         sh.n_kv_heads))
        return K, V

    def assemble(self, gathered):
        """The whole prompt's [T, ...] tensor from the ranks' gathered row
        buffers [R, 2c, ...] (each rank's two chunks in order)."""
        c, R = self.c, self.R
        out = torch.empty((self.shape.T,) + tuple(gathered.shape[2:]), dtype=gathered.dtype,
                          device=gathered.device)
        for r in range(R):
            out[r * c:(r + 1) * c] = gathered[r, :c]
            out[(2 * R - 1 - r) * c:(2 * R - r) * c] = gathered[r, c:]
        return out

    def block(self, K, V, Q_rows, O_rows, lse_rows, idx_rows, Qs_rows, Os_rows, stream=None):
        """The block for this rank's rows, given the whole prompt's K/V."""
        c = self.c
        for i, (b, e) in enumerate(self.chunks):
            sl = slice(i * c, (i + 1) * c)
            hs2_block_prefill_rows(b, K[:e], V[:e], Q_rows[sl], O_rows[sl], lse_rows[sl],
                                   idx_rows[sl], [q[sl] for q in Qs_rows],
                                   [o[sl] for o in Os_rows], self.chunk_shape, self.ws, stream)

    def run(self, all_gather, H_rows, W_k, W_v, Q_rows, O_rows, lse_rows, idx_rows, Qs_rows,
            Os_rows, stream=None):
        K_own, V_own = self.bridge(H_rows, W_k, W_v)
        K = self.assemble(all_gather(K_own))
        V = self.assemble(all_gather(V_own))
        self.block(K, V, Q_rows, O_rows, lse_rows, idx_rows, Qs_rows, Os_rows, stream)
        return K, V
