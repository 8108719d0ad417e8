"""Decode step of one CSA sequence whose compressed cache is split over the
ranks of a process group (one rank per GPU).

Rank r holds the entries [lo_r, hi_r) of the compressed KV cache and of the
indexer keys (contiguous, in rank order); the token stream and the query are
available on every rank, and the window is attended by one rank.  A step
runs in three phases with one exchange after each of the first two (the
pages give no parallel scheme for this path; this is the library's, see
include/csa.h "Context split"):

  A  indexer + local top-k on the shard, then the shard's candidates
     (score, sequence index)                      -> all-gather candidates
  B  global top-k over all candidates and this rank's share of it, then the
     attention partials over that share           -> all-gather partials
  C  merge of every rank's partials with the sink: the output (the same on
     every rank)

Every computation runs in libcsa.so kernels; this module only sequences the
calls, holds the buffers and performs the exchanges (torch.distributed
all-gathers, NCCL on GPUs).  `ops` replaces the library calls (a test passes
CPU implementations to exercise the exchange logic with gloo ranks).
"""
from __future__ import annotations

import torch


class LibraryOps:
    """The library's calls (CUDA)."""

    def __init__(self):
        from . import binding
        self.b = binding

    def index_topk(self, p, q_idx, q_scale, w, key, ksc, pos2, tidx, tcnt, scores):
        self.b.lightning_index_topk(p, 1, q_idx, q_scale, w, key, ksc, pos2, tidx, tcnt,
                                    scores_out=scores)

    def candidates(self, p, scores, tidx, tcnt, cand_s, cand_i):
        self.b.csa_shard_candidates(p, 1, scores, tidx, tcnt, cand_s, cand_i)

    def merge_candidates(self, p, G, cand_s, cand_i, cand_c, N_cap, tidx, tcnt, lidx, lcnt):
        self.b.csa_merge_candidates(p, 1, G, cand_s, cand_i, cand_c, N_cap, tidx, tcnt, lidx, lcnt)

    def partials(self, p, S, q, pos, kv_c, lidx, lcnt, kv_tok, part_o, part_ml):
        self.b.sparse_mqa_partials(p, S, q, pos, kv_c, lidx, lcnt, kv_tok, part_o, part_ml)

    def merge_partials(self, p, S, part_o, part_ml, pos, sink, out, lse):
        self.b.mqa_merge_partials(p, S, part_o, part_ml, pos, sink, out, lse)


class ContextSplitStep:
    """Buffers and phases of one rank.

    p_shard: csa_params of this rank (B = 1, entry_offset = lo, and window =
    the layer's window on the window rank, 0 on the others); N_shard: its
    cache capacity; G: ranks; S: attention splits per rank."""

    def __init__(self, p_shard, N_shard, G, S, device, ops=None):
        self.p, self.N, self.G, self.S = p_shard, N_shard, G, S
        self.ops = ops or LibraryOps()
        k, H, d = p_shard.k, p_shard.H, p_shard.d
        f32, i32 = torch.float32, torch.int32
        e = dict(device=device)
        self.scores = torch.empty(1, 1, N_shard, dtype=f32, **e)
        self.tidx = torch.empty(1, 1, k, dtype=i32, **e)
        self.tcnt = torch.empty(1, 1, dtype=i32, **e)
        self.cand_s = torch.empty(1, 1, k, dtype=f32, **e)
        self.cand_i = torch.empty(1, 1, k, dtype=i32, **e)
        self.sel = torch.empty(1, k, dtype=i32, **e)       # global selection
        self.sel_cnt = torch.empty(1, dtype=i32, **e)
        self.lidx = torch.empty(1, k, dtype=i32, **e)      # this rank's share (local)
        self.lcnt = torch.empty(1, dtype=i32, **e)
        self.part_o = torch.empty(1, S, H, d, dtype=torch.float16, **e)
        self.part_ml = torch.empty(1, S, 2, H, dtype=f32, **e)

    # -- phase A: local candidates ------------------------------------------
    def phase_a(self, q_idx, q_scale, w, key, ksc, pos):
        """Indexer and top-k on the shard; returns the tensors to all-gather:
        (candidate scores [1,1,k], sequence indices [1,1,k], count [1,1])."""
        self.ops.index_topk(self.p, q_idx, q_scale, w, key, ksc, pos.view(1, 1), self.tidx,
                            self.tcnt, self.scores)
        self.ops.candidates(self.p, self.scores, self.tidx, self.tcnt, self.cand_s, self.cand_i)
        return self.cand_s, self.cand_i, self.tcnt

    # -- phase B: global selection, attention partials -----------------------
    def phase_b(self, g_cand_s, g_cand_i, g_cnt, q, pos, kv_c, kv_tok):
        """g_*: the all-gathered phase-A tensors [G, ...] in rank order.
        Returns the tensors to all-gather: (partials [1,S,H,d] fp16, max/sum
        [1,S,2,H])."""
        self.ops.merge_candidates(self.p, self.G, g_cand_s, g_cand_i, g_cnt, self.N, self.sel,
                                  self.sel_cnt, self.lidx, self.lcnt)
        self.ops.partials(self.p, self.S, q, pos, kv_c, self.lidx, self.lcnt, kv_tok, self.part_o,
                          self.part_ml)
        return self.part_o, self.part_ml

    # -- phase C: merge -------------------------------------------------------
    def phase_c(self, g_part_o, g_part_ml, pos, sink, out, lse=None):
        """g_*: the all-gathered partials [G*S, ...] in rank order (as
        [1, G*S, ...]).  Writes out [1, H, d] (and lse [1, H])."""
        self.ops.merge_partials(self.p, self.G * self.S, g_part_o, g_part_ml, pos, sink, out, lse)


def all_gather_cat(t, group=None):
    """All-gather of a tensor from every rank, stacked in rank order along a
    new leading dim (torch.distributed; NCCL for CUDA tensors)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    return out.view((world,) + tuple(t.shape))


def decode_step(step: ContextSplitStep, q, q_idx, q_scale, w, pos, key, ksc, kv_c, kv_tok, sink,
                out, lse=None, group=None, gather=all_gather_cat):
    """One decode step on this rank (every rank of the group calls it with
    its own shard; all take the same collective steps in the same order)."""
    cs, ci, cc = step.phase_a(q_idx, q_scale, w, key, ksc, pos)
    g_s, g_i, g_c = gather(cs, group), gather(ci, group), gather(cc, group)
    po, pm = step.phase_b(g_s, g_i, g_c, q, pos, kv_c, kv_tok)
    g_po, g_pm = gather(po, group), gather(pm, group)
    # [G, 1, S, ...] -> [1, G*S, ...] (B = 1: rank-major is split-major)
    G, S = step.G, step.S
    step.phase_c(g_po.reshape((1, G * S) + tuple(po.shape[2:])),
                 g_pm.reshape((1, G * S) + tuple(pm.shape[2:])), pos, sink, out, lse)
    return step.sel, step.sel_cnt
