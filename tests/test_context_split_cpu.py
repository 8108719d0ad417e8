"""The context split's exchange logic on CPU: two gloo ranks on 127.0.0.1.

Each rank holds half of one sequence's compressed cache and runs the same
decode_step driver as on GPUs (phase A, all-gather of candidates, phase B,
all-gather of partials, phase C) with the library's calls replaced by CPU
stand-ins built from the fp64 oracle (test infrastructure).  The stand-ins
keep the library's buffer formats where the exchange depends on them:
candidates as (score, sequence index) with NaN/-1 padding, partials as one
(output, log2-domain max, sum) per split.  The two-rank result must equal the
oracle on the whole sequence: the same selection (ties across the shards
resolved to the lower index) and the same output."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.4426950408889634

# Sizes: H heads of D, N entries (m = 4), k kept, window W, indexer 4 x 16.
H, D, N, M, K, W, HI, DI, R = 4, 32, 48, 4, 8, 6, 4, 16, 8


def _inputs():
    rng = np.random.default_rng(11)
    import sys
    sys.path.insert(0, ROOT)
    from oracle import oracle as orc

    def bf16(x):
        return orc.bf16_encode(np.asarray(x, np.float64))

    L = N * M
    kv_c = bf16(rng.standard_normal((1, N, D)))
    kv_tok = bf16(rng.standard_normal((1, L, D)))
    key = torch.from_numpy((rng.standard_normal((1, N, DI)) * 64).clip(-448, 448).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    key[:, N // 2 + 3] = key[:, 3]          # a tie across the two shards
    ksc = rng.uniform(0.005, 0.02, (1, N)).astype(np.float32)
    ksc[:, N // 2 + 3] = ksc[:, 3]
    q_idx = torch.from_numpy((rng.standard_normal((1, 1, HI, DI)) * 64).clip(-448, 448).astype(
        np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    q_scale = rng.uniform(0.005, 0.02, (1, 1, HI)).astype(np.float32)
    w = rng.uniform(0, 1, (1, 1, HI)).astype(np.float32)
    q = bf16(rng.standard_normal((1, H, D)))
    sink = rng.standard_normal(H).astype(np.float32)
    return dict(kv_c=kv_c, kv_tok=kv_tok, key=key, ksc=ksc, q_idx=q_idx, q_scale=q_scale, w=w, q=q,
                sink=sink, pos=L - 1)


class _P:
    """The few csa_params fields the CPU stand-ins read."""

    def __init__(self, entry_offset, window):
        self.k, self.H, self.d, self.m = K, H, D, M
        self.entry_offset, self.window = entry_offset, window


class CpuOps:
    """CPU stand-ins for the library calls (oracle arithmetic)."""

    def __init__(self, orc, inp):
        self.orc, self.inp = orc, inp

    def index_topk(self, p, q_idx, q_scale, w, key, ksc, pos2, tidx, tcnt, scores):
        orc = self.orc
        n = key.shape[1]
        pos = int(pos2.reshape(-1)[0])
        nv = min(max((pos + 1) // M - p.entry_offset, 0), n)
        # The oracle's scores of the shard (its own visibility rule, on a
        # position that shows the whole shard), masked to the visible count.
        s = orc.index_scores(q_idx.numpy(), q_scale.numpy(), w.numpy(), key.numpy(), ksc.numpy(),
                             np.array([[n * M - 1]]), M)
        s[..., nv:] = -np.inf
        idx, cnt = orc.topk(s, np.array([[nv]]), p.k)
        scores.copy_(torch.from_numpy(s.astype(np.float32)))
        tidx.copy_(torch.from_numpy(idx))
        tcnt.copy_(torch.from_numpy(cnt))

    def candidates(self, p, scores, tidx, tcnt, cand_s, cand_i):
        c = int(tcnt.reshape(-1)[0])
        idx = tidx.reshape(-1).numpy()
        cand_s.fill_(float("nan"))
        cand_i.fill_(-1)
        for j in range(c):
            cand_s.view(-1)[j] = scores.view(-1)[int(idx[j])]
            cand_i.view(-1)[j] = int(idx[j]) + p.entry_offset

    def merge_candidates(self, p, G, cand_s, cand_i, cand_c, N_cap, tidx, tcnt, lidx, lcnt):
        s = [cand_s[r].reshape(-1)[: int(cand_c[r].reshape(-1)[0])] for r in range(G)]
        gi = [cand_i[r].reshape(-1)[: int(cand_c[r].reshape(-1)[0])] for r in range(G)]
        s = torch.cat(s).numpy().astype(np.float64)
        gi = torch.cat(gi).numpy()
        idx, cnt = self.orc.topk(s[None], np.array([len(s)]), p.k)
        sel = gi[idx[0, : cnt[0]]]
        tidx.fill_(-1)
        tidx.view(-1)[: len(sel)] = torch.from_numpy(sel.astype(np.int32))
        tcnt.fill_(int(cnt[0]))
        mine = sel[(sel >= p.entry_offset) & (sel < p.entry_offset + N_cap)] - p.entry_offset
        lidx.fill_(-1)
        lidx.view(-1)[: len(mine)] = torch.from_numpy(mine.astype(np.int32))
        lcnt.fill_(len(mine))

    def partials(self, p, S, q, pos, kv_c, lidx, lcnt, kv_tok, part_o, part_ml):
        assert S == 1
        c = int(lcnt.reshape(-1)[0])
        pos_i = int(pos.reshape(-1)[0])
        # This rank's KV set alone (no sink): the oracle's output and lse over
        # the whole cache with this rank's share as sequence indices (the
        # entries are stored rotated to their sequence positions).
        no_sink = np.full(H, -np.inf, np.float32)
        sel = lidx.numpy().reshape(1, 1, -1).astype(np.int32).copy()
        sel[0, 0, :c] += p.entry_offset
        o, lse = self.orc.mqa(q.numpy().reshape(1, 1, H, D), np.array([[pos_i]]),
                              self.inp["kv_c"], self.inp["kv_tok"], no_sink, M, p.window, R,
                              sel, np.array([[c]], np.int32))
        # (stored output, log2-domain max, sum) with the output's own scale.
        part_o[0, 0] = torch.from_numpy(np.nan_to_num(o[0, 0]).astype(np.float16))
        m2 = np.where(np.isfinite(lse[0, 0]), lse[0, 0] * LOG2E, -np.inf)
        part_ml[0, 0, 0] = torch.from_numpy(m2.astype(np.float32))
        part_ml[0, 0, 1] = torch.from_numpy(np.isfinite(m2).astype(np.float32))

    def merge_partials(self, p, S, part_o, part_ml, pos, sink, out, lse):
        m = part_ml[0, :, 0].numpy().astype(np.float64)       # [S, H]
        l = part_ml[0, :, 1].numpy().astype(np.float64)
        z2 = sink.numpy().astype(np.float64) * LOG2E
        Mx = np.maximum(m.max(0), z2)
        wgt = np.where(np.isfinite(m), l * np.exp2(m - Mx), 0.0)
        L = wgt.sum(0) + np.exp2(z2 - Mx)
        o = (wgt[:, :, None] * part_o[0].numpy().astype(np.float64)).sum(0) / L[:, None]
        out.copy_(torch.from_numpy(o[None].astype(np.float32)))
        lse.copy_(torch.from_numpy(((Mx + np.log2(L)) / LOG2E)[None].astype(np.float32)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from compressed_sparse_kv_04_b200 import context_split as cs
    from oracle import oracle as orc

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs()
        n = N // world
        lo = rank * n
        p = _P(lo, W if rank == world - 1 else 0)
        step = cs.ContextSplitStep(p, n, world, 1, torch.device("cpu"), ops=CpuOps(orc, inp))
        # Tokens are indexed by sequence position on every rank; the shard
        # holds entries lo .. lo+n-1.  The CPU stand-ins address the token
        # rows through the oracle's tok_base, so hand them the whole stream.
        t = torch.from_numpy
        out = torch.empty(1, H, D)
        lse = torch.empty(1, H)
        pos = torch.tensor([inp["pos"]])
        sel, cnt = cs.decode_step(step, t(inp["q"].astype(np.int32)), t(inp["q_idx"]),
                                  t(inp["q_scale"]), t(inp["w"]), pos,
                                  t(inp["key"][:, lo:lo + n].copy()), t(inp["ksc"][:, lo:lo + n].copy()),
                                  t(inp["kv_c"][:, lo:lo + n].astype(np.int32)),
                                  t(inp["kv_tok"].astype(np.int32)), t(inp["sink"]), out, lse)
        q.put((rank, sel.numpy().copy(), int(cnt[0]), out.numpy().copy(), lse.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_context_split_two_gloo_ranks_equal_whole_sequence(orc):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=150) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    inp = _inputs()
    # Whole sequence, one rank: scores, top-k, attention with window and sink.
    s = orc.index_scores(inp["q_idx"], inp["q_scale"], inp["w"], inp["key"], inp["ksc"],
                         np.array([[inp["pos"]]]), M)
    ridx, rcnt = orc.topk(s, np.array([[N]]), K)
    assert 3 in ridx[0, 0] or N // 2 + 3 not in ridx[0, 0]  # the tie goes to the lower index
    ref, rlse = orc.mqa(inp["q"].reshape(1, 1, H, D), np.array([[inp["pos"]]]), inp["kv_c"],
                        inp["kv_tok"], inp["sink"], M, W, R, ridx, rcnt)
    for rank, sel, cnt, out, lse in res:
        assert cnt == rcnt[0, 0]
        assert np.array_equal(sel[0], ridx[0, 0]), rank
        assert np.allclose(out[0], ref[0, 0], rtol=0, atol=2e-3), np.abs(out[0] - ref[0, 0]).max()
        assert np.allclose(lse[0], rlse[0, 0], rtol=0, atol=1e-5)
