"""GPU parity of the context split (one sequence's compressed cache over G
ranks), on one GPU: the G ranks' phases run one after another on shards of
one cache, and the exchanges are concatenations in rank order (no rank waits
on another).  Checked against the whole sequence:

  - every rank's scores equal the whole-sequence indexer's (same kernel);
  - the merged selection equals the oracle's top-k over the whole sequence's
    scores, bit for bit (ties across shards included);
  - the merged output and log-sum-exp equal the oracle's attention over the
    whole cache with that selection, within the attention tolerance.
"""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from compressed_sparse_kv_04_b200.context_split import ContextSplitStep
from gpuhelp import assert_attention_close, assert_lse_close, bits16, bits8, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def run_split(w, G, S, N, pos, tie_copy=False, seed=0):
    """Returns (per-rank outputs, selection, count, scores, inputs)."""
    L = N * w.m
    g = torch.Generator(device=DEV).manual_seed(500 + seed)
    kv_c = torch.randn(1, N, w.d, generator=g, device=DEV)
    kv_c = (kv_c / kv_c.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    kv_tok = torch.randn(1, L, w.d, generator=g, device=DEV).to(torch.bfloat16)
    key = synth.e4m3_codes((1, N, w.D_I), 501 + seed, "q_idx", DEV)
    ksc = synth.uniform_f32((1, N), 502 + seed, "q_scale", 0.005, 0.02, DEV)
    if tie_copy:  # shard 2 repeats shard 0's keys: equal scores at different indices
        n = N // G
        key[:, 2 * n: 3 * n] = key[:, :n]
        ksc[:, 2 * n: 3 * n] = ksc[:, :n]
    qi = synth.queries(configs.scaled(w, B=1, seed=503 + seed), Q=1, device=DEV)
    q = qi["q"][:, 0].contiguous()
    sink = qi["sink"]
    pos_t = torch.tensor([pos], dtype=torch.int64, device=DEV)
    n = N // G
    steps = []
    for r in range(G):
        p = binding.params_for(w, B=1, entry_offset=r * n)
        if r != G - 1:
            p.window = 0  # the window is attended by the last rank only
        steps.append(ContextSplitStep(p, n, G, S, DEV))
    shards = [(kv_c[:, r * n:(r + 1) * n].contiguous(), key[:, r * n:(r + 1) * n].contiguous(),
               ksc[:, r * n:(r + 1) * n].contiguous()) for r in range(G)]
    a = [st.phase_a(qi["q_idx"], qi["q_scale"], qi["w"], sh[1], sh[2], pos_t)
         for st, sh in zip(steps, shards)]
    g_s = torch.stack([x[0] for x in a])
    g_i = torch.stack([x[1] for x in a])
    g_c = torch.stack([x[2] for x in a])
    b = [st.phase_b(g_s, g_i, g_c, q, pos_t, sh[0], kv_tok) for st, sh in zip(steps, shards)]
    g_po = torch.cat([x[0] for x in b], 1)
    g_pm = torch.cat([x[1] for x in b], 1)
    outs, lses = [], []
    for st in steps:
        out = torch.empty(1, w.H, w.d, dtype=torch.bfloat16, device=DEV)
        lse = torch.empty(1, w.H, dtype=torch.float32, device=DEV)
        st.phase_c(g_po, g_pm, pos_t, sink, out, lse)
        outs.append(out)
        lses.append(lse)
    torch.cuda.synchronize()
    scores = torch.cat([st.scores for st in steps], -1)
    return dict(outs=outs, lses=lses, sel=steps[0].sel, cnt=steps[0].sel_cnt, scores=scores,
                kv_c=kv_c, kv_tok=kv_tok, key=key, ksc=ksc, qi=qi, q=q, sink=sink, steps=steps)


def check(orc, w, r, pos, N):
    nv = min((pos + 1) // w.m, N)
    # Scores: the whole-sequence indexer on the same inputs.
    p = binding.params_for(w, B=1)
    full = torch.empty(1, 1, N, dtype=torch.float32, device=DEV)
    binding.lightning_index_scores(p, 1, r["qi"]["q_idx"], r["qi"]["q_scale"], r["qi"]["w"], r["key"],
                                   r["ksc"], torch.tensor([[pos]], device=DEV), full)
    torch.cuda.synchronize()
    assert torch.equal(full[..., :nv], r["scores"][..., :nv])
    # Selection: the oracle's top-k over the whole sequence's scores.
    s = f32(full)[0, 0, :N].astype(np.float64)
    ridx, rcnt = orc.topk(s[None], np.array([nv]), w.k)
    assert int(r["cnt"][0]) == rcnt[0]
    assert np.array_equal(r["sel"].cpu().numpy()[0], ridx[0])
    # Every rank merged to the same output.
    for o in r["outs"][1:]:
        assert torch.equal(o, r["outs"][0])
    ref, rlse = orc.mqa(bits16(r["q"]).reshape(1, 1, w.H, w.d), np.array([[pos]]), bits16(r["kv_c"]),
                        bits16(r["kv_tok"]), f32(r["sink"]), w.m, w.W, w.rope_dim,
                        ridx[:, None], rcnt[:, None])
    got = r["outs"][0].double().cpu().numpy()
    assert np.isfinite(got).all()
    assert_attention_close(got, ref[:, 0], "context split")
    assert_lse_close(f32(r["lses"][0]), rlse[:, 0], ref[:, 0], "context split")


@pytest.mark.parametrize("G,S", [(4, 1), (4, 2), (2, 3), (8, 1)])
def test_context_split_matches_whole_sequence(orc, G, S):
    w = configs.scaled(configs.CSA_128K, k=256)
    N = 4096
    pos = N * w.m - 1
    r = run_split(w, G, S, N, pos, seed=G * 10 + S)
    check(orc, w, r, pos, N)


def test_context_split_ties_across_shards(orc):
    """Shard 2 holds the same keys as shard 0: equal scores at different
    sequence indices; the lower index must win, as on one device."""
    w = configs.scaled(configs.CSA_128K, k=256)
    N, G = 4096, 4
    pos = N * w.m - 1
    r = run_split(w, G, 1, N, pos, tie_copy=True, seed=7)
    check(orc, w, r, pos, N)


def test_context_split_partial_last_shard(orc):
    """The query sits inside the last shard (its later entries are not yet
    visible), and one shard has fewer visible entries than k."""
    w = configs.scaled(configs.CSA_128K, k=256)
    N, G = 4096, 4
    pos = (3 * 1024 + 100) * w.m + 2  # 3172 visible entries: shard 3 holds 100 of them
    r = run_split(w, G, 1, N, pos, seed=9)
    check(orc, w, r, pos, N)
