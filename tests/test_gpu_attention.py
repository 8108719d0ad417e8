"""GPU parity: shared-KV MQA decode (sparse CSA and dense HCA) with window and
sink, through the C ABI, against the fp64 oracle.

Tolerance (bf16 storage, fp32 accumulation): max abs <= 2e-2 and relative L2
<= 5e-3 on the output.  The log-sum-exp is checked per head against the
bound gpuhelp.lse_tolerance derives from the bf16 rounding of the
normalised query (shared by every logit of the head) and of the keys."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from gpuhelp import assert_attention_close, assert_lse_close, bits16, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def out_values(t):
    return t.double().cpu().numpy()


def run_attention(w, q, pos, kv_c, kv_tok, sink, sel=None, cnt=None, gamma_q=None,
                  gamma_kv=None, expect_status=0):
    B = q.shape[0]
    p = binding.params_for(w, B=B)
    out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, w.H), float("nan"), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pos_t = torch.as_tensor(pos, dtype=torch.int64, device=DEV).reshape(B)
    if sel is not None:
        ws = binding.workspace(p, binding.OP_SPARSE_MQA, 1, kv_c.shape[1])
        binding.sparse_mqa_decode(p, q, pos_t, kv_c, sel, cnt, kv_tok, sink, out, gamma_q,
                                  gamma_kv, lse=lse, ws=ws, dev_status=status)
    else:
        ws = binding.workspace(p, binding.OP_DENSE_MQA, 1, kv_c.shape[1])
        binding.dense_mqa_decode(p, q, pos_t, kv_c, kv_tok, sink, out, gamma_q, gamma_kv,
                                 lse=lse, ws=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == expect_status, status.item()
    return out, lse


def oracle_attention(orc, w, q, pos, kv_c, kv_tok, sink, sel=None, cnt=None, gamma_q=None,
                     gamma_kv=None, tok_base=0):
    B = q.shape[0]
    o, l = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), np.asarray(pos).reshape(B, 1), bits16(kv_c),
                   bits16(kv_tok), f32(sink), w.m, w.W, w.rope_dim,
                   None if sel is None else sel.cpu().numpy().reshape(B, 1, -1),
                   None if cnt is None else cnt.cpu().numpy().reshape(B, 1),
                   None if gamma_q is None else f32(gamma_q),
                   None if gamma_kv is None else f32(gamma_kv), tok_base=tok_base)
    return o[:, 0], l[:, 0]


def check(orc, w, q, pos, kv_c, kv_tok, sink, sel=None, cnt=None, gamma_q=None, gamma_kv=None,
          what=""):
    out, lse = run_attention(w, q, pos, kv_c, kv_tok, sink, sel, cnt, gamma_q, gamma_kv)
    ref, rlse = oracle_attention(orc, w, q, pos, kv_c, kv_tok, sink, sel, cnt, gamma_q, gamma_kv)
    got = out_values(out)
    assert np.isfinite(got).all()
    mx, rl2 = assert_attention_close(got, ref, what)
    qg = 1.0 if gamma_q is None else max(1.0, float(gamma_q.abs().max()))
    assert_lse_close(f32(lse), rlse, ref, what, qnorm_gain=qg)
    return mx, rl2


def random_cache(w, B, N_cap, L_cap, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    kv_c = torch.randn(B, N_cap, w.D, generator=g, device=DEV).to(torch.bfloat16)
    # Stored entries are RMSNorm'd by compression: give them unit RMS.
    kv_c = (kv_c.float() / kv_c.float().pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    kv_tok = torch.randn(B, L_cap, w.D, generator=g, device=DEV).to(torch.bfloat16)
    return kv_c, kv_tok


def random_selection(B, k, n_vis, seed, cnt=None):
    rng = np.random.default_rng(seed)
    sel = np.full((B, k), -1, np.int32)
    cn = np.zeros(B, np.int32)
    for b in range(B):
        c = min(k, n_vis[b]) if cnt is None else cnt[b]
        sel[b, :c] = np.sort(rng.choice(n_vis[b], c, replace=False))
        cn[b] = c
    return torch.from_numpy(sel).to(DEV), torch.from_numpy(cn).to(DEV)


def test_sparse_tiny_end_to_end(orc):
    """C1: compress -> indexer -> top-k -> sparse MQA, checked step-chained."""
    w = configs.TINY_CSA
    kv_tok, idx_tok = synth.token_streams(w, device=DEV)
    w_s, b_pos = synth.pool_params(w, DEV)
    w_si, b_pi = synth.pool_params(w, DEV, indexer=True)
    qi = synth.queries(w, Q=1, device=DEV)
    ctx = torch.full((w.B,), w.L, dtype=torch.int64, device=DEV)
    kv_c = torch.zeros(w.B, w.N_c, w.d, dtype=torch.bfloat16, device=DEV)
    key = torch.zeros(w.B, w.N_c, w.D_I, dtype=torch.uint8, device=DEV)
    ksc = torch.zeros(w.B, w.N_c, dtype=torch.float32, device=DEV)
    p = binding.params_for(w)
    binding.csa_compress(p, kv_tok, ctx, w_s, b_pos, None, 0, w.N_c, kv_c, idx_tok, w_si, b_pi,
                         key, ksc)
    tidx = torch.empty(w.B, 1, w.k, dtype=torch.int32, device=DEV)
    tcnt = torch.empty(w.B, 1, dtype=torch.int32, device=DEV)
    ws = binding.workspace(p, binding.OP_INDEX_TOPK, 1, w.N_c)
    binding.lightning_index_topk(p, 1, qi["q_idx"], qi["q_scale"], qi["w"], key, ksc,
                                 (ctx - 1).view(w.B, 1), tidx, tcnt, ws=ws)
    q = qi["q"][:, 0].contiguous()
    check(orc, w, q, [w.L - 1], kv_c, kv_tok, qi["sink"], tidx.view(w.B, w.k), tcnt.view(w.B),
          what="tiny CSA")


@pytest.mark.parametrize("pos", [0, 3, 100, 127, 128, 1000])
def test_sparse_small_d512_ragged(orc, pos):
    w = configs.scaled(configs.CSA_128K, B=2, k=100)
    B, N_cap, L_cap = 2, 300, 1200
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 5 + pos)
    q = synth.normal_bf16((B, w.H, w.D), 7 + pos, "q", DEV)
    sink = synth.normal_f32((w.H,), 7, "sink", 1.0, DEV)
    n_vis = [min((pos + 1) // w.m, N_cap)] * B
    sel, cnt = random_selection(B, w.k, n_vis, pos)
    check(orc, w, q, [pos, pos], kv_c, kv_tok, sink, sel, cnt, what=f"pos {pos}")


def test_sparse_with_gains_and_partial_heads(orc):
    w = configs.scaled(configs.CSA_128K, B=3, k=130, H=100)
    B, N_cap, L_cap = 3, 700, 2900
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 11)
    q = synth.normal_bf16((B, w.H, w.D), 12, "q", DEV)
    sink = synth.normal_f32((w.H,), 13, "sink", 1.0, DEV)
    gq = synth.gains(w.D, 14, DEV)
    gk = synth.gains(w.D, 15, DEV)
    pos = [2799, 1500, 640]
    n_vis = [min((x + 1) // w.m, N_cap) for x in pos]
    sel, cnt = random_selection(B, w.k, n_vis, 16, cnt=[130, 77, 1])
    check(orc, w, q, pos, kv_c, kv_tok, sink, sel, cnt, gq, gk, what="gains")


def test_sink_limits(orc):
    w = configs.scaled(configs.CSA_128K, B=1, k=64)
    kv_c, kv_tok = random_cache(w, 1, 100, 400, 17)
    q = synth.normal_bf16((1, w.H, w.D), 18, "q", DEV)
    sel, cnt = random_selection(1, w.k, [99], 19)
    sink = torch.full((w.H,), float("-inf"), device=DEV)
    sink[::3] = float("inf")
    out, lse = run_attention(w, q, [399], kv_c, kv_tok, sink, sel, cnt)
    ref, rlse = oracle_attention(orc, w, q, [399], kv_c, kv_tok, sink, sel, cnt)
    got = out_values(out)
    assert (got[0, ::3] == 0).all() and np.isposinf(f32(lse)[0, ::3]).all()
    assert_attention_close(got, ref, "sink limits")


def test_sparse_bad_index_reported_and_skipped(orc):
    w = configs.scaled(configs.CSA_128K, B=1, k=64)
    kv_c, kv_tok = random_cache(w, 1, 100, 400, 21)
    q = synth.normal_bf16((1, w.H, w.D), 22, "q", DEV)
    sink = synth.normal_f32((w.H,), 23, "sink", 1.0, DEV)
    sel, cnt = random_selection(1, w.k, [99], 24)
    sel[0, 5] = 100  # == n_vis (and == N_cap): not visible
    sel[0, 9] = -1
    out, _ = run_attention(w, q, [399], kv_c, kv_tok, sink, sel, cnt, expect_status=7)
    ref, _ = oracle_attention(orc, w, q, [399], kv_c, kv_tok, sink, sel, cnt)
    assert_attention_close(out_values(out), ref, "bad index")


@pytest.mark.parametrize("L", [128 * 20, 128 * 20 + 5, 127, 128 * 3 + 64])
def test_dense_hca_small(orc, L):
    w = configs.scaled(configs.HCA_1M, B=2)
    N_cap = math.ceil(L / w.m) + 2
    kv_c, kv_tok = random_cache(w, 2, N_cap, L + 3, 30 + L)
    q = synth.normal_bf16((2, w.H, w.D), 31, "q", DEV)
    sink = synth.normal_f32((w.H,), 32, "sink", 1.0, DEV)
    gq = synth.gains(w.D, 33, DEV)
    check(orc, w, q, [L - 1, max(0, L - 100)], kv_c, kv_tok, sink, gamma_q=gq, what=f"dense L={L}")


def test_sparse_csa_128k_shape(orc):
    w = configs.CSA_128K
    kv_c, kv_tok = random_cache(w, w.B, w.N_c, w.L, 40)
    q = synth.normal_bf16((w.B, w.H, w.D), 41, "q", DEV)
    sink = synth.normal_f32((w.H,), 42, "sink", 1.0, DEV)
    sel, cnt = random_selection(w.B, w.k, [w.N_c] * w.B, 43)
    check(orc, w, q, [w.L - 1] * w.B, kv_c, kv_tok, sink, sel, cnt, what="CSA 128K")


def test_dense_hca_1m_shape(orc):
    """C3 at full size: 8 x 8192 entries + 128-token window at position 2^20 - 1.

    Only the window tail of the 1M-token stream is materialised for the
    oracle (rows L-128 .. L-1); the kernel reads the full-size device stream."""
    w = configs.HCA_1M
    g = torch.Generator(device=DEV).manual_seed(50)
    kv_c = torch.randn(w.B, w.N_c, w.D, generator=g, device=DEV)
    kv_c = (kv_c / kv_c.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    tail = torch.randn(w.B, w.W, w.D, generator=g, device=DEV).to(torch.bfloat16)
    kv_tok = torch.empty(w.B, w.L, w.D, dtype=torch.bfloat16, device=DEV)
    kv_tok[:, -w.W:] = tail
    q = synth.normal_bf16((w.B, w.H, w.D), 51, "q", DEV)
    sink = synth.normal_f32((w.H,), 52, "sink", 1.0, DEV)
    out, lse = run_attention(w, q, [w.L - 1] * w.B, kv_c, kv_tok, sink)
    del kv_tok
    ref, rlse = oracle_attention(orc, w, q, [w.L - 1] * w.B, kv_c, tail, sink, tok_base=w.L - w.W)
    mx, rl2 = assert_attention_close(out_values(out), ref, "HCA 1M")
    assert_lse_close(f32(lse), rlse, ref, "HCA 1M")


@pytest.mark.parametrize("dense", [False, True])
def test_garbage_workspace_and_unwritten_cache_rows(orc, dense):
    """Workspace bytes and cache rows the method never reads may hold any
    bits (here NaN): empty splits, masked rows of a partial tile and unused
    selection slots must not leak into the output."""
    w = configs.scaled(configs.CSA_128K, B=2, k=100)
    B, N_cap, L_cap = 2, 300, 1200
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 77)
    q = synth.normal_bf16((B, w.H, w.D), 78, "q", DEV)
    sink = synth.normal_f32((w.H,), 79, "sink", 1.0, DEV)
    pos = [5, 190]  # 1 and 47 visible entries: mostly masked tiles
    n_vis = [(x + 1) // w.m for x in pos]
    for b in range(B):
        kv_c[b, n_vis[b]:] = float("nan")
    p = binding.params_for(w, B=B)
    op = binding.OP_DENSE_MQA if dense else binding.OP_SPARSE_MQA
    ws = binding.workspace(p, op, 1, N_cap)
    ws.fill_(0xFF)
    out = torch.empty(B, w.H, w.D, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pos_t = torch.tensor(pos, dtype=torch.int64, device=DEV)
    if dense:
        binding.dense_mqa_decode(p, q, pos_t, kv_c, kv_tok, sink, out, ws=ws, dev_status=status)
        sel = cnt = None
    else:
        sel, cnt = random_selection(B, w.k, n_vis, 80)
        binding.sparse_mqa_decode(p, q, pos_t, kv_c, sel, cnt, kv_tok, sink, out, ws=ws,
                                  dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    got = out_values(out)
    assert np.isfinite(got).all()
    ref, _ = oracle_attention(orc, w, q, pos, kv_c, kv_tok, sink, sel, cnt)
    assert_attention_close(got, ref, "garbage workspace")


@pytest.mark.parametrize("dense", [False, True])
def test_one_split_rows_finish_in_the_attention_kernel(orc, dense):
    """80 sequences give one split per row, so the attention kernel itself
    folds in the sink, normalises, inverse-rotates and writes bf16 (no merge
    launch).  Sinks include +inf and -inf; some rows see no complete block."""
    w = configs.scaled(configs.CSA_128K, B=80, k=64)
    B, N_cap, L_cap = 80, 200, 800
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 90 + dense)
    q = synth.normal_bf16((B, w.H, w.D), 91, "q", DEV)
    sink = synth.normal_f32((w.H,), 92, "sink", 1.0, DEV)
    sink[3], sink[5] = float("inf"), float("-inf")
    rng = np.random.default_rng(93)
    pos = rng.integers(0, L_cap, B)
    pos[:3] = [0, 2, L_cap - 1]
    n_vis = [min((int(t) + 1) // w.m, N_cap) for t in pos]
    sel, cnt = (None, None) if dense else random_selection(B, w.k, n_vis, 94)
    check(orc, w, q, pos.tolist(), kv_c, kv_tok, sink, sel, cnt, what=f"one split, dense={dense}")


def test_one_split_rows_with_nothing_to_attend(orc):
    """No window and positions before the first complete block: an empty KV
    set, a zero output, and the sink's own log-sum-exp (one split per row)."""
    w = configs.scaled(configs.HCA_1M, B=80, W=0)
    B, N_cap, L_cap = 80, 8, 1024
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 95)
    q = synth.normal_bf16((B, w.H, w.D), 96, "q", DEV)
    sink = synth.normal_f32((w.H,), 97, "sink", 1.0, DEV)
    sink[7], sink[9] = float("inf"), float("-inf")
    pos = [t % 128 if t % 3 else 128 * (1 + t % 7) + 5 for t in range(B)]
    check(orc, w, q, pos, kv_c, kv_tok, sink, what="one split, empty KV sets")


def test_sparse_csa_1m_shape(orc):
    """C4 at full size: 4 sequences x 262144 compressed entries (indices up to
    2^18 - 1), 1024 selected per sequence, the 128-token window at position
    2^20 - 1.  Only the window tail of the 1M-token stream is materialised for
    the oracle; the kernel reads the full-size device stream."""
    w = configs.CSA_1M
    g = torch.Generator(device=DEV).manual_seed(60)
    kv_c = torch.randn(w.B, w.N_c, w.D, generator=g, device=DEV)
    kv_c = (kv_c / kv_c.pow(2).mean(-1, keepdim=True).sqrt()).to(torch.bfloat16)
    tail = torch.randn(w.B, w.W, w.D, generator=g, device=DEV).to(torch.bfloat16)
    kv_tok = torch.empty(w.B, w.L, w.D, dtype=torch.bfloat16, device=DEV)
    kv_tok[:, -w.W:] = tail
    q = synth.normal_bf16((w.B, w.H, w.D), 61, "q", DEV)
    sink = synth.normal_f32((w.H,), 62, "sink", 1.0, DEV)
    sel, cnt = random_selection(w.B, w.k, [w.N_c] * w.B, 63)
    assert int(sel.max()) >= 1 << 17
    out, lse = run_attention(w, q, [w.L - 1] * w.B, kv_c, kv_tok, sink, sel, cnt)
    del kv_tok
    ref, rlse = oracle_attention(orc, w, q, [w.L - 1] * w.B, kv_c, tail, sink, sel, cnt,
                                 tok_base=w.L - w.W)
    assert_attention_close(out_values(out), ref, "CSA 1M")
    assert_lse_close(f32(lse), rlse, ref, "CSA 1M")


@pytest.mark.parametrize("cnt", [2048, 1500])
def test_sparse_top_2048(orc, cnt):
    """k = 2048 selected entries (the largest supported), full and partial."""
    w = configs.scaled(configs.CSA_128K, B=2, k=2048)
    B, N_cap, L_cap = 2, 4096, 4 * 4096
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 70 + cnt)
    q = synth.normal_bf16((B, w.H, w.D), 71, "q", DEV)
    sink = synth.normal_f32((w.H,), 72, "sink", 1.0, DEV)
    sel, c = random_selection(B, w.k, [N_cap] * B, 73, cnt=[cnt, cnt - 77])
    check(orc, w, q, [L_cap - 1] * B, kv_c, kv_tok, sink, sel, c, what=f"k=2048 cnt={cnt}")
