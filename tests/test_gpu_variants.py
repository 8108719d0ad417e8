"""GPU parity of the V4-Flash attention shapes ("DeepSeek V4-Pro" (llm-arch-kb),
"Family": 64 query heads, top-k 512) with the YaRN RoPE frequencies of
"5. 1M context, gradually" (factor 16, beta_fast 32, beta_slow 1), through
the C ABI, against the fp64 oracle with its own YaRN table and logit gain.

The library's table comes from csa_rope_yarn (binding.params_for applies it
for a workload with YaRN settings); the oracle's from oracle.yarn_inv_freq.
With 64 heads every (query row, split) of the attention is one CTA."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from gpuhelp import assert_attention_close, assert_bf16_storage_close, assert_lse_close, bits16, f32
from test_gpu_attention import random_cache
from test_gpu_compress_index import check_index

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def oracle_rope(orc, w):
    return (orc.yarn_inv_freq(w.rope_dim, *w.yarn),
            orc.yarn_logit_gain(w.yarn[0]) / math.sqrt(w.d))


def check_lse(lse, rlse, ref, scale):
    assert_lse_close(f32(lse), rlse, ref, "LSE", scale)


@pytest.mark.parametrize("L", [8192, 4 * 600 + 4])
def test_flash_yarn_decode_step_chained(orc, L):
    """Compression (entries stored with the YaRN rotation) -> indexer ->
    top-512 -> sparse MQA over 64 heads with the YaRN logit gain."""
    w = configs.scaled(configs.CSA_FLASH_128K, B=2, L=L)
    B, N = w.B, w.N_c
    freq, scale = oracle_rope(orc, w)
    p = binding.params_for(w)
    kv_tok, idx_tok = synth.token_streams(w, device=DEV)
    w_s, b_pos = synth.pool_params(w, DEV)
    w_si, b_pi = synth.pool_params(w, DEV, indexer=True)
    ctx = torch.full((B,), L, dtype=torch.int64, device=DEV)
    kv_c = torch.zeros(B, N, w.d, dtype=torch.bfloat16, device=DEV)
    key = torch.zeros(B, N, w.D_I, dtype=torch.uint8, device=DEV)
    ksc = torch.zeros(B, N, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    binding.csa_compress(p, kv_tok, ctx, w_s, b_pos, None, 0, N, kv_c, idx_tok, w_si, b_pi, key,
                         ksc, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    # 1. Entries against the oracle's compression with its YaRN table.
    _, _, vals = orc.compress_kv(bits16(kv_tok), [L] * B, f32(w_s), f32(b_pos), None, w.m, 0, N,
                                 N, rope_dim=w.rope_dim, rope_freq=freq)
    assert_bf16_storage_close(bits16(kv_c), vals, "YaRN-rotated entries")
    # 2. Indexer scores and top-512, the latter bit-exact on the GPU's scores.
    qi = synth.queries(w, Q=1, device=DEV)
    pos_t = torch.full((B, 1), L - 1, dtype=torch.int64, device=DEV)
    tidx = torch.full((B, 1, w.k), -7, dtype=torch.int32, device=DEV)
    tcnt = torch.full((B, 1), -7, dtype=torch.int32, device=DEV)
    scores = torch.full((B, 1, N), float("nan"), dtype=torch.float32, device=DEV)
    binding.lightning_index_topk(p, 1, qi["q_idx"], qi["q_scale"], qi["w"], key, ksc, pos_t,
                                 tidx, tcnt, scores_out=scores, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    check_index(orc, w, qi, pos_t, key, ksc, scores, tidx, tcnt, w.k)
    # 3. Attention with the GPU's selection and entries.
    q = qi["q"][:, 0].contiguous()
    out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, w.H), float("nan"), dtype=torch.float32, device=DEV)
    ws = binding.workspace(p, binding.OP_SPARSE_MQA, 1, N)
    binding.sparse_mqa_decode(p, q, pos_t.view(B), kv_c, tidx.view(B, w.k), tcnt.view(B), kv_tok,
                              qi["sink"], out, lse=lse, ws=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref, rlse = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), np.full((B, 1), L - 1), bits16(kv_c),
                        bits16(kv_tok), f32(qi["sink"]), w.m, w.W, w.rope_dim,
                        tidx.cpu().numpy(), tcnt.cpu().numpy(), scale=scale, rope_freq=freq)
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert_attention_close(got, ref[:, 0], "V4-Flash shapes, YaRN")
    check_lse(lse, rlse[:, 0], ref[:, 0], scale)
    # The YaRN table and gain matter here: plain RoPE and 1/sqrt(d) give
    # another output (so the check above can fail).
    plain, _ = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), np.full((B, 1), L - 1), bits16(kv_c),
                       bits16(kv_tok), f32(qi["sink"]), w.m, w.W, w.rope_dim,
                       tidx.cpu().numpy(), tcnt.cpu().numpy())
    assert np.abs(plain[:, 0] - ref[:, 0]).max() > 0.05


@pytest.mark.parametrize("H,pos", [(64, 128 * 30 + 127), (48, 128 * 7 + 5), (64, 60)])
def test_dense_yarn_heads_le_64(orc, H, pos):
    """HCA dense decode with 64 or fewer heads (one CTA per split) and the
    YaRN table, including a query before the first complete block."""
    w = configs.scaled(configs.HCA_1M, B=2, H=H, yarn=configs.YARN_V4)
    B, N_cap, L_cap = 2, 40, 128 * 32
    freq, scale = oracle_rope(orc, w)
    p = binding.params_for(w, B=B)
    kv_c, kv_tok = random_cache(w, B, N_cap, L_cap, 70 + H)
    q = synth.normal_bf16((B, w.H, w.D), 71 + H, "q", DEV)
    sink = synth.normal_f32((w.H,), 72, "sink", 1.0, DEV)
    out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, w.H), float("nan"), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pos_t = torch.tensor([pos, pos - 1], dtype=torch.int64, device=DEV)
    ws = binding.workspace(p, binding.OP_DENSE_MQA, 1, N_cap)
    binding.dense_mqa_decode(p, q, pos_t, kv_c, kv_tok, sink, out, lse=lse, ws=ws,
                             dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref, rlse = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), pos_t.cpu().numpy().reshape(B, 1),
                        bits16(kv_c), bits16(kv_tok), f32(sink), w.m, w.W, w.rope_dim,
                        scale=scale, rope_freq=freq)
    got = out.double().cpu().numpy()
    assert np.isfinite(got).all()
    assert_attention_close(got, ref[:, 0], f"dense H={H}, YaRN")
    check_lse(lse, rlse[:, 0], ref[:, 0], scale)
