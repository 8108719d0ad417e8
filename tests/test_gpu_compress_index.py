"""GPU parity: KV compression, Lightning-Indexer scores and top-k against the
fp64 oracle, through the C ABI (binding -> libcsa.so)."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from gpuhelp import assert_bf16_storage_close, bits8, bits16, f32

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def e4m3_spacing(y):
    a = np.abs(y)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 2.0 ** (e - 3)


def check_keys(orc, gpu_codes, gpu_scale, ref_vals, what):
    """GPU E4M3 rows against the oracle's fp64 pre-quantisation values."""
    sc_ref = np.abs(ref_vals.astype(np.float32)).max(-1) / np.float32(448.0)
    assert np.allclose(gpu_scale, sc_ref, rtol=1e-5, atol=0), what + " scale"
    deq = orc.e4m3_decode(gpu_codes) * gpu_scale[..., None].astype(np.float64)
    y = ref_vals / gpu_scale[..., None].astype(np.float64)
    bound = 0.5 * e4m3_spacing(y) * gpu_scale[..., None] * (1 + 1e-4) + 1e-5 * np.abs(ref_vals) + 1e-7
    err = np.abs(deq - ref_vals)
    assert (err <= bound).all(), f"{what}: {(err > bound).sum()} codes off by more than half a step"


def run_compress(w, L_ctx, gamma=None, first=0, nblk=None, with_idx=True, seed_shift=0):
    B = w.B
    L_cap = max(L_ctx) if hasattr(L_ctx, "__len__") else L_ctx
    ctx = torch.tensor(L_ctx if hasattr(L_ctx, "__len__") else [L_ctx] * B, dtype=torch.int64, device=DEV)
    kv_tok, idx_tok = synth.token_streams(w, L_cap=L_cap, device=DEV)
    w_s, b_pos = synth.pool_params(w, DEV)
    N_cap = math.ceil(L_cap / w.m)
    nblk = N_cap - first if nblk is None else nblk
    kv_c = torch.zeros(B, N_cap, w.d, dtype=torch.bfloat16, device=DEV)
    p = binding.params_for(w)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = dict(kv_tok=kv_tok, idx_tok=idx_tok, w_s=w_s, b_pos=b_pos, ctx=ctx, kv_c=kv_c, N_cap=N_cap)
    if with_idx and w.csa:
        w_si, b_pi = synth.pool_params(w, DEV, indexer=True)
        idx_key = torch.zeros(B, N_cap, w.D_I, dtype=torch.uint8, device=DEV)
        idx_scale = torch.zeros(B, N_cap, dtype=torch.float32, device=DEV)
        binding.csa_compress(p, kv_tok, ctx, w_s, b_pos, gamma, first, nblk, kv_c, idx_tok, w_si,
                             b_pi, idx_key, idx_scale, dev_status=status)
        out.update(w_si=w_si, b_pi=b_pi, idx_key=idx_key, idx_scale=idx_scale)
    else:
        binding.hca_compress(p, kv_tok, ctx, w_s, b_pos, gamma, first, nblk, kv_c, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out


@pytest.mark.parametrize("L_ctx", [4096, 4094, 3])
def test_csa_compress_tiny(orc, L_ctx):
    w = configs.TINY_CSA
    r = run_compress(w, L_ctx)
    n = math.ceil(L_ctx / w.m)
    ref_bits, written, vals = orc.compress_kv(bits16(r["kv_tok"]), [L_ctx], f32(r["w_s"]), f32(r["b_pos"]),
                                              None, w.m, 0, r["N_cap"], r["N_cap"],
                                              rope_dim=w.rope_dim)
    assert written[0, :n].all() and not written[0, n:].any()
    assert_bf16_storage_close(bits16(r["kv_c"])[:, :n], vals[:, :n], "kv_c")
    assert not bits16(r["kv_c"])[:, n:].any()  # blocks past the context untouched
    codes, scale, ivals, _ = orc.compress_index(bits16(r["idx_tok"]), [L_ctx], f32(r["w_si"]),
                                                f32(r["b_pi"]), w.m, 0, r["N_cap"], r["N_cap"])
    check_keys(orc, bits8(r["idx_key"])[:, :n], f32(r["idx_scale"])[:, :n], ivals[:, :n], "idx_key")
    agree = (bits8(r["idx_key"])[:, :n] == codes[:, :n]).mean()
    assert agree > 0.999


def test_hca_compress_ragged_with_gain(orc):
    w = configs.scaled(configs.HCA_1M, B=3, L=128 * 9)
    lens = [128 * 9, 128 * 7 + 77, 5]
    gamma = synth.gains(w.d, w.seed, DEV)
    r = run_compress(w, lens, gamma=gamma)
    _, written, vals = orc.compress_kv(bits16(r["kv_tok"]), lens, f32(r["w_s"]), f32(r["b_pos"]),
                                       f32(gamma), w.m, 0, r["N_cap"], r["N_cap"],
                                       rope_dim=w.rope_dim)
    got = bits16(r["kv_c"])
    for b, L in enumerate(lens):
        n = math.ceil(L / w.m)
        assert_bf16_storage_close(got[b, :n], vals[b, :n], f"seq {b}")
        assert not got[b, n:].any()


def test_compress_newest_block_only(orc):
    # Decode-time use: compress just the block the newest token completes.
    w = configs.scaled(configs.CSA_128K, B=2, L=4096)
    r = run_compress(w, 4096, first=1023, nblk=1)
    got = bits16(r["kv_c"])
    assert not got[:, :1023].any()
    _, _, vals = orc.compress_kv(bits16(r["kv_tok"]), [4096, 4096], f32(r["w_s"]), f32(r["b_pos"]),
                                 None, w.m, 1023, 1, r["N_cap"], rope_dim=w.rope_dim)
    assert_bf16_storage_close(got[:, 1023:], vals[:, 1023:], "newest block")


# -------------------------------------------------------------- indexer --
def rand_keys(B, N, D_I, seed, device=DEV, distinct=None):
    g = torch.Generator(device="cpu").manual_seed(seed)
    if distinct is None:
        x = (torch.randn(B, N, D_I, generator=g) * 64).clamp(-448, 448)
    else:
        base = (torch.randn(distinct, D_I, generator=g) * 64).clamp(-448, 448)
        x = base[torch.randint(0, distinct, (B, N), generator=g)]
    codes = x.to(torch.float8_e4m3fn).view(torch.uint8)
    scale = torch.rand(B, N, generator=g) * 0.01 + 0.005
    if distinct is not None:
        scale[:] = 0.01
    return codes.to(device), scale.to(device)


def run_index(w, Q, N_cap, pos, key, key_scale, k=None):
    qi = synth.queries(w, Q=Q, device=DEV)
    B = w.B
    p = binding.params_for(w, **({} if k is None else {}))
    if k is not None:
        p.k = k
    topk_idx = torch.full((B, Q, p.k), -7, dtype=torch.int32, device=DEV)
    topk_cnt = torch.full((B, Q), -7, dtype=torch.int32, device=DEV)
    scores = torch.full((B, Q, N_cap), float("nan"), dtype=torch.float32, device=DEV)
    pos_t = torch.as_tensor(pos, dtype=torch.int64, device=DEV).reshape(B, Q)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    binding.lightning_index_topk(p, Q, qi["q_idx"], qi["q_scale"], qi["w"], key, key_scale, pos_t,
                                 topk_idx, topk_cnt, scores_out=scores, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return qi, pos_t, scores, topk_idx, topk_cnt


def check_index(orc, w, qi, pos_t, key, key_scale, scores, topk_idx, topk_cnt, k):
    pos = pos_t.cpu().numpy()
    N_cap = key.shape[1]
    ref = orc.index_scores(bits8(qi["q_idx"]), f32(qi["q_scale"]), f32(qi["w"]), bits8(key),
                           f32(key_scale), pos, w.m)
    got = f32(scores).astype(np.float64)
    nvis = np.minimum((pos + 1) // w.m, N_cap)
    # A-priori bound of fp32 accumulation: ~200 roundings of the absolute score.
    q8 = orc.e4m3_decode(bits8(qi["q_idx"]))
    k8 = orc.e4m3_decode(bits8(key))
    wq = np.abs(f32(qi["w"]).astype(np.float64) * f32(qi["q_scale"]).astype(np.float64))
    for b in range(w.B):
        absdot = np.einsum("qhd,nd->qhn", np.abs(q8[b]), np.abs(k8[b]))
        A = np.einsum("qh,qhn->qn", wq[b], absdot) * f32(key_scale)[b][None].astype(np.float64)
        for q in range(pos.shape[1]):
            n = nvis[b, q]
            err = np.abs(got[b, q, :n] - ref[b, q, :n])
            assert (err <= 200 * 2.0 ** -24 * A[q, :n] + 1e-30).all(), (b, q, err.max())
            assert np.isnan(got[b, q, n:]).all()  # entries past n_vis are not written
    # Top-k: bit-exact against the oracle ranking the GPU's own fp32 scores.
    gs = np.where(np.isnan(got), -np.inf, got)
    ridx, rcnt = orc.topk(gs, nvis, k)
    assert np.array_equal(topk_cnt.cpu().numpy(), rcnt)
    assert np.array_equal(topk_idx.cpu().numpy(), ridx)


def test_indexer_topk_tiny_end_to_end(orc):
    w = configs.TINY_CSA
    r = run_compress(w, w.L)
    qi, pos_t, scores, tidx, tcnt = run_index(w, 1, r["N_cap"], [[w.L - 1]], r["idx_key"], r["idx_scale"])
    check_index(orc, w, qi, pos_t, r["idx_key"], r["idx_scale"], scores, tidx, tcnt, w.k)
    # End to end against the oracle's own keys: differences only at near-ties
    # or where a key code flipped at a rounding midpoint.
    codes, scale, _, _ = orc.compress_index(bits16(r["idx_tok"]), [w.L], f32(r["w_si"]), f32(r["b_pi"]),
                                            w.m, 0, r["N_cap"], r["N_cap"])
    ref = orc.index_scores(bits8(qi["q_idx"]), f32(qi["q_scale"]), f32(qi["w"]), codes, scale,
                           pos_t.cpu().numpy(), w.m)
    ridx, _ = orc.topk(ref, np.array([[r["N_cap"]]]), w.k)
    a, b_ = set(ridx[0, 0].tolist()), set(tidx[0, 0].cpu().tolist())
    kth = np.sort(ref[0, 0])[::-1][w.k - 1]
    flipped = (bits8(r["idx_key"])[0] != codes[0]).any(-1)
    for i in a ^ b_:
        assert abs(ref[0, 0, i] - kth) <= 1e-6 * abs(kth) or flipped[i], i


@pytest.mark.parametrize("H_I,D_I,Q", [(64, 128, 37), (4, 64, 5), (64, 64, 1), (7, 128, 9),
                                        (64, 128, 2), (64, 128, 3)])
def test_indexer_causal_multi_query(orc, H_I, D_I, Q):
    w = configs.scaled(configs.CSA_128K, B=2, H_I=H_I, D_I=D_I, k=100)
    N_cap = 2048 + 13 if D_I == 128 else 2048 + 14
    key, ks = rand_keys(w.B, N_cap, D_I, 5)
    rng = np.random.default_rng(3)
    pos = rng.integers(0, 4 * N_cap, (w.B, Q))
    pos[0, 0] = 0
    pos[-1, -1] = 4 * 57 + 2
    qi, pos_t, scores, tidx, tcnt = run_index(w, Q, N_cap, pos, key, ks)
    check_index(orc, w, qi, pos_t, key, ks, scores, tidx, tcnt, w.k)


def test_topk_all_equal_scores_pick_lowest_indices(orc):
    w = configs.scaled(configs.CSA_128K, B=2)
    N_cap = 5000
    key, ks = rand_keys(w.B, N_cap, 128, 9, distinct=1)
    qi, pos_t, scores, tidx, tcnt = run_index(w, 1, N_cap, [[4 * N_cap - 1], [4 * 3000 + 1]], key, ks)
    got = tidx.cpu().numpy()
    assert np.array_equal(got[0, 0], np.arange(w.k))
    assert np.array_equal(got[1, 0], np.arange(w.k))
    check_index(orc, w, qi, pos_t, key, ks, scores, tidx, tcnt, w.k)


def test_topk_tie_heavy(orc):
    w = configs.scaled(configs.CSA_128K, B=1)
    N_cap = 20000
    key, ks = rand_keys(w.B, N_cap, 128, 11, distinct=6)
    qi, pos_t, scores, tidx, tcnt = run_index(w, 1, N_cap, [[4 * N_cap - 1]], key, ks)
    check_index(orc, w, qi, pos_t, key, ks, scores, tidx, tcnt, w.k)


def test_indexer_topk_csa_128k_shape(orc):
    w = configs.CSA_128K
    key, ks = rand_keys(w.B, w.N_c, w.D_I, 21)
    qi, pos_t, scores, tidx, tcnt = run_index(w, 1, w.N_c, [[w.L - 1]] * w.B, key, ks)
    check_index(orc, w, qi, pos_t, key, ks, scores, tidx, tcnt, w.k)


def test_indexer_topk_csa_1m_shape_sampled(orc):
    w = configs.CSA_1M
    key, ks = rand_keys(w.B, w.N_c, w.D_I, 22)
    qi, pos_t, scores, tidx, tcnt = run_index(w, 1, w.N_c, [[w.L - 1]] * w.B, key, ks)
    got = f32(scores).astype(np.float64)
    # Scores: a sample of 4096 entries per sequence through the oracle.
    rng = np.random.default_rng(0)
    samp = np.sort(rng.choice(w.N_c, 4096, replace=False))
    keys_s = bits8(key)[:, samp]
    ks_s = f32(ks)[:, samp]
    ref = orc.index_scores(bits8(qi["q_idx"]), f32(qi["q_scale"]), f32(qi["w"]), keys_s, ks_s,
                           np.full((w.B, 1), 4 * 4096 - 1), w.m)
    assert np.allclose(got[:, 0, samp], ref[:, 0], rtol=2e-5, atol=1e-6 * np.abs(ref).mean())
    # Top-k: exact against the oracle ranking the GPU scores (all 262144).
    ridx, rcnt = orc.topk(got, np.full((w.B, 1), w.N_c), w.k)
    assert np.array_equal(tidx.cpu().numpy(), ridx)
    assert (tcnt.cpu().numpy() == w.k).all()


@pytest.mark.parametrize("overlap,L_ctx", [(4, 4096), (4, 4094), (2, 37), (4, 3)])
def test_csa_compress_overlapping(orc, overlap, L_ctx):
    """Overlapping compression: entry i pools tokens i*m - overlap .. (i+1)*m - 1
    (b_pos has m + overlap values), both streams, ragged context ends."""
    w = configs.scaled(configs.TINY_CSA, overlap=overlap)
    r = run_compress(w, L_ctx)
    n = math.ceil(L_ctx / w.m)
    _, written, vals = orc.compress_kv(bits16(r["kv_tok"]), [L_ctx], f32(r["w_s"]), f32(r["b_pos"]),
                                       None, w.m, 0, r["N_cap"], r["N_cap"], rope_dim=w.rope_dim,
                                       overlap=overlap)
    assert written[0, :n].all()
    assert_bf16_storage_close(bits16(r["kv_c"])[:, :n], vals[:, :n], f"kv_c overlap={overlap}")
    _, _, ivals, _ = orc.compress_index(bits16(r["idx_tok"]), [L_ctx], f32(r["w_si"]), f32(r["b_pi"]),
                                        w.m, 0, r["N_cap"], r["N_cap"], overlap=overlap)
    check_keys(orc, bits8(r["idx_key"])[:, :n], f32(r["idx_scale"])[:, :n], ivals[:, :n],
               f"idx_key overlap={overlap}")
    # The overlap changes the entries (so the check above can fail).
    _, _, plain = orc.compress_kv(bits16(r["kv_tok"]), [L_ctx], f32(r["w_s"]), f32(r["b_pos"])[:w.m],
                                  None, w.m, 0, r["N_cap"], r["N_cap"], rope_dim=w.rope_dim)
    if n > 1:
        assert np.abs(plain[:, 1:n] - vals[:, 1:n]).max() > 1e-2


def test_csa_compress_overlapping_d512_partial_range(orc):
    """d = 512, a block range that starts mid-sequence (the borrowed tokens
    come from the block before the range)."""
    w = configs.scaled(configs.CSA_128K, B=2, overlap=4)
    r = run_compress(w, [1027, 1000], first=100, nblk=157)
    for b, L in enumerate([1027, 1000]):
        n = math.ceil(L / w.m)
        _, _, vals = orc.compress_kv(bits16(r["kv_tok"])[b: b + 1], [L], f32(r["w_s"]), f32(r["b_pos"]),
                                     None, w.m, 100, n - 100, r["N_cap"], rope_dim=w.rope_dim,
                                     overlap=4)
        assert_bf16_storage_close(bits16(r["kv_c"])[b: b + 1, 100:n], vals[:, 100:n], f"seq {b}")
