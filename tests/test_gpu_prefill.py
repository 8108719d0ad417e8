"""GPU parity of csa_prefill_chunk (one CSA prefill chunk: compression of the
new blocks, causal Lightning Indexer, top-k and sparse MQA per query) against
the fp64 oracle, through the C ABI.

The cached part of the caches (blocks before the chunk) is written from the
oracle's own compression, so no oracle input comes from the GPU.  The checks
follow the layered protocol of the other parity tests: compressed rows
against the oracle; scores against the oracle fed the GPU's E4M3 keys; the
top-k bit-exact against the oracle ranking the GPU's scores; attention
against the oracle fed the GPU's selection and compressed rows."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from gpuhelp import (assert_attention_close, assert_bf16_storage_close, assert_lse_close, bits8,
                     bits16, f32)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def _e4m3_half_step(y):
    a = np.abs(y)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return 0.5 * 2.0 ** (e - 3)


def run_prefill(orc, w, P, T):
    m = w.m
    L_cap = P + T
    N_cap = math.ceil(L_cap / m)
    b0 = P // m
    kv_tok, idx_tok = synth.token_streams(w, L_cap=L_cap)
    w_s, b_pos = synth.pool_params(w)
    w_si, b_pi = synth.pool_params(w, indexer=True)
    qi = synth.queries(w, Q=T)
    kv_bits, idx_bits = bits16(kv_tok), bits16(idx_tok)
    # Cached blocks 0 .. b0-1 from the oracle.
    kv_c0, _, _ = orc.compress_kv(kv_bits, [P], f32(w_s), f32(b_pos), None, m, 0, b0, N_cap,
                                  rope_dim=w.rope_dim, overlap=w.overlap)
    key0, ks0, _, _ = orc.compress_index(idx_bits, [P], f32(w_si), f32(b_pi), m, 0, b0, N_cap,
                                         overlap=w.overlap)
    kv_c = torch.from_numpy(kv_c0.view(np.int16)).view(torch.bfloat16).to(DEV)
    idx_key = torch.from_numpy(key0).to(DEV)
    idx_scale = torch.from_numpy(ks0).to(DEV)
    p = binding.params_for(w, B=1)
    ws = binding.workspace(p, binding.OP_PREFILL, T, N_cap)
    out = torch.empty(T, w.H, w.D, dtype=torch.bfloat16, device=DEV)
    tidx = torch.full((T, w.k), -7, dtype=torch.int32, device=DEV)
    tcnt = torch.full((T,), -7, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    d = {k: v.to(DEV) for k, v in qi.items()}
    binding.csa_prefill_chunk(p, P, T, kv_tok.to(DEV), idx_tok.to(DEV), w_s.to(DEV),
                              b_pos.to(DEV), None, w_si.to(DEV), b_pi.to(DEV), kv_c, idx_key,
                              idx_scale, d["q"][0].contiguous(), d["q_idx"][0].contiguous(),
                              d["q_scale"][0].contiguous(), d["w"][0].contiguous(), d["sink"],
                              tidx, tcnt, out, ws=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    scores = ws[: T * N_cap * 4].view(torch.float32).reshape(T, N_cap)
    return dict(P=P, T=T, N_cap=N_cap, b0=b0, kv_bits=kv_bits, idx_bits=idx_bits, w_s=w_s,
                b_pos=b_pos, w_si=w_si, b_pi=b_pi, qi=qi, kv_c0=kv_c0, key0=key0, ks0=ks0,
                kv_c=bits16(kv_c), idx_key=bits8(idx_key), idx_scale=f32(idx_scale),
                scores=f32(scores).astype(np.float64), idx=tidx.cpu().numpy(),
                cnt=tcnt.cpu().numpy(), out=f32(out).astype(np.float64))


def check_prefill(orc, w, r, rows):
    m, P, T, N_cap, b0 = w.m, r["P"], r["T"], r["N_cap"], r["b0"]
    # 1. Compression: cached rows untouched, new rows against the oracle.
    assert np.array_equal(r["kv_c"][:, :b0], r["kv_c0"][:, :b0])
    assert np.array_equal(r["idx_key"][:, :b0], r["key0"][:, :b0])
    _, _, vals = orc.compress_kv(r["kv_bits"], [P + T], f32(r["w_s"]), f32(r["b_pos"]), None, m,
                                 b0, N_cap - b0, N_cap, rope_dim=w.rope_dim, overlap=w.overlap)
    assert_bf16_storage_close(r["kv_c"][:, b0:], vals[:, b0:], "new KV entries")
    _, ks_ref, kvals, _ = orc.compress_index(r["idx_bits"], [P + T], f32(r["w_si"]),
                                             f32(r["b_pi"]), m, b0, N_cap - b0, N_cap,
                                             overlap=w.overlap)
    sc = r["idx_scale"][:, b0:]
    assert np.allclose(sc, ks_ref[:, b0:], rtol=1e-5, atol=0), "key scales"
    deq = orc.e4m3_decode(r["idx_key"][:, b0:]) * sc[..., None].astype(np.float64)
    ref = kvals[:, b0:]
    bound = _e4m3_half_step(ref / sc[..., None]) * sc[..., None] * (1 + 1e-4) + 1e-5 * np.abs(ref)
    assert (np.abs(deq - ref) <= bound + 1e-7).all(), "new indexer keys"
    # 2. Scores of the sampled rows (visible entries only) against the oracle.
    pos = (P + np.arange(T)).reshape(1, T)
    nv = np.minimum((pos[0] + 1) // m, N_cap)
    qi = r["qi"]
    ref_sc = orc.index_scores(bits8(qi["q_idx"])[:, rows], f32(qi["q_scale"])[:, rows],
                              f32(qi["w"])[:, rows], r["idx_key"], r["idx_scale"],
                              pos[:, rows], m)[0]
    for j, t in enumerate(rows):
        n = nv[t]
        if n == 0:
            continue
        got, want = r["scores"][t, :n], ref_sc[j, :n]
        assert np.allclose(got, want, rtol=2e-5, atol=1e-6 * max(np.abs(want).mean(), 1e-30)), \
            f"scores of query {t}"
    # 3. Top-k of every row, bit-exact against the oracle ranking the GPU's scores.
    ridx, rcnt = orc.topk(r["scores"], nv, w.k)
    assert np.array_equal(r["cnt"], rcnt)
    bad = np.nonzero((r["idx"] != ridx).any(-1))[0]
    assert bad.size == 0, f"top-k rows {bad[:8]} differ"
    # 4. Attention of the sampled rows with the GPU's selection and entries.
    ref_out, _ = orc.mqa(bits16(qi["q"])[:, rows], pos[:, rows], r["kv_c"], r["kv_bits"],
                         f32(qi["sink"]), m, w.W, w.rope_dim, r["idx"][None, rows],
                         r["cnt"][None, rows])
    assert_attention_close(r["out"][rows], ref_out[0], "prefill attention")


def _sample_rows(T, m, n_rand, seed):
    rng = np.random.default_rng(seed)
    rows = set(range(min(T, 6))) | set(range(max(0, T - 6), T))
    rows |= {t for t in range(T) if t % m in (m - 2, m - 1) and t < 4 * m}
    rows |= set(rng.choice(T, min(T, n_rand), replace=False).tolist())
    return np.array(sorted(rows))


@pytest.mark.parametrize("P,T", [(8192, 299), (0, 150), (4096 + 4 * 200, 64)])
def test_prefill_small(orc, P, T):
    """Ragged chunks: a partial last block, a chunk that starts the sequence
    (windows clipped at 0, fewer visible entries than k), one in the middle."""
    w = configs.scaled(configs.CSA_PREFILL, L=P + T, P=P, T=T)
    r = run_prefill(orc, w, P, T)
    check_prefill(orc, w, r, _sample_rows(T, w.m, 24, P + T))


@pytest.mark.parametrize("P,T", [(4096, 203), (0, 90)])
def test_prefill_small_overlapping(orc, P, T):
    """Overlapping compression (window of 2m tokens at stride m) through the
    prefill chunk: the first new block borrows the last cached tokens."""
    w = configs.scaled(configs.CSA_PREFILL, L=P + T, P=P, T=T, overlap=4)
    r = run_prefill(orc, w, P, T)
    check_prefill(orc, w, r, _sample_rows(T, w.m, 16, P + T + 1))


@pytest.mark.slow
def test_prefill_full_shape_sampled(orc):
    """The 4096-token chunk after 65536 cached tokens; every row's top-k, the
    scores and attention of sampled rows."""
    w = configs.CSA_PREFILL
    r = run_prefill(orc, w, w.P, w.T)
    check_prefill(orc, w, r, _sample_rows(w.T, w.m, 6, 7))


# ------------------------------------------------------------ HCA prefill --
def run_hca_prefill(orc, w, P, T, gamma=False):
    m = w.m
    L_cap = P + T
    N_cap = math.ceil(L_cap / m)
    b0 = P // m
    kv_tok, _ = synth.token_streams(w, L_cap=L_cap)
    w_s, b_pos = synth.pool_params(w)
    qi = synth.queries(w, Q=T)
    kv_bits = bits16(kv_tok)
    g = synth.gains(w.d, w.seed) if gamma else None
    # Cached blocks 0 .. b0-1 from the oracle.
    kv_c0, _, _ = orc.compress_kv(kv_bits, [P], f32(w_s), f32(b_pos), None if g is None else f32(g),
                                  m, 0, b0, N_cap, rope_dim=w.rope_dim)
    kv_c = torch.from_numpy(kv_c0.view(np.int16)).view(torch.bfloat16).to(DEV)
    p = binding.params_for(w, B=1)
    ws = binding.workspace(p, binding.OP_HCA_PREFILL, T, N_cap)
    out = torch.full((T, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((T, w.H), float("nan"), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    binding.hca_prefill_chunk(p, P, T, kv_tok.to(DEV), w_s.to(DEV), b_pos.to(DEV),
                              None if g is None else g.to(DEV), kv_c, qi["q"][0].contiguous().to(DEV),
                              qi["sink"].to(DEV), out, lse=lse, ws=ws, dev_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return dict(P=P, T=T, N_cap=N_cap, b0=b0, kv_bits=kv_bits, w_s=w_s, b_pos=b_pos, g=g, qi=qi,
                kv_c0=kv_c0, kv_c=bits16(kv_c), out=f32(out).astype(np.float64),
                lse=f32(lse).astype(np.float64))


def check_hca_prefill(orc, w, r, rows):
    m, P, T, N_cap, b0 = w.m, r["P"], r["T"], r["N_cap"], r["b0"]
    g = None if r["g"] is None else f32(r["g"])
    # 1. Compression: cached rows untouched, new rows (partial last block
    # included) against the oracle.
    assert np.array_equal(r["kv_c"][:, :b0], r["kv_c0"][:, :b0])
    _, _, vals = orc.compress_kv(r["kv_bits"], [P + T], f32(r["w_s"]), f32(r["b_pos"]), g, m, b0,
                                 N_cap - b0, N_cap, rope_dim=w.rope_dim)
    assert_bf16_storage_close(r["kv_c"][:, b0:], vals[:, b0:], "new HCA entries")
    # 2. Dense attention of the sampled rows with the GPU's entries.
    pos = (P + np.arange(T)).reshape(1, T)
    ref, rlse = orc.mqa(bits16(r["qi"]["q"])[:, rows], pos[:, rows], r["kv_c"], r["kv_bits"],
                        f32(r["qi"]["sink"]), m, w.W, w.rope_dim)
    got = r["out"][rows]
    assert np.isfinite(got).all()
    assert_attention_close(got, ref[0], "HCA prefill attention")
    gl, rl = r["lse"][rows], rlse[0]
    assert_lse_close(gl, rl, ref[0], "HCA prefill LSE")


@pytest.mark.parametrize("P,T,gamma", [(128 * 10, 300, False), (0, 260, True), (128 * 3, 128, False)])
def test_hca_prefill_small(orc, P, T, gamma):
    """Ragged chunks through the HCA layer: a partial last block, a chunk that
    starts the sequence (queries before the first complete block see only
    their window), one that ends on a block boundary; with and without a gain."""
    w = configs.scaled(configs.HCA_PREFILL, L=P + T, P=P, T=T)
    r = run_hca_prefill(orc, w, P, T, gamma)
    rows = _sample_rows(T, w.m, 24, P + T)
    rows = np.union1d(rows, [t for t in (126, 127, 128, 255, 256) if t < T])
    check_hca_prefill(orc, w, r, rows)


@pytest.mark.slow
def test_hca_prefill_full_shape_sampled(orc):
    """The 4096-token chunk after 65,536 cached tokens: the 32 new entries and
    sampled rows' attention."""
    w = configs.HCA_PREFILL
    r = run_hca_prefill(orc, w, w.P, w.T)
    check_hca_prefill(orc, w, r, _sample_rows(w.T, w.m, 8, 11))
