"""Pins of the fp64 oracle against things other than itself.

Each test ties one oracle function to a library routine, a closed form, an
invariant of the method, or brute force on tiny inputs, chosen so that a
plausible slip (dropped term, wrong sign or index, transposed operand) fails.
No GPU is used.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from scipy.special import logsumexp

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16_bits(x):
    return torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ formats --
def test_bf16_encode_matches_torch_rne(orc):
    r = rng(1)
    x32 = np.concatenate([r.standard_normal(20000).astype(np.float32) * 10.0 ** r.integers(-30, 30, 20000),
                          np.array([1.00390625, 1.01171875, -1.00390625, 3.0e38, 1e-40, 0.0, -0.0], np.float32)])
    x32 = x32.astype(np.float32)
    ours = orc.bf16_encode(x32.astype(np.float64))
    ref = bf16_bits(x32)
    finite = np.isfinite(x32)
    assert np.array_equal(ours[finite], ref[finite])


def test_bf16_encode_is_direct_from_fp64(orc):
    # 1 + 2^-8 + 2^-30 is above the bf16 midpoint in fp64 but rounds to the
    # midpoint in fp32; a direct fp64 rounding must go up.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert orc.bf16_decode(orc.bf16_encode(np.array([x])))[0] == 1.0078125


def test_e4m3_decode_all_codes_match_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours) == -448.0


def test_e4m3_encode_roundtrip_midpoints_saturation(orc):
    vals = orc.e4m3_decode(np.arange(256, dtype=np.uint8))
    for c in range(256):
        v = vals[c]
        if np.isnan(v):
            continue
        assert orc.e4m3_encode_scalar(v) == c
    pos = np.sort(vals[(vals >= 0) & ~np.isnan(vals)])
    pos = np.unique(pos)
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (a + b) / 2
        ca, cb = orc.e4m3_encode_scalar(a), orc.e4m3_encode_scalar(b)
        even = ca if (ca & 1) == 0 else cb
        assert orc.e4m3_encode_scalar(mid) == even, (a, b)
    assert orc.e4m3_encode_scalar(1e6) == 0x7E
    assert orc.e4m3_encode_scalar(-1e6) == 0xFE
    assert orc.e4m3_encode_scalar(460.0) == 0x7E
    assert orc.e4m3_encode_scalar(float("nan")) & 0x7F == 0x7F


def test_e4m3_encode_matches_torch_in_range(orc):
    x = (rng(2).standard_normal(5000) * 60).clip(-440, 440).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([orc.e4m3_encode_scalar(v) for v in x], np.uint8)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------- compression --
def _tok(B, L, d, seed):
    return bf16_bits(rng(seed).standard_normal((B, L, d)).astype(np.float32))


@pytest.mark.parametrize("L", [1, 3, 4, 5, 127, 128, 129, 4096])
@pytest.mark.parametrize("m", [4, 128])
def test_compressed_length_is_ceil(orc, L, m):
    d = 8
    tok = _tok(1, max(L, 1), d, 3)
    N_cap = L // m + 3
    _, written = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(m), None, m, 0, N_cap, N_cap)
    assert written.sum() == math.ceil(L / m)
    assert written[0, : math.ceil(L / m)].all()


def test_pool_uniform_weights_is_block_mean(orc):
    B, L, d, m = 2, 37, 16, 4
    tok = _tok(B, L, d, 4)
    x = orc.bf16_decode(tok)
    N = math.ceil(L / m)
    vals, _ = orc.pool(tok, np.array([L, L]), np.zeros(d), np.zeros(m), None, m, 0, N, N, normalize=False)
    for i in range(N):
        ref = x[:, i * m: min(L, (i + 1) * m)].mean(axis=1)
        assert np.allclose(vals[:, i], ref, rtol=0, atol=1e-15)


def test_pool_uniform_then_rmsnorm_matches_torch(orc):
    B, L, d, m = 1, 256, 64, 128
    tok = _tok(B, L, d, 5)
    gamma = (1 + 0.3 * rng(6).standard_normal(d)).astype(np.float32)
    x = torch.from_numpy(orc.bf16_decode(tok))
    vals, _ = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(m), gamma, m, 0, 2, 2, eps=1e-6)
    mean = x.view(B, 2, m, d).mean(2)
    ref = F.rms_norm(mean, (d,), torch.from_numpy(gamma.astype(np.float64)), eps=1e-6)
    assert torch.allclose(torch.from_numpy(vals), ref, rtol=1e-13, atol=1e-13)


def test_pool_m1_is_rmsnorm_of_token(orc):
    B, L, d = 1, 9, 32
    tok = _tok(B, L, d, 7)
    w_s = rng(8).standard_normal(d).astype(np.float32)
    vals, _ = orc.pool(tok, np.array([L]), w_s, np.array([0.3], np.float32), None, 1, 0, L, L)
    ref = F.rms_norm(torch.from_numpy(orc.bf16_decode(tok)), (d,), eps=1e-6).numpy()
    assert np.allclose(vals, ref, rtol=1e-13, atol=1e-13)


def test_pool_position_bias_selects_token(orc):
    B, L, d, m = 1, 8, 16, 4
    tok = _tok(B, L, d, 9)
    x = orc.bf16_decode(tok)
    b_pos = np.array([0, 0, 80, 0], np.float32)
    vals, _ = orc.pool(tok, np.array([L]), np.zeros(d), b_pos, None, m, 0, 2, 2, normalize=False)
    assert np.allclose(vals[0, 0], x[0, 2], rtol=0, atol=1e-30)
    assert np.allclose(vals[0, 1], x[0, 6], rtol=0, atol=1e-30)


def test_pool_content_score_selects_token(orc):
    # s_j = c_j . w_s: a w_s aligned with token 1 makes it dominate its block.
    B, L, d, m = 1, 4, 64, 4
    tok = _tok(B, L, d, 10)
    x = orc.bf16_decode(tok)
    w_s = (x[0, 1] * 50).astype(np.float32)
    s = x[0] @ w_s.astype(np.float64)
    assert s[1] - np.max(np.delete(s, 1)) > 60
    vals, _ = orc.pool(tok, np.array([L]), w_s, np.zeros(m), None, m, 0, 1, 1, normalize=False)
    assert np.allclose(vals[0, 0], x[0, 1], rtol=0, atol=1e-20)


def test_pool_permutation_and_shift_invariance(orc):
    B, L, d, m = 1, 4, 32, 4
    tok = _tok(B, L, d, 11)
    w_s = (0.3 * rng(12).standard_normal(d)).astype(np.float32)
    b_pos = np.array([0.5, -1.0, 0.25, 2.0], np.float32)
    base, _ = orc.pool(tok, np.array([L]), w_s, b_pos, None, m, 0, 1, 1)
    perm = np.array([2, 0, 3, 1])
    alt, _ = orc.pool(tok[:, perm], np.array([L]), w_s, b_pos[perm], None, m, 0, 1, 1)
    assert np.allclose(alt, base, rtol=1e-13, atol=1e-14)
    sh, _ = orc.pool(tok, np.array([L]), w_s, b_pos + 3.0, None, m, 0, 1, 1)
    assert np.allclose(sh, base, rtol=1e-13, atol=1e-14)
    # Swapping tokens WITHOUT swapping the biases must change the result.
    diff, _ = orc.pool(tok[:, perm], np.array([L]), w_s, b_pos, None, m, 0, 1, 1)
    assert not np.allclose(diff, base, rtol=1e-6, atol=1e-6)


def test_pool_partial_block_uses_present_tokens(orc):
    B, L, d, m = 1, 6, 8, 4
    tok = _tok(B, 8, d, 13)
    x = orc.bf16_decode(tok)
    vals, w = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(m), None, m, 0, 2, 2, normalize=False)
    assert w[0].tolist() == [True, True]
    assert np.allclose(vals[0, 1], x[0, 4:6].mean(0), rtol=0, atol=1e-15)


def test_quant_rows_matches_torch_cast_and_bound(orc):
    x = rng(14).standard_normal((50, 128)) * rng(15).uniform(0.01, 10, (50, 1))
    codes, scale = orc.quant_rows_e4m3(x)
    x32 = torch.from_numpy(x.astype(np.float32))
    amax = x32.abs().amax(1)
    assert np.array_equal(scale, (amax / 448.0).numpy())
    ref = (x32 / torch.from_numpy(scale)[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    deq = orc.e4m3_decode(codes) * scale[:, None].astype(np.float64)
    # Relative E4M3 spacing is 2^-3 (normals): error <= half a spacing of the value.
    assert np.all(np.abs(deq - x) <= np.abs(x) * 2.0 ** -4 + scale[:, None] * 2.0 ** -10 + 1e-6 * np.abs(x))
    zero_codes, zero_scale = orc.quant_rows_e4m3(np.zeros((1, 16)))
    assert zero_scale[0] == 1.0 and not zero_codes.any()


# ------------------------------------------------------------------- indexer --
def _idx_inputs(B, Q, H_I, D_I, N, seed):
    r = rng(seed)
    q_idx = torch.from_numpy((r.standard_normal((B, Q, H_I, D_I)) * 64).clip(-448, 448).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    key = torch.from_numpy((r.standard_normal((B, N, D_I)) * 64).clip(-448, 448).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    q_scale = r.uniform(0.005, 0.02, (B, Q, H_I)).astype(np.float32)
    k_scale = r.uniform(0.005, 0.02, (B, N)).astype(np.float32)
    w = r.uniform(0, 1, (B, Q, H_I)).astype(np.float32)
    return q_idx, q_scale, w, key, k_scale


def test_index_scores_brute_force(orc):
    B, Q, H_I, D_I, N, m = 2, 3, 4, 16, 40, 4
    q_idx, q_scale, w, key, k_scale = _idx_inputs(B, Q, H_I, D_I, N, 16)
    pos = np.array([[159, 100, 3], [50, 159, 0]])
    got = orc.index_scores(q_idx, q_scale, w, key, k_scale, pos, m)
    qf = torch.from_numpy(q_idx).view(torch.float8_e4m3fn).to(torch.float64).numpy() * q_scale[..., None]
    kf = torch.from_numpy(key).view(torch.float8_e4m3fn).to(torch.float64).numpy() * k_scale[..., None]
    dots = np.einsum("bqhd,bnd->bqhn", qf, kf)
    ref = np.einsum("bqh,bqhn->bqn", w.astype(np.float64), np.maximum(dots, 0))
    nvis = (pos + 1) // m
    for b in range(B):
        for q in range(Q):
            n = nvis[b, q]
            assert np.allclose(got[b, q, :n], ref[b, q, :n], rtol=1e-12, atol=0)
            assert np.all(np.isneginf(got[b, q, n:]))


def test_index_scores_single_head_is_relu_dot_and_factoring(orc):
    B, Q, H_I, D_I, N = 1, 1, 1, 32, 64
    q_idx, q_scale, w, key, k_scale = _idx_inputs(B, Q, H_I, D_I, N, 17)
    w[:] = 1.0
    pos = np.array([[4 * N - 1]])
    got = orc.index_scores(q_idx, q_scale, w, key, k_scale, pos, 4)[0, 0]
    qf = torch.from_numpy(q_idx).view(torch.float8_e4m3fn).to(torch.float64).numpy()[0, 0, 0] * q_scale[0, 0, 0]
    kf = torch.from_numpy(key).view(torch.float8_e4m3fn).to(torch.float64).numpy()[0] * k_scale[0][:, None]
    assert np.allclose(got, np.maximum(kf @ qf, 0), rtol=1e-12, atol=0)
    # Factored form (integer-code dot, scales pulled out of the ReLU) gives the same.
    B, Q, H_I = 1, 1, 8
    q_idx, q_scale, w, key, k_scale = _idx_inputs(B, Q, H_I, D_I, N, 18)
    got = orc.index_scores(q_idx, q_scale, w, key, k_scale, pos, 4)[0, 0]
    q8 = torch.from_numpy(q_idx).view(torch.float8_e4m3fn).to(torch.float64).numpy()[0, 0]
    k8 = torch.from_numpy(key).view(torch.float8_e4m3fn).to(torch.float64).numpy()[0]
    fact = k_scale[0].astype(np.float64) * (np.maximum(k8 @ q8.T, 0) @ (w[0, 0].astype(np.float64) * q_scale[0, 0].astype(np.float64)))
    assert np.allclose(got, fact, rtol=1e-12, atol=0)


# --------------------------------------------------------------------- top-k --
def _ref_topk(s, n, k):
    order = np.argsort(-s[:n], kind="stable")
    sel = np.sort(order[: min(k, n)])
    return np.concatenate([sel, -np.ones(k - len(sel), np.int64)])


@pytest.mark.parametrize("distinct", [None, 8, 1])
def test_topk_matches_stable_sort(orc, distinct):
    r = rng(19)
    BQ, N, k = 6, 500, 37
    s = r.standard_normal((BQ, N))
    if distinct:
        s = r.integers(0, distinct, (BQ, N)).astype(np.float64)
    n_vis = np.array([500, 37, 36, 1, 0, 250])
    idx, cnt = orc.topk(s, n_vis, k)
    for i in range(BQ):
        ref = _ref_topk(s[i], n_vis[i], k)
        assert np.array_equal(idx[i], ref)
        assert cnt[i] == min(k, n_vis[i])


def test_topk_nan_last_and_signed_zero_ties(orc):
    s = np.array([[np.nan, 0.0, -0.0, 1.0, np.nan, -1.0]])
    idx, cnt = orc.topk(s, np.array([6]), 3)
    assert idx[0].tolist() == [1, 2, 3]
    idx, cnt = orc.topk(s, np.array([6]), 5)
    assert idx[0].tolist() == [0, 1, 2, 3, 5]


# ----------------------------------------------------------------- attention --
def _mqa_case(B, Q, H, D, L, m, seed):
    r = rng(seed)
    q = bf16_bits(r.standard_normal((B, Q, H, D)))
    kv_tok = bf16_bits(r.standard_normal((B, L, D)))
    N = L // m
    kv_c = bf16_bits(r.standard_normal((B, N, D)))
    sink = r.standard_normal(H).astype(np.float32)
    return q, kv_tok, kv_c, sink


def test_sparse_with_all_entries_equals_dense(orc):
    B, Q, H, D, L, m, W = 2, 1, 4, 32, 64, 4, 8
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 20)
    pos = np.array([[63], [40]])
    nvis = (pos + 1) // m
    sel = np.full((B, Q, 32), -1, np.int32)
    cnt = np.zeros((B, Q), np.int32)
    for b in range(B):
        sel[b, 0, : nvis[b, 0]] = np.arange(nvis[b, 0])
        cnt[b, 0] = nvis[b, 0]
    o_s, l_s = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, 16, sel, cnt)
    o_d, l_d = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, 16)
    assert np.allclose(o_s, o_d, rtol=1e-14, atol=1e-14)
    assert np.allclose(l_s, l_d, rtol=1e-14, atol=1e-14)
    # Order of the selection list does not matter.
    sel2 = sel.copy()
    sel2[0, 0, : cnt[0, 0]] = sel2[0, 0, : cnt[0, 0]][::-1]
    o_r, _ = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, 16, sel2, cnt)
    assert np.allclose(o_r, o_s, rtol=1e-14, atol=1e-14)


def test_window_only_no_sink_is_textbook_attention(orc):
    # pos < m-1: no complete block, so the KV set is the window; r = 0 and a
    # sink of -inf make it plain softmax attention with K = V.
    B, Q, H, D, L, m, W = 1, 1, 8, 64, 128, 128, 128
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 21)
    sink[:] = -np.inf
    gq = (1 + 0.2 * rng(22).standard_normal(D)).astype(np.float32)
    gk = (1 + 0.2 * rng(23).standard_normal(D)).astype(np.float32)
    pos = np.array([[100]])
    out, lse = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, 0, None, None, gq, gk)
    qt = F.rms_norm(torch.from_numpy(orc.bf16_decode(q))[0, 0], (D,), torch.from_numpy(gq.astype(np.float64)), 1e-6)
    kt = F.rms_norm(torch.from_numpy(orc.bf16_decode(kv_tok))[0, :101], (D,), torch.from_numpy(gk.astype(np.float64)), 1e-6)
    ref = F.scaled_dot_product_attention(qt[None], kt[None, None].expand(1, H, -1, -1)[0][None],
                                         kt[None, None].expand(1, H, -1, -1)[0][None])[0]
    assert np.allclose(out[0, 0], ref.numpy(), rtol=1e-12, atol=1e-12)
    logits = (qt @ kt.T).numpy() / math.sqrt(D)
    assert np.allclose(lse[0, 0], logsumexp(logits, axis=1), rtol=1e-13, atol=1e-13)


def test_window_clipped_at_sequence_start(orc):
    B, Q, H, D, L, m, W = 1, 1, 2, 16, 16, 128, 128
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 24)
    sink[:] = -np.inf
    out5, _ = orc.mqa(q, np.array([[5]]), kv_c, kv_tok, sink, m, W, 0)
    # Tokens after the query position are never read.
    kv2 = kv_tok.copy()
    kv2[0, 6:] = bf16_bits(np.full((L - 6, D), 7.0))
    out5b, _ = orc.mqa(q, np.array([[5]]), kv_c, kv2, sink, m, W, 0)
    assert np.array_equal(out5, out5b)


def test_sink_limits_and_closed_form(orc):
    B, Q, H, D, L, m, W = 1, 1, 3, 32, 4, 4, 1
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 25)
    pos = np.array([[0]])  # the KV set is the single window token 0
    x = orc.bf16_decode(kv_tok)[0, 0]
    v = x / np.sqrt(np.mean(x * x) + 1e-6)
    # Sink -inf: output is the (inverse-roped) roped vector, i.e. v itself.
    s_inf = np.full(H, -np.inf, np.float32)
    out, _ = orc.mqa(q, pos, kv_c, kv_tok, s_inf, m, W, 8)
    assert np.allclose(out[0, 0], np.broadcast_to(v, (H, D)), rtol=1e-13, atol=1e-13)
    # Sink +inf: zero output.
    out, lse = orc.mqa(q, pos, kv_c, kv_tok, np.full(H, np.inf, np.float32), m, W, 8)
    assert not out.any() and np.all(np.isposinf(lse))
    # Finite sink: o = sigmoid(s - z) v with s = scale * qhat . v.
    qh = orc.bf16_decode(q)[0, 0]
    qn = qh / np.sqrt(np.mean(qh * qh, axis=1, keepdims=True) + 1e-6)
    s = (qn @ v) / math.sqrt(D)
    z = np.array([0.5, -2.0, 3.0], np.float32)
    out, lse = orc.mqa(q, pos, kv_c, kv_tok, z, m, W, 0)
    p = 1 / (1 + np.exp(z.astype(np.float64) - s))
    assert np.allclose(out[0, 0], p[:, None] * v[None], rtol=1e-12, atol=1e-13)
    assert np.allclose(lse[0, 0], np.logaddexp(s, z.astype(np.float64)), rtol=1e-13)


def _rotate(v, pos, r_dim, base=10000.0, theta=None):
    """Rotate-half rotation of the last r_dim dims of v by position pos (the
    textbook form, written out here to check the oracle against it); theta
    overrides the per-pair frequencies."""
    D = v.shape[-1]
    half = r_dim // 2
    th = base ** (-2.0 * np.arange(half) / r_dim) if theta is None else np.asarray(theta)
    c, s = np.cos(pos * th), np.sin(pos * th)
    out = v.copy()
    x1, x2 = v[..., D - r_dim: D - half], v[..., D - half:]
    out[..., D - r_dim: D - half] = x1 * c - x2 * s
    out[..., D - half:] = x2 * c + x1 * s
    return out


def test_rope_inverse_on_output_closed_form(orc):
    # One stored entry (stored already rotated to its position), no window,
    # sink -inf: the output is that stored vector rotated back by the query
    # position.
    B, Q, H, D, m, r_dim = 1, 1, 2, 32, 4, 16
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, 16, m, 26)
    sink[:] = -np.inf
    pos = np.array([[11]])  # n_vis = 3
    cnt = np.array([[1]], np.int32)
    for ent in (0, 2):
        out, _ = orc.mqa(q, pos, kv_c, kv_tok, sink, m, 0, r_dim, np.array([[[ent, -1]]], np.int32),
                         cnt)
        ref = _rotate(orc.bf16_decode(kv_c)[0, ent], -11.0, r_dim)
        assert np.allclose(out[0, 0], np.broadcast_to(ref, (H, D)), rtol=1e-12, atol=1e-12)
    # Window token t (one token window at the query position): rotated to t
    # and back, so the output is the normalised token itself.
    x = orc.bf16_decode(kv_tok)[0, 11]
    v = x / np.sqrt(np.mean(x * x) + 1e-6)
    out_w, _ = orc.mqa(q, pos, kv_c, kv_tok, sink, m, 1, r_dim, np.array([[[-1, -1]]], np.int32),
                       np.array([[0]], np.int32))
    assert np.allclose(out_w[0, 0], np.broadcast_to(v, (H, D)), rtol=1e-12, atol=1e-12)


def test_compression_stores_entry_rotated_to_its_position(orc):
    # m = 1 with uniform weights: the entry is RMSNorm(c_t) rotated to t.
    B, L, d, r_dim = 1, 6, 32, 16
    r = rng(31)
    tok = bf16_bits(r.standard_normal((B, L, d)))
    vals, _ = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(1), None, 1, 0, L, L,
                       rope_dim=r_dim)
    x = orc.bf16_decode(tok)[0]
    nrm = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6)
    for t in range(L):
        assert np.allclose(vals[0, t], _rotate(nrm[t], float(t), r_dim), rtol=1e-12, atol=1e-13)
    # m = 4: block i is rotated to its last token, 4i + 3 (and only the last
    # r_dim dims move).
    m, N = 4, 3
    tok = bf16_bits(r.standard_normal((B, m * N, d)))
    w_s = (r.standard_normal(d) * 0.1).astype(np.float32)
    b_pos = (r.standard_normal(m) * 0.1).astype(np.float32)
    plain, _ = orc.pool(tok, np.array([m * N]), w_s, b_pos, None, m, 0, N, N)
    roped, _ = orc.pool(tok, np.array([m * N]), w_s, b_pos, None, m, 0, N, N, rope_dim=r_dim)
    for i in range(N):
        assert np.allclose(roped[0, i], _rotate(plain[0, i], float(4 * i + 3), r_dim), rtol=1e-12,
                           atol=1e-13)
    assert np.array_equal(roped[0, :, : d - r_dim], plain[0, :, : d - r_dim])


def test_rope_translation_invariance(orc):
    # Shifting every position (query, window, entries) by S leaves the output
    # unchanged.  Stored entries are kept exactly: their rotated dims are
    # zero, so re-rotating them to the shifted positions is exact in bf16.
    B, Q, H, D, L, m, W, r_dim = 1, 1, 4, 64, 64, 4, 16, 32
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 27)
    kv_c[..., D - r_dim:] = 0
    pos = np.array([[59]])
    sel = np.array([[[1, 5, 9, 14]]], np.int32)
    cnt = np.array([[4]], np.int32)
    base, lb = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, r_dim, sel, cnt)
    for shift_blocks in (1, 1000, 250000):
        S = shift_blocks * m
        kv_tok2 = np.concatenate([np.zeros((B, S, D), np.uint16), kv_tok], 1)
        kv_c2 = np.concatenate([np.zeros((B, shift_blocks, D), np.uint16), kv_c], 1)
        out, l2 = orc.mqa(q, pos + S, kv_c2, kv_tok2, sink, m, W, r_dim, sel + shift_blocks, cnt)
        assert np.allclose(out, base, rtol=1e-9, atol=1e-9)
        assert np.allclose(l2, lb, rtol=1e-9, atol=1e-9)
    # Without the inverse rotation the output would not be invariant: a check
    # that the test can fail (the rotated dims do move when the window moves).
    out_other, _ = orc.mqa(q, pos + 4, np.concatenate([np.zeros((B, 1, D), np.uint16), kv_c], 1),
                           kv_tok.copy(), sink, m, W, r_dim, sel + 1, cnt)
    assert not np.allclose(out_other, base, rtol=1e-6, atol=1e-6)


def test_incomplete_block_is_invisible(orc):
    B, Q, H, D, L, m, W = 1, 1, 2, 16, 32, 4, 4
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 28)
    pos = np.array([[9]])  # blocks 0 and 1 complete; block 2 (tokens 8..11) incomplete
    o1, _ = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, 8)
    kv_c2 = kv_c.copy()
    kv_c2[0, 2:] = bf16_bits(np.full((kv_c.shape[1] - 2, D), 5.0))
    o2, _ = orc.mqa(q, pos, kv_c2, kv_tok, sink, m, W, 8)
    assert np.array_equal(o1, o2)
    kv_c2[0, 1] = bf16_bits(np.full(D, 5.0))
    o3, _ = orc.mqa(q, pos, kv_c2, kv_tok, sink, m, W, 8)
    assert not np.allclose(o3, o1)


# ------------------------------------------------------ YaRN (context extension)
def test_yarn_factor_one_is_plain_rope(orc):
    plain = 10000.0 ** (-np.arange(32) / 32.0)
    assert np.allclose(orc.yarn_inv_freq(64, 1.0, 32.0, 1.0, 4096), plain, rtol=1e-15, atol=0)
    assert orc.yarn_logit_gain(1.0) == 1.0


def test_yarn_regions_kept_interpolated_and_blended(orc):
    # r = 64, base 1e4, original context 4096: pair j turns 4096 * 1e4^(-j/32)
    # / 2pi times.  It keeps its frequency while that is >= 32 turns, i.e. for
    # j <= 8 log10(4096 / (64 pi)); it is divided by the factor once it is <= 1
    # turn, i.e. for j >= 8 log10(4096 / (2 pi)); between, the ratio falls
    # strictly from 1 to 1/factor.
    s = 16.0
    tab = orc.yarn_inv_freq(64, s, 32.0, 1.0, 4096)
    ratio = tab / 10000.0 ** (-np.arange(32) / 32.0)
    j_keep = math.floor(8 * math.log10(4096 / (64 * math.pi)))
    j_interp = math.ceil(8 * math.log10(4096 / (2 * math.pi)))
    assert 0 < j_keep < j_interp < 31
    assert np.allclose(ratio[: j_keep + 1], 1.0, rtol=1e-14, atol=0)
    assert np.allclose(ratio[j_interp:], 1.0 / s, rtol=1e-14, atol=0)
    mid = ratio[j_keep + 1: j_interp]
    assert ((mid < 1.0) & (mid > 1.0 / s)).all() and (np.diff(ratio[j_keep: j_interp + 1]) < 0).all()


def test_yarn_ramp_midpoint(orc):
    # An original context on which pair 5 turns exactly (32 + 1) / 2 times sits
    # half way up the ramp: its frequency is the mean of theta and theta / s.
    s, th5 = 16.0, 10000.0 ** (-10.0 / 64)
    L0 = 16.5 * 2 * math.pi / th5
    tab = orc.yarn_inv_freq(64, s, 32.0, 1.0, L0)
    assert math.isclose(tab[5], th5 * (1 + 1 / s) / 2, rel_tol=1e-13)


def test_yarn_logit_gain_factor_16(orc):
    # sqrt(1/t) = 1 + 0.1 ln 16 = 1 + 0.4 ln 2.
    assert math.isclose(orc.yarn_logit_gain(16.0), (1 + 0.4 * math.log(2.0)) ** 2, rel_tol=1e-15)


def test_frequency_table_reaches_compression_and_attention(orc):
    # m = 1: the stored entry of token t is RMSNorm(c_t) rotated by t * theta'_j
    # with the table's frequencies.
    B, L, d, r_dim = 1, 5, 32, 16
    r = rng(41)
    tab = orc.yarn_inv_freq(r_dim, 16.0, 32.0, 1.0, 64)
    tok = bf16_bits(r.standard_normal((B, L, d)))
    vals, _ = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(1), None, 1, 0, L, L,
                       rope_dim=r_dim, rope_freq=tab)
    x = orc.bf16_decode(tok)[0]
    nrm = x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + 1e-6)
    for t in range(L):
        assert np.allclose(vals[0, t], _rotate(nrm[t], float(t), r_dim, theta=tab),
                           rtol=1e-12, atol=1e-13)
    # Attention: shifting every position leaves the output unchanged under any
    # frequency table, and the table does change the output.
    B, Q, H, D, L, m, W, r_dim = 1, 1, 4, 64, 64, 4, 16, 32
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 43)
    kv_c[..., D - r_dim:] = 0
    tab = orc.yarn_inv_freq(r_dim, 16.0, 32.0, 1.0, 256)
    pos = np.array([[59]])
    sel = np.array([[[2, 6, 11]]], np.int32)
    cnt = np.array([[3]], np.int32)
    base, lb = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, r_dim, sel, cnt, rope_freq=tab)
    S = 4 * 777
    out, l2 = orc.mqa(q, pos + S, np.concatenate([np.zeros((B, 777, D), np.uint16), kv_c], 1),
                      np.concatenate([np.zeros((B, S, D), np.uint16), kv_tok], 1), sink, m, W,
                      r_dim, sel + 777, cnt, rope_freq=tab)
    assert np.allclose(out, base, rtol=1e-9, atol=1e-9) and np.allclose(l2, lb, rtol=1e-9, atol=1e-9)
    plain, _ = orc.mqa(q, pos, kv_c, kv_tok, sink, m, W, r_dim, sel, cnt)
    assert not np.allclose(plain, base, rtol=1e-6, atol=1e-6)


# --------------------------------- joint softmax over entries and window ---
def _rms(x, gamma=None, eps=1e-6):
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if gamma is None else y * gamma.astype(np.float64)


@pytest.mark.parametrize("r_dim", [0, 16])
def test_joint_softmax_over_entries_window_and_sink(orc, r_dim):
    # Selected compressed entries and window tokens share ONE softmax whose
    # denominator also holds e^z (the sink), and the output is rotated back
    # by the query position.  Written out here as textbook attention over the
    # concatenated key list [entries (as stored); RMSNorm'd, rotated window],
    # with the sink as one extra logit that has no value vector.
    B, Q, H, D, L, m, W = 1, 1, 4, 32, 64, 4, 9
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 51)
    sink = np.array([0.7, -1.5, 2.5, -0.2], np.float32)
    gq = (1 + 0.2 * rng(52).standard_normal(D)).astype(np.float32)
    gk = (1 + 0.2 * rng(53).standard_normal(D)).astype(np.float32)
    pos = 58  # n_vis = 14; window = tokens 50..58
    sel = np.array([[[2, 7, 11, 13, -1]]], np.int32)
    cnt = np.array([[4]], np.int32)
    out, lse = orc.mqa(q, np.array([[pos]]), kv_c, kv_tok, sink, m, W, r_dim, sel, cnt, gq, gk)

    ents = orc.bf16_decode(kv_c)[0, [2, 7, 11, 13]]
    toks = np.arange(pos - W + 1, pos + 1)
    win = _rms(orc.bf16_decode(kv_tok)[0, toks], gk)
    if r_dim:
        win = np.stack([_rotate(win[j], float(t), r_dim) for j, t in enumerate(toks)])
    keys = np.concatenate([ents, win], 0)  # K = V
    qh = _rms(orc.bf16_decode(q)[0, 0], gq)
    if r_dim:
        qh = _rotate(qh, float(pos), r_dim)
    logits = qh @ keys.T / math.sqrt(D)                       # [H, 4 + W]
    full = np.concatenate([logits, sink.astype(np.float64)[:, None]], 1)
    ref_lse = logsumexp(full, axis=1)
    p = np.exp(logits - ref_lse[:, None])                      # sink column dropped
    ref = p @ keys
    if r_dim:
        ref = _rotate(ref, -float(pos), r_dim)
    assert np.allclose(out[0, 0], ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0, 0], ref_lse, rtol=1e-13, atol=1e-13)
    # Two separate softmaxes (entries alone, window alone) averaged would be
    # a different number: the case does distinguish the readings.
    def branch(k):
        lg = qh @ k.T / math.sqrt(D)
        pw = np.exp(lg - lg.max(1, keepdims=True))
        return (pw / pw.sum(1, keepdims=True)) @ k
    assert not np.allclose(ref, 0.5 * (branch(ents) + branch(win)), rtol=1e-3, atol=1e-3)


def test_joint_softmax_without_sink_is_sdpa_over_concatenated_keys(orc):
    # Sink -inf, r = 0: plain scaled-dot-product attention (torch, fp64) over
    # the selected entries followed by the window tokens.
    B, Q, H, D, L, m, W = 1, 1, 8, 64, 96, 4, 16
    q, kv_tok, kv_c, sink = _mqa_case(B, Q, H, D, L, m, 54)
    sink[:] = -np.inf
    pos = 90  # n_vis = 22; window = tokens 75..90
    idx = [0, 5, 9, 17, 21]
    sel = np.array([[idx + [-1, -1, -1]]], np.int32)
    cnt = np.array([[len(idx)]], np.int32)
    out, lse = orc.mqa(q, np.array([[pos]]), kv_c, kv_tok, sink, m, W, 0, sel, cnt)
    ents = torch.from_numpy(orc.bf16_decode(kv_c)[0, idx])
    win = F.rms_norm(torch.from_numpy(orc.bf16_decode(kv_tok)[0, pos - W + 1: pos + 1]), (D,),
                     eps=1e-6)
    keys = torch.cat([ents, win], 0)
    qh = F.rms_norm(torch.from_numpy(orc.bf16_decode(q)[0, 0]), (D,), eps=1e-6)
    ref = F.scaled_dot_product_attention(qh[None], keys[None], keys[None])[0]
    assert np.allclose(out[0, 0], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(lse[0, 0], torch.logsumexp(qh @ keys.T / math.sqrt(D), 1).numpy(),
                       rtol=1e-13, atol=1e-13)


# -------------------------------------------- grouped output projection ---
def _gop_case(T, H, D, g, d_g, d, seed):
    r = rng(seed)
    o = bf16_bits(r.standard_normal((T, H, D)))
    w_g = bf16_bits(r.standard_normal((g, d_g, (H // g) * D)) / math.sqrt((H // g) * D))
    w_o = bf16_bits(r.standard_normal((d, g * d_g)) / math.sqrt(g * d_g))
    return o, w_g, w_o


def test_grouped_out_proj_matches_einsum(orc):
    # Group j reads heads j*H/g .. (j+1)*H/g - 1 (concatenated, head-major),
    # W_g[j] maps them to d_g values, W_o maps the concatenation to d.
    T, H, D, g, d_g, d = 3, 8, 16, 4, 8, 12
    o, w_g, w_o = _gop_case(T, H, D, g, d_g, d, 61)
    y, z = orc.grouped_out_proj(o, w_g, w_o, y_bf16=False)
    of = orc.bf16_decode(o).reshape(T, g, (H // g) * D)
    wg = orc.bf16_decode(w_g)
    wo = orc.bf16_decode(w_o)
    y_ref = np.einsum("tgk,gnk->tgn", of, wg).reshape(T, g * d_g)
    assert np.allclose(y, y_ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(z, y_ref @ wo.T, rtol=1e-12, atol=1e-12)
    # Another reading -- groups of interleaved heads (head h in group h % g) --
    # gives another result, so the grouping is pinned.
    inter = orc.bf16_decode(o).reshape(T, H // g, g, D).transpose(0, 2, 1, 3).reshape(T, g, -1)
    assert not np.allclose(y, np.einsum("tgk,gnk->tgn", inter, wg).reshape(T, -1), atol=1e-3)


def test_grouped_out_proj_single_group_is_two_matmuls(orc):
    T, H, D, g, d_g, d = 2, 4, 8, 1, 5, 7
    o, w_g, w_o = _gop_case(T, H, D, g, d_g, d, 62)
    _, z = orc.grouped_out_proj(o, w_g, w_o, y_bf16=False)
    x = torch.from_numpy(orc.bf16_decode(o).reshape(T, H * D))
    ref = (x @ torch.from_numpy(orc.bf16_decode(w_g)[0]).T) @ torch.from_numpy(orc.bf16_decode(w_o)).T
    assert np.allclose(z, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_grouped_out_proj_is_block_diagonal(orc):
    # The grouped first projection equals one dense projection whose weight is
    # block diagonal over the groups.
    T, H, D, g, d_g, d = 2, 6, 4, 3, 5, 4
    o, w_g, w_o = _gop_case(T, H, D, g, d_g, d, 63)
    y, _ = orc.grouped_out_proj(o, w_g, w_o, y_bf16=False)
    wg = orc.bf16_decode(w_g)
    k = (H // g) * D
    big = np.zeros((g * d_g, H * D))
    for j in range(g):
        big[j * d_g:(j + 1) * d_g, j * k:(j + 1) * k] = wg[j]
    assert np.allclose(y, orc.bf16_decode(o).reshape(T, H * D) @ big.T, rtol=1e-13, atol=1e-13)


def test_grouped_out_proj_selection_weights_are_exact(orc):
    # 0/1 weights that pick input c_j of group j, then the identity: y and z
    # are exactly those inputs.
    T, H, D, g, d_g = 2, 4, 8, 2, 3
    o, _, _ = _gop_case(T, H, D, g, d_g, 1, 64)
    k = (H // g) * D
    picks = [[0, 5, 15], [1, 8, 9]]
    w = np.zeros((g, d_g, k), np.float32)
    for j in range(g):
        for r, c in enumerate(picks[j]):
            w[j, r, c] = 1.0
    w_o = np.eye(g * d_g, dtype=np.float32)
    y, z = orc.grouped_out_proj(o, bf16_bits(w), bf16_bits(w_o))
    of = orc.bf16_decode(o).reshape(T, g, k)
    ref = np.stack([of[:, j, picks[j]] for j in range(g)], 1).reshape(T, -1)
    assert np.array_equal(y, ref) and np.array_equal(z, ref)


def test_grouped_out_proj_intermediate_storage_and_chaining(orc):
    T, H, D, g, d_g, d = 3, 8, 16, 4, 8, 12
    o, w_g, w_o = _gop_case(T, H, D, g, d_g, d, 65)
    y_exact, _ = orc.grouped_out_proj(o, w_g, w_o, y_bf16=False)
    y, z = orc.grouped_out_proj(o, w_g, w_o, y_bf16=True)
    # y is stored in bf16: a bf16 value within half a bf16 ulp of the exact y.
    assert np.array_equal(orc.bf16_decode(orc.bf16_encode(y)), y)
    assert np.all(np.abs(y - y_exact) <= np.abs(y_exact) * 2.0 ** -8)
    # Feeding that bf16 y as y_in gives the same z (the second projection alone).
    _, z2 = orc.grouped_out_proj(o, w_g, w_o, y_in=orc.bf16_encode(y))
    assert np.array_equal(z, z2)
    assert np.allclose(z, y @ orc.bf16_decode(w_o).T, rtol=1e-12, atol=1e-12)


# ------------------------------------------ overlapping compression (CSA) ---
def test_pool_overlap_zero_is_the_plain_pooling(orc):
    B, L, d, m = 1, 22, 16, 4
    tok = _tok(B, L, d, 71)
    r = rng(72)
    w_s = (0.3 * r.standard_normal(d)).astype(np.float32)
    b_pos = r.standard_normal(m).astype(np.float32)
    N = math.ceil(L / m)
    a, _ = orc.pool(tok, np.array([L]), w_s, b_pos, None, m, 0, N, N)
    b, _ = orc.pool(tok, np.array([L]), w_s, b_pos, None, m, 0, N, N, overlap=0)
    assert np.array_equal(a, b)


def test_pool_overlap_uniform_is_window_mean(orc):
    # Uniform weights: entry i is the mean of tokens max(0, i*m - ov) .. (i+1)*m - 1
    # (present ones): the window reaches back `ov` tokens into block i-1.
    B, L, d, m = 1, 23, 8, 4
    tok = _tok(B, L, d, 73)
    x = orc.bf16_decode(tok)[0]
    N = math.ceil(L / m)
    for ov in (1, 2, 4):
        vals, w = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(m + ov), None, m, 0, N, N,
                           normalize=False, overlap=ov)
        assert w[0].all()
        for i in range(N):
            lo, hi = max(0, i * m - ov), min(L, (i + 1) * m)
            assert np.allclose(vals[0, i], x[lo:hi].mean(0), rtol=0, atol=1e-15), (ov, i)


def test_pool_overlap_position_bias_addresses_the_window(orc):
    # A large bias at window position j selects token i*m - ov + j: position
    # 0 is the first borrowed token of block i-1, position ov the block's own
    # first token.  For block 0 the borrowed positions do not exist.
    B, L, d, m, ov = 1, 16, 8, 4, 4
    tok = _tok(B, L, d, 74)
    x = orc.bf16_decode(tok)[0]
    for j in (0, 2, 4, 7):
        b_pos = np.zeros(m + ov, np.float32)
        b_pos[j] = 90.0
        vals, _ = orc.pool(tok, np.array([L]), np.zeros(d), b_pos, None, m, 0, 4, 4,
                           normalize=False, overlap=ov)
        for i in range(1, 4):
            assert np.allclose(vals[0, i], x[i * m - ov + j], rtol=0, atol=1e-30), (j, i)
        if j >= ov:  # block 0: only its own tokens are present
            assert np.allclose(vals[0, 0], x[j - ov], rtol=0, atol=1e-30)
        else:        # the selected position is absent: uniform over tokens 0..3
            assert np.allclose(vals[0, 0], x[0:4].mean(0), rtol=0, atol=1e-15)


def test_pool_overlap_partial_newest_block(orc):
    # Context ends inside block i: the window is clipped at the context end too.
    B, L, d, m, ov = 1, 10, 8, 4, 4
    tok = _tok(B, 12, d, 75)
    x = orc.bf16_decode(tok)[0]
    vals, w = orc.pool(tok, np.array([L]), np.zeros(d), np.zeros(m + ov), None, m, 0, 3, 3,
                       normalize=False, overlap=ov)
    assert w[0].tolist() == [True, True, True]
    assert np.allclose(vals[0, 2], x[4:10].mean(0), rtol=0, atol=1e-15)
