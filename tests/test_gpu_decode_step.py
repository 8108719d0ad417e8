"""GPU parity of the decode loop: csa_decode_step / hca_decode_step called for
consecutive positions, each sequence at its own position, against the fp64
oracle through the C ABI.

The caches start with the blocks the oracle compresses from the tokens
before each sequence's first step, so no oracle input comes from the GPU.
Every step is checked layer by layer: the newest block of every sequence
against the oracle's compression of the tokens up to its position; scores
against the oracle fed the GPU's E4M3 keys; the top-k bit-exact against the
oracle ranking the GPU's scores; attention against the oracle fed the GPU's
selection and cache.  After the loop the whole cache is checked."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_kv_04_b200 import binding, configs, synth
from gpuhelp import (assert_attention_close, assert_bf16_storage_close, assert_lse_close, bits8,
                     bits16, f32)
from test_gpu_compress_index import check_keys

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.lib()


def _to_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def _check_lse(lse, rlse, ref):
    assert_lse_close(f32(lse), rlse, ref, "decode-step LSE")


@pytest.mark.parametrize("overlap", [0, 4])
def test_csa_decode_loop(orc, overlap):
    """Three sequences at positions 301, 514 and 127, six steps each: blocks
    complete mid-loop (at 303, 515/519, 127/131), and the third sequence
    starts with fewer visible entries (32) than k (64).  overlap = 4: the
    newest entry also pools the previous block's tokens."""
    w = configs.scaled(configs.CSA_128K, B=3, k=64, L=2048, overlap=overlap)
    B, m, L_cap = w.B, w.m, 2048
    N_cap = L_cap // m
    start = np.array([301, 514, 127])
    kv_tok, idx_tok = synth.token_streams(w, L_cap=L_cap, device=DEV)
    kv_bits, idx_bits = bits16(kv_tok), bits16(idx_tok)
    w_s, b_pos = synth.pool_params(w, DEV)
    w_si, b_pi = synth.pool_params(w, DEV, indexer=True)
    kv_c0, _, _ = orc.compress_kv(kv_bits, start, f32(w_s), f32(b_pos), None, m, 0, N_cap, N_cap,
                                  rope_dim=w.rope_dim, overlap=w.overlap)
    key0, ks0, _, _ = orc.compress_index(idx_bits, start, f32(w_si), f32(b_pi), m, 0, N_cap, N_cap,
                                         overlap=w.overlap)
    kv_c = _to_bf16(kv_c0)
    idx_key = torch.from_numpy(key0).to(DEV)
    idx_scale = torch.from_numpy(ks0).to(DEV)
    p = binding.params_for(w, B=B)
    ws = binding.workspace(p, binding.OP_CSA_DECODE_STEP, 1, N_cap)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for step in range(6):
        pos = start + step
        qi = synth.queries(configs.scaled(w, seed=w.seed + 100 + step), Q=1, device=DEV)
        q = qi["q"][:, 0].contiguous()
        out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
        lse = torch.full((B, w.H), float("nan"), dtype=torch.float32, device=DEV)
        tidx = torch.full((B, w.k), -7, dtype=torch.int32, device=DEV)
        tcnt = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        ws.fill_(0xFF)  # unwritten scores read as NaN
        pos_t = torch.from_numpy(pos).to(DEV)
        binding.csa_decode_step(p, pos_t, kv_tok, idx_tok, w_s, b_pos, None, w_si, b_pi, kv_c,
                                idx_key, idx_scale, q, qi["q_idx"][:, 0].contiguous(),
                                qi["q_scale"][:, 0].contiguous(), qi["w"][:, 0].contiguous(),
                                qi["sink"], tidx, tcnt, out, lse=lse, ws=ws, dev_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, status.item()
        # 1. Each sequence's newest block (pooled over tokens up to pos).
        got_c, got_k, got_s = bits16(kv_c), bits8(idx_key), f32(idx_scale)
        for b in range(B):
            i = pos[b] // m
            _, _, vals = orc.compress_kv(kv_bits[b: b + 1], [pos[b] + 1], f32(w_s), f32(b_pos),
                                         None, m, i, 1, N_cap, rope_dim=w.rope_dim, overlap=w.overlap)
            assert_bf16_storage_close(got_c[b: b + 1, i], vals[:, i], f"step {step} seq {b} entry")
            _, _, kvals, _ = orc.compress_index(idx_bits[b: b + 1], [pos[b] + 1], f32(w_si),
                                                f32(b_pi), m, i, 1, N_cap, overlap=w.overlap)
            check_keys(orc, got_k[b: b + 1, i], got_s[b: b + 1, i], kvals[:, i],
                       f"step {step} seq {b} key")
        # 2. Scores of the visible entries against the oracle on the GPU's keys.
        nv = (pos + 1) // m
        scores = f32(ws[: B * N_cap * 4].view(torch.float32).view(B, N_cap)).astype(np.float64)
        ref = orc.index_scores(bits8(qi["q_idx"]), f32(qi["q_scale"]), f32(qi["w"]), got_k, got_s,
                               pos.reshape(B, 1), m)[:, 0]
        for b in range(B):
            g, r = scores[b, : nv[b]], ref[b, : nv[b]]
            assert np.allclose(g, r, rtol=2e-5, atol=1e-6 * np.abs(r).mean()), (step, b)
        # 3. Top-k bit-exact on the GPU's scores.
        gs = np.where(np.isnan(scores), -np.inf, scores)
        ridx, rcnt = orc.topk(gs, nv, w.k)
        assert np.array_equal(tcnt.cpu().numpy(), rcnt), step
        assert np.array_equal(tidx.cpu().numpy(), ridx), step
        # 4. Attention with the GPU's selection and cache.
        ro, rl = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), pos.reshape(B, 1), got_c, kv_bits,
                         f32(qi["sink"]), m, w.W, w.rope_dim, tidx.cpu().numpy()[:, None],
                         tcnt.cpu().numpy()[:, None])
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert_attention_close(got, ro[:, 0], f"step {step}")
        _check_lse(lse, rl[:, 0], ro[:, 0])
    # The whole cache after the loop: every block of tokens up to the last
    # position, the partial newest one included.
    last = start + 5
    _, _, vals = orc.compress_kv(kv_bits, last + 1, f32(w_s), f32(b_pos), None, m, 0, N_cap, N_cap,
                                 rope_dim=w.rope_dim, overlap=w.overlap)
    got_c = bits16(kv_c)
    for b in range(B):
        n = last[b] // m + 1
        assert_bf16_storage_close(got_c[b, :n], vals[b, :n], f"seq {b} cache")


def test_hca_decode_loop(orc):
    """Two sequences at positions 125 and 640, six steps each: the first
    block of the first sequence completes at 127 (its first visible entry)."""
    w = configs.scaled(configs.HCA_1M, B=2, L=1536)
    B, m, L_cap = w.B, w.m, 1536
    N_cap = L_cap // m
    start = np.array([125, 640])
    kv_tok, _ = synth.token_streams(w, L_cap=L_cap, device=DEV)
    kv_bits = bits16(kv_tok)
    w_s, b_pos = synth.pool_params(w, DEV)
    kv_c0, _, _ = orc.compress_kv(kv_bits, start, f32(w_s), f32(b_pos), None, m, 0, N_cap, N_cap,
                                  rope_dim=w.rope_dim)
    kv_c = _to_bf16(kv_c0)
    p = binding.params_for(w, B=B)
    ws = binding.workspace(p, binding.OP_HCA_DECODE_STEP, 1, N_cap)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for step in range(6):
        pos = start + step
        qi = synth.queries(configs.scaled(w, seed=w.seed + 100 + step), Q=1, device=DEV)
        q = qi["q"][:, 0].contiguous()
        out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
        lse = torch.full((B, w.H), float("nan"), dtype=torch.float32, device=DEV)
        binding.hca_decode_step(p, torch.from_numpy(pos).to(DEV), kv_tok, w_s, b_pos, None, kv_c,
                                q, qi["sink"], out, lse=lse, ws=ws, dev_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, status.item()
        got_c = bits16(kv_c)
        for b in range(B):
            i = pos[b] // m
            _, _, vals = orc.compress_kv(kv_bits[b: b + 1], [pos[b] + 1], f32(w_s), f32(b_pos),
                                         None, m, i, 1, N_cap, rope_dim=w.rope_dim)
            assert_bf16_storage_close(got_c[b: b + 1, i], vals[:, i], f"step {step} seq {b} entry")
        ro, rl = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), pos.reshape(B, 1), got_c, kv_bits,
                         f32(qi["sink"]), m, w.W, w.rope_dim)
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert_attention_close(got, ro[:, 0], f"HCA step {step}")
        _check_lse(lse, rl[:, 0], ro[:, 0])


# ----------------------------------------------------------------------------
# The histogram-seeded top-k of the decode step (a few long rows: one cluster
# of CTAs per row).  The workspace holds the scores [B, N_cap] fp32 from byte
# 0, then the score histogram [B, 4096] u32 and one path word per sequence
# (0 every visible entry kept, 1 histogram path, 2 full radix select).

def _ws_layout(B, N_cap):
    sb = (B * N_cap * 4 + 255) // 256 * 256
    return sb, sb + B * 4096 * 4


def _hist_and_path(ws, B, N_cap):
    h0, p0 = _ws_layout(B, N_cap)
    hist = ws[h0:p0].view(torch.int32).view(B, 4096).cpu().numpy()
    path = ws[p0:p0 + 4 * B].view(torch.int32).cpu().numpy()
    return hist, path


class _Step:
    """A decode step over caches compressed from random token streams (the
    construction of the timed workload), or over given caches."""

    def __init__(self, w, L_cap, seed=0):
        w = configs.scaled(w, seed=w.seed + seed)
        self.w, self.B, self.N = w, w.B, L_cap // w.m
        B, d = w.B, w.d
        self.kv_tok, self.idx_tok = synth.token_streams(w, L_cap=L_cap, device=DEV)
        self.w_s, self.b_pos = synth.pool_params(w, DEV)
        self.w_si, self.b_pi = synth.pool_params(w, DEV, indexer=True)
        self.p = binding.params_for(w, B=B)
        self.kv_c = torch.zeros(B, self.N, d, dtype=torch.bfloat16, device=DEV)
        self.key = torch.zeros(B, self.N, w.D_I, dtype=torch.uint8, device=DEV)
        self.ksc = torch.zeros(B, self.N, dtype=torch.float32, device=DEV)
        self.ws = binding.workspace(self.p, binding.OP_CSA_DECODE_STEP, 1, self.N)
        self.status = torch.zeros(1, dtype=torch.int32, device=DEV)

    def compress_all(self, L):
        ctx = torch.full((self.B,), L, dtype=torch.int64, device=DEV)
        binding.csa_compress(self.p, self.kv_tok, ctx, self.w_s, self.b_pos, None, 0, self.N,
                             self.kv_c, self.idx_tok, self.w_si, self.b_pi, self.key, self.ksc,
                             dev_status=self.status)

    def run(self, pos, qseed):
        w, B = self.w, self.B
        qi = synth.queries(configs.scaled(w, seed=qseed), Q=1, device=DEV)
        out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
        lse = torch.full((B, w.H), float("nan"), dtype=torch.float32, device=DEV)
        tidx = torch.full((B, w.k), -7, dtype=torch.int32, device=DEV)
        tcnt = torch.full((B,), -7, dtype=torch.int32, device=DEV)
        pos_t = torch.as_tensor(pos, dtype=torch.int64, device=DEV)
        binding.csa_decode_step(self.p, pos_t, self.kv_tok, self.idx_tok, self.w_s, self.b_pos,
                                None, self.w_si, self.b_pi, self.kv_c, self.key, self.ksc,
                                qi["q"][:, 0].contiguous(), qi["q_idx"][:, 0].contiguous(),
                                qi["q_scale"][:, 0].contiguous(), qi["w"][:, 0].contiguous(),
                                qi["sink"], tidx, tcnt, out, lse=lse, ws=self.ws,
                                dev_status=self.status)
        torch.cuda.synchronize()
        assert self.status.item() == 0, self.status.item()
        self.out, self.lse = out, lse
        return qi, tidx, tcnt

    def check(self, orc, pos, qi, tidx, tcnt, path_expect, n_sample=256):
        """Scores (sampled) against the oracle on the GPU's keys; the top-k
        bit-exact against the oracle ranking the GPU's scores; the path
        taken; the histogram cleared."""
        w, B, N = self.w, self.B, self.N
        pos = np.asarray(pos)
        nv = (pos + 1) // w.m
        scores = self.ws[: B * N * 4].view(torch.float32).view(B, N).cpu().numpy().astype(np.float64)
        keys, ks = bits8(self.key), f32(self.ksc)
        rng = np.random.default_rng(int(pos.sum()))
        for b in range(B):
            smp = np.union1d(rng.choice(nv[b], min(n_sample, nv[b]), replace=False),
                             [0, nv[b] - 1])
            ref = orc.index_scores(bits8(qi["q_idx"][b: b + 1]), f32(qi["q_scale"][b: b + 1]),
                                   f32(qi["w"][b: b + 1]), keys[b: b + 1, smp], ks[b: b + 1, smp],
                                   np.array([[len(smp) * w.m - 1]]), w.m)[0, 0]
            g = scores[b, smp]
            assert np.allclose(g, ref, rtol=2e-5, atol=1e-6 * np.abs(ref).mean()), b
        gs = np.full((B, N), -np.inf)
        for b in range(B):
            gs[b, : nv[b]] = scores[b, : nv[b]]
        ridx, rcnt = orc.topk(gs, nv, w.k)
        assert np.array_equal(tcnt.cpu().numpy(), rcnt)
        assert np.array_equal(tidx.cpu().numpy(), ridx)
        hist, path = _hist_and_path(self.ws, B, N)
        assert not hist.any(), "histogram not cleared"
        assert path.tolist() == list(path_expect), path

    def check_attention(self, orc, pos, qi, tidx, tcnt):
        """The step's attention output and LSE against the oracle fed the
        GPU's selection and cache (the window tail of the token stream)."""
        w, B = self.w, self.B
        pos = np.asarray(pos)
        lo = int(pos.min()) - w.W + 1
        hi = int(pos.max()) + 1
        tail = bits16(self.kv_tok[:, lo:hi])
        q = qi["q"][:, 0].contiguous()
        kw = {}
        if w.yarn:  # the oracle's own YaRN table and logit gain
            kw = dict(rope_freq=orc.yarn_inv_freq(w.rope_dim, *w.yarn),
                      scale=orc.yarn_logit_gain(w.yarn[0]) / math.sqrt(w.d))
        ro, rl = orc.mqa(bits16(q).reshape(B, 1, w.H, w.D), pos.reshape(B, 1), bits16(self.kv_c),
                         tail, f32(qi["sink"]), w.m, w.W, w.rope_dim, tidx.cpu().numpy()[:, None],
                         tcnt.cpu().numpy()[:, None], tok_base=lo, **kw)
        got = self.out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert_attention_close(got, ro[:, 0], "decode step, Qhat from the top-k")
        if w.yarn:
            assert_lse_close(f32(self.lse), rl[:, 0], ro[:, 0], "decode-step LSE", kw["scale"])
        else:
            _check_lse(self.lse, rl[:, 0], ro[:, 0])


def test_histogram_topk_csa_128k_shape(orc):
    """The timed 128K workload (8 sequences x 32768 entries, k = 1024):
    every row takes the histogram path, on a fresh workspace and on the one
    the previous step left.  The indexer adds its counts to what the
    workspace holds: N spurious counts in the top bin (keys no finite score
    has) make that bin the guess, which the keys' own counts refute, so every
    row takes the full select, with the same result; counts below the
    threshold change nothing."""
    w = configs.CSA_128K
    st = _Step(w, w.L, seed=1)
    st.compress_all(w.L)
    pos = np.full(w.B, w.L - 1)
    for step in range(2):
        qi, tidx, tcnt = st.run(pos, w.seed + 1000 + step)
        st.check(orc, pos, qi, tidx, tcnt, [1] * w.B)
        if step == 0:
            st.check_attention(orc, pos, qi, tidx, tcnt)
    h0, _ = _ws_layout(w.B, st.N)
    for top_bin, path in ((4095, 2), (0, 1)):
        bad = torch.zeros(w.B, 4096, dtype=torch.int32, device=DEV)
        bad[:, top_bin] = st.N
        st.ws[h0: h0 + bad.numel() * 4].copy_(bad.view(-1).view(torch.uint8))
        qi, tidx, tcnt = st.run(pos, w.seed + 1002 + top_bin)
        st.check(orc, pos, qi, tidx, tcnt, [path] * w.B)


def test_histogram_topk_csa_1m_shape(orc):
    """The timed 1M workload (4 sequences x 262144 entries, 16-CTA clusters
    of 256 candidate slots each): the histogram path, bit-exact."""
    w = configs.CSA_1M
    st = _Step(w, w.L, seed=2)
    st.compress_all(w.L)
    pos = np.full(w.B, w.L - 1)
    qi, tidx, tcnt = st.run(pos, w.seed + 1000)
    st.check(orc, pos, qi, tidx, tcnt, [1] * w.B)
    st.check_attention(orc, pos, qi, tidx, tcnt)


@pytest.mark.parametrize("case", ["ties", "all_equal", "few_visible", "recent_block"])
def test_histogram_topk_structures(orc, case):
    """Two sequences x 16384 entries, k = 512 (4-CTA clusters, 1024 slots):
    ties: one key row for every entry and 64 key scales, so scores take 64
    values and the threshold bin holds 8 of them (the tie rule across CTAs);
    all_equal: one score everywhere, more candidates than slots (the full
    select, lowest indices); few_visible: one sequence with fewer visible
    entries than k next to one on the histogram path; recent_block: the 600
    highest scores on the last 600 entries (each warp chunk there holds more
    keys at or above the threshold bin than its position list: the emission
    over the whole slice, on the histogram path)."""
    w = configs.scaled(configs.CSA_128K, B=2, k=512, L=65536)
    st = _Step(w, w.L, seed=5)
    N = st.N
    row = synth.e4m3_codes((1, 1, w.D_I), 6, "q_idx", DEV)
    st.key.copy_(row.expand(w.B, N, w.D_I))
    if case == "recent_block":
        # The sign of each sequence's score for this key row (its query and
        # head weights), so that the block holds the largest scores.
        qi0 = synth.queries(configs.scaled(st.w, seed=w.seed + 1000), Q=1, device=DEV)
        t = torch.arange(N, device=DEV, dtype=torch.float32)
        blk = (t - (N - 600)).clamp(min=0) / 600
        for b in range(w.B):
            c = orc.index_scores(bits8(qi0["q_idx"][b: b + 1]), f32(qi0["q_scale"][b: b + 1]),
                                 f32(qi0["w"][b: b + 1]), bits8(row), np.ones((1, 1)),
                                 np.array([[w.m - 1]]), w.m)[0, 0][0]
            assert c != 0
            base = (1 + t / N) / 64
            top = (4 + 3.9 * blk) / 64 if c > 0 else (0.49 - 0.24 * blk) / 64
            st.ksc[b].copy_(torch.where(t >= N - 600, top, base))
    elif case == "ties":
        vals = 1.0 + torch.arange(64, device=DEV, dtype=torch.float32) / 64
        rng = torch.Generator(device=DEV).manual_seed(7)
        st.ksc.copy_(vals[torch.randint(0, 64, (w.B, N), generator=rng, device=DEV)] / 64)
    else:
        st.ksc.fill_(1.0 / 64)
    pos = np.full(w.B, w.L - 1)
    expect = [1, 1] if case in ("ties", "recent_block") else [2, 2]
    if case == "few_visible":
        pos[0] = 4 * 400 - 1
        expect = [0, 2]
    qi, tidx, tcnt = st.run(pos, w.seed + 1000)
    st.check(orc, pos, qi, tidx, tcnt, expect)
    st.check_attention(orc, pos, qi, tidx, tcnt)


def test_histogram_topk_flash_yarn(orc):
    """V4-Flash shapes through the decode step ("DeepSeek V4-Pro" (llm-arch-kb),
    "Family": 64 heads, top-512; YaRN RoPE): two sequences x 16384 entries at
    different positions, on the histogram path, with the attention's Qhat
    formed by the top-k kernel (one attention CTA per row and split)."""
    w = configs.scaled(configs.CSA_FLASH_128K, B=2, L=65536)
    st = _Step(w, w.L, seed=9)
    st.compress_all(w.L)
    pos = np.array([w.L - 1, w.L - 1 - 37])
    qi, tidx, tcnt = st.run(pos, w.seed + 1000)
    st.check(orc, pos, qi, tidx, tcnt, [1, 1])
    st.check_attention(orc, pos, qi, tidx, tcnt)


def test_prepared_decode_steps_match_the_plain_calls():
    """binding.CsaDecodeStep / HcaDecodeStep (the unchanging arguments
    converted once), called per step or bound to the step's buffers, run the
    same C entry points: the same outputs, bit for bit, as csa_decode_step /
    hca_decode_step."""
    for csa in (True, False):
        w = configs.scaled(configs.CSA_128K if csa else configs.HCA_1M, B=2, L=4096)
        p = binding.params_for(w)
        kv_tok, idx_tok = synth.token_streams(w, device=DEV)
        w_s, b_pos = synth.pool_params(w, DEV)
        N = w.L // w.m
        kv_c = torch.zeros(w.B, N, w.d, dtype=torch.bfloat16, device=DEV)
        qi = synth.queries(w, Q=1, device=DEV)
        q = qi["q"][:, 0].contiguous()
        pos = torch.tensor([w.L - 1, w.L - 7], dtype=torch.int64, device=DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        outs = []
        if csa:
            w_si, b_pi = synth.pool_params(w, DEV, indexer=True)
            key = torch.zeros(w.B, N, w.D_I, dtype=torch.uint8, device=DEV)
            ksc = torch.zeros(w.B, N, dtype=torch.float32, device=DEV)
            ctx = torch.full((w.B,), w.L, dtype=torch.int64, device=DEV)
            binding.csa_compress(p, kv_tok, ctx, w_s, b_pos, None, 0, N, kv_c, idx_tok, w_si, b_pi,
                                 key, ksc, dev_status=status)
            ws = binding.workspace(p, binding.OP_CSA_DECODE_STEP, 1, N)
            args = (q, qi["q_idx"][:, 0].contiguous(), qi["q_scale"][:, 0].contiguous(),
                    qi["w"][:, 0].contiguous())
            tidx = torch.zeros(w.B, w.k, dtype=torch.int32, device=DEV)
            tcnt = torch.zeros(w.B, dtype=torch.int32, device=DEV)
            for mode in ("plain", "prepared", "bound"):
                out = torch.full((w.B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
                lse = torch.full((w.B, w.H), float("nan"), dtype=torch.float32, device=DEV)
                if mode != "plain":
                    f = binding.CsaDecodeStep(p, kv_tok, idx_tok, w_s, b_pos, None, w_si, b_pi,
                                              kv_c, key, ksc, qi["sink"], tidx, tcnt, ws,
                                              dev_status=status)
                    if mode == "bound":
                        f.bind(pos, *args, out, lse=lse)()
                    else:
                        f(pos, *args, out, lse=lse)
                else:
                    binding.csa_decode_step(p, pos, kv_tok, idx_tok, w_s, b_pos, None, w_si, b_pi,
                                            kv_c, key, ksc, *args, qi["sink"], tidx, tcnt, out,
                                            lse=lse, ws=ws, dev_status=status)
                torch.cuda.synchronize()
                outs.append((out.clone(), lse.clone(), tidx.clone()))
        else:
            ctx = torch.full((w.B,), w.L, dtype=torch.int64, device=DEV)
            binding.hca_compress(p, kv_tok, ctx, w_s, b_pos, None, 0, N, kv_c, dev_status=status)
            ws = binding.workspace(p, binding.OP_HCA_DECODE_STEP, 1, N)
            for mode in ("plain", "prepared", "bound"):
                out = torch.full((w.B, w.H, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
                lse = torch.full((w.B, w.H), float("nan"), dtype=torch.float32, device=DEV)
                if mode != "plain":
                    f = binding.HcaDecodeStep(p, kv_tok, w_s, b_pos, None, kv_c, qi["sink"], ws,
                                              dev_status=status)
                    if mode == "bound":
                        f.bind(pos, q, out, lse=lse)()
                    else:
                        f(pos, q, out, lse=lse)
                else:
                    binding.hca_decode_step(p, pos, kv_tok, w_s, b_pos, None, kv_c, q, qi["sink"],
                                            out, lse=lse, ws=ws, dev_status=status)
                torch.cuda.synchronize()
                outs.append((out.clone(), lse.clone(), None))
        assert status.item() == 0
        o0, l0, t0 = outs[0]
        assert torch.isfinite(o0.float()).all()
        for o1, l1, t1 in outs[1:]:
            assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
            assert torch.equal(l0, l1)
            if csa:
                assert torch.equal(t0, t1)


def test_decode_step_newest_entries_match_compress():
    """The decode step's newest entry of each sequence (KV row, indexer key
    and scale) has the same bits as csa_compress over the same tokens.
    Positions: a complete block, a partial one, and a partial block that
    opens an indexer tile past the visible ones."""
    w = configs.scaled(configs.CSA_128K, B=3, L=8192)
    st = _Step(w, w.L, seed=13)
    st.compress_all(w.L)
    pos = np.array([w.L - 1, w.L - 3, 4096])
    st.run(pos, w.seed + 1000)
    N = st.N
    kv_c = torch.zeros_like(st.kv_c)
    key = torch.zeros_like(st.key)
    ksc = torch.zeros_like(st.ksc)
    ctx = torch.from_numpy(pos + 1).to(DEV)
    binding.csa_compress(st.p, st.kv_tok, ctx, st.w_s, st.b_pos, None, 0, N, kv_c, st.idx_tok,
                         st.w_si, st.b_pi, key, ksc, dev_status=st.status)
    torch.cuda.synchronize()
    assert st.status.item() == 0
    for b in range(w.B):
        i = int(pos[b]) // w.m
        assert torch.equal(st.kv_c[b, i].view(torch.int16), kv_c[b, i].view(torch.int16)), b
        assert torch.equal(st.key[b, i], key[b, i]), b
        assert torch.equal(st.ksc[b, i], ksc[b, i]), b


def test_prepared_copies_round_trip():
    """binding.PreparedCopy (csa_copy_async / csa_copy_rows_async): pinned
    host rows into one strided row per sequence of a device token buffer, a
    contiguous upload, and a download, each on its own stream; every byte
    arrives and no other byte of the buffer changes."""
    g = torch.Generator().manual_seed(5)
    B, L_cap, d = 3, 37, 512
    buf = torch.randn(B, L_cap, d, generator=g).to(torch.bfloat16).to(DEV)
    before = buf.clone()
    rows = torch.randn(B, 1, d, generator=g).to(torch.bfloat16).pin_memory()
    flat = torch.randint(0, 256, (4099,), dtype=torch.uint8, generator=g).pin_memory()
    dflat = torch.zeros(4099, dtype=torch.uint8, device=DEV)
    back = torch.zeros(B, L_cap, d, dtype=torch.bfloat16).pin_memory()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    c_rows = binding.PreparedCopy(buf[:, 11:12], rows, up)
    c_flat = binding.PreparedCopy(dflat, flat, up)
    c_back = binding.PreparedCopy(back, buf, down)
    assert c_rows.bytes == B * d * 2 and c_flat.bytes == 4099
    c_rows()
    c_flat()
    down.wait_stream(up)
    c_back()
    torch.cuda.synchronize()
    want = before.clone()
    want[:, 11:12] = rows.to(DEV)
    assert torch.equal(buf.view(torch.int16), want.view(torch.int16))
    assert torch.equal(back.view(torch.int16), want.cpu().view(torch.int16))
    assert torch.equal(dflat.cpu(), flat)


def test_histogram_topk_single_sequence(orc):
    """One sequence x 16384 entries, k = 512: the widest top-k cluster per row
    and one indexer chunk per tile; the histogram path, bit-exact, with the
    step's attention against the oracle."""
    w = configs.scaled(configs.CSA_128K, B=1, k=512, L=65536)
    st = _Step(w, w.L, seed=11)
    st.compress_all(w.L)
    pos = np.array([w.L - 2])
    qi, tidx, tcnt = st.run(pos, w.seed + 1000)
    st.check(orc, pos, qi, tidx, tcnt, [1])
    st.check_attention(orc, pos, qi, tidx, tcnt)
