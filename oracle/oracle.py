"""Python face of the fp64 CPU oracle (TEST INFRASTRUCTURE ONLY).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg
import this module.  It marshals numpy arrays into oracle/liboracle.so and
composes the oracle's steps in the order the source pages give them:

  CSA layer ([P2] steps 1-3, [P5] "Hybrid attention"): compress (m=4),
      Lightning-Indexer scores, top-k, shared-KV MQA with window and sink.
  HCA layer ([P2] HCA, [P5] "Hybrid attention"): compress (m'=128), dense
      shared-KV MQA with window and sink.

Storage contract mirrored from the library: compressed KV entries and the
attention output are stored as bfloat16; indexer keys as E4M3 codes with one
binary32 scale per row.  Nothing else is rounded.

Inputs are numpy arrays holding the raw storage bits: bfloat16 as uint16,
E4M3 as uint8, binary32 as float32, positions and lengths as int64.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import numpy as np

from . import build_oracle

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build_oracle.build())
        _declare(_lib)
    return _lib


def _p(a, ct):
    if a is None:
        return None
    return a.ctypes.data_as(C.POINTER(ct))


def _declare(L):
    i32, i64, f64, f32 = C.c_int, C.c_int64, C.c_double, C.c_float
    P = C.POINTER
    L.orc_abi_version.restype = i32
    L.orc_bf16_decode.argtypes = [C.c_uint16]
    L.orc_bf16_decode.restype = f64
    L.orc_bf16_encode.argtypes = [f64]
    L.orc_bf16_encode.restype = C.c_uint16
    L.orc_e4m3_decode.argtypes = [C.c_uint8]
    L.orc_e4m3_decode.restype = f64
    L.orc_e4m3_encode.argtypes = [f32]
    L.orc_e4m3_encode.restype = C.c_uint8
    L.orc_bf16_encode_array.argtypes = [i64, P(f64), P(C.c_uint16)]
    L.orc_pool.argtypes = [i32, i64, i32, i32, i32, P(C.c_uint16), P(i64), P(f32), P(f32),
                           P(f32), f64, i32, i32, f64, P(f64), i64, i64, i64, P(f64),
                           P(C.c_uint8), i32]
    L.orc_quant_rows_e4m3.argtypes = [i64, i32, P(f64), P(C.c_uint8), P(f32)]
    L.orc_index_scores.argtypes = [i32, i32, i32, i32, i32, P(C.c_uint8), P(f32), P(f32),
                                   P(C.c_uint8), P(f32), i64, P(i64), P(f64), i32]
    L.orc_topk.argtypes = [i64, i64, P(f64), P(i64), i32, P(C.c_int32), P(C.c_int32), i32]
    L.orc_mqa.argtypes = [i32, i32, i32, i32, i32, i32, i32, f64, P(f64), P(C.c_uint16), P(i64),
                          P(C.c_uint16), i64, P(C.c_int32), P(C.c_int32), i32, P(C.c_uint16),
                          i64, i64, P(f32), P(f32), P(f32), f64, f64, P(f64), P(f64), i32]
    L.orc_grouped_out_proj.argtypes = [i64, i32, i32, i32, i32, i32, P(C.c_uint16),
                                       P(C.c_uint16), P(C.c_uint16), i32, P(C.c_uint16),
                                       P(f64), P(f64), i32]


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ------------------------------------------------------------------ formats --
def bf16_decode(u16: np.ndarray) -> np.ndarray:
    u = _c(u16, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_encode(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_encode_array(x.size, _p(x, C.c_double), _p(out, C.c_uint16))
    return out


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    lut = np.array([lib().orc_e4m3_decode(c) for c in range(256)], np.float64)
    return lut[_c(codes, np.uint8)]


def e4m3_encode_scalar(x: float) -> int:
    return int(lib().orc_e4m3_encode(float(np.float32(x))))


# ------------------------------------------------- RoPE frequency tables --
def rope_inv_freq(rope_dim, base=10000.0):
    """Plain RoPE frequencies theta_j = base^(-2j/r), j < r/2."""
    j = np.arange(rope_dim // 2, dtype=np.float64)
    return base ** (-2.0 * j / rope_dim)


def yarn_inv_freq(rope_dim, factor, beta_fast, beta_slow, original_len, base=10000.0):
    """YaRN context-extension frequencies (the DeepSeek-V4 pages' training
    section: YaRN with factor 16, beta_fast 32 and beta_slow 1 extends the
    context to 1,048,576 tokens), following the published method (Peng et
    al., "YaRN: Efficient Context Window Extension of Large Language Models",
    2023, the "NTK-by-parts" interpolation):

      theta_j   = base^(-2j/r)                  plain frequency of pair j
      rot_j     = original_len * theta_j / 2pi  full turns of pair j over the
                                                original context
      gamma_j   = clamp((rot_j - beta_slow) / (beta_fast - beta_slow), 0, 1)
      theta'_j  = gamma_j * theta_j + (1 - gamma_j) * theta_j / factor

    Pairs that turn many times over the original context keep their
    frequency; pairs that turn less than once are interpolated by `factor`;
    the ones between are blended linearly in rot_j."""
    theta = rope_inv_freq(rope_dim, base)
    rot = original_len * theta / (2.0 * math.pi)
    g = np.clip((rot - beta_slow) / (beta_fast - beta_slow), 0.0, 1.0)
    return g * theta + (1.0 - g) * theta / factor


def yarn_logit_gain(factor):
    """YaRN attention temperature: q and k are both scaled by
    sqrt(1/t) = 0.1 ln(factor) + 1 (same paper), i.e. the logits by its square."""
    return (0.1 * math.log(factor) + 1.0) ** 2


# -------------------------------------------------------------------- steps --
def _freq(rope_freq, rope_dim):
    if rope_freq is None:
        return None
    f = _c(rope_freq, np.float64)
    if f.shape != (rope_dim // 2,):
        raise ValueError(f"rope_freq must hold rope_dim/2 = {rope_dim // 2} values")
    return f


def pool(tok, ctx_len, w_s, b_pos, gamma, m, first_block, n_blocks, N_cap, eps=1e-6,
         normalize=True, nthreads=0, rope_dim=0, rope_base=10000.0, rope_freq=None, overlap=0):
    """Compression step (a1) in fp64.  Returns (values[B,N_cap,d], written[B,N_cap]).
    rope_dim > 0: each entry is stored rotated to its position (i+1)*m - 1.
    rope_freq [rope_dim/2] replaces the frequencies rope_base^(-2j/rope_dim).
    overlap > 0: entry i pools tokens i*m - overlap .. (i+1)*m - 1 (b_pos has
    m + overlap values)."""
    rope_freq = _freq(rope_freq, rope_dim)
    tok = _c(tok, np.uint16)
    B, L_cap, d = tok.shape
    ctx_len = _c(ctx_len, np.int64)
    if len(np.ravel(b_pos)) != m + overlap:
        raise ValueError("b_pos must hold m + overlap values")
    out = np.zeros((B, N_cap, d), np.float64)
    written = np.zeros((B, N_cap), np.uint8)
    lib().orc_pool(B, L_cap, d, m, overlap, _p(tok, C.c_uint16), _p(ctx_len, C.c_int64),
                   _p(_c(w_s, np.float32), C.c_float), _p(_c(b_pos, np.float32), C.c_float),
                   _p(None if gamma is None else _c(gamma, np.float32), C.c_float),
                   eps, 1 if normalize else 0, rope_dim, rope_base, _p(rope_freq, C.c_double),
                   first_block, n_blocks, N_cap,
                   _p(out, C.c_double), _p(written, C.c_uint8), nthreads)
    return out, written.astype(bool)


def quant_rows_e4m3(x):
    """E4M3 storage of indexer keys, decision in binary32.  x: [..., dim] fp64."""
    x = _c(x, np.float64)
    dim = x.shape[-1]
    rows = x.size // dim
    codes = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[:-1], np.float32)
    lib().orc_quant_rows_e4m3(rows, dim, _p(x, C.c_double), _p(codes, C.c_uint8),
                              _p(scale, C.c_float))
    return codes, scale


def index_scores(q_idx, q_scale, w, key, key_scale, pos_q, m, nthreads=0):
    """Lightning-Indexer scores (a2) in fp64.  q_idx [B,Q,H_I,D_I] codes; key [B,N_cap,D_I]."""
    q_idx = _c(q_idx, np.uint8)
    B, Q, H_I, D_I = q_idx.shape
    key = _c(key, np.uint8)
    N_cap = key.shape[1]
    scores = np.empty((B, Q, N_cap), np.float64)
    lib().orc_index_scores(B, Q, H_I, D_I, m, _p(q_idx, C.c_uint8),
                           _p(_c(q_scale, np.float32), C.c_float),
                           _p(_c(w, np.float32), C.c_float), _p(key, C.c_uint8),
                           _p(_c(key_scale, np.float32), C.c_float), N_cap,
                           _p(_c(pos_q, np.int64), C.c_int64), _p(scores, C.c_double), nthreads)
    return scores


def topk(scores, n_vis, k, nthreads=0):
    """Top-k selection (a3).  scores [...,N]; n_vis [...]; returns (idx [...,k] int32, cnt [...])."""
    s = _c(scores, np.float64)
    lead = s.shape[:-1]
    N = s.shape[-1]
    BQ = int(np.prod(lead)) if lead else 1
    nv = _c(np.broadcast_to(n_vis, lead), np.int64)
    idx = np.empty(lead + (k,), np.int32)
    cnt = np.empty(lead, np.int32)
    lib().orc_topk(BQ, N, _p(s, C.c_double), _p(nv, C.c_int64), k, _p(idx, C.c_int32),
                   _p(cnt, C.c_int32), nthreads)
    return idx, cnt


def mqa(q, pos_q, kv_c, kv_tok, sink, m, W, rope_dim, sel_idx=None, sel_cnt=None,
        gamma_q=None, gamma_kv=None, eps=1e-6, scale=None, rope_base=10000.0, nthreads=0,
        tok_base=0, rope_freq=None):
    """Shared-KV MQA with window and sink (a4 sparse when sel_idx is given, else a5 dense).

    q [B,Q,H,D] bf16 bits; pos_q [B,Q]; kv_c [B,N_cap,D]; kv_tok [B,L_cap,D] holding
    token rows tok_base .. tok_base+L_cap-1.  rope_freq [rope_dim/2] replaces
    the frequencies rope_base^(-2j/rope_dim).
    Returns (out fp64 [B,Q,H,D], lse fp64 [B,Q,H]).
    """
    rope_freq = _freq(rope_freq, rope_dim)
    q = _c(q, np.uint16)
    B, Q, H, D = q.shape
    kv_c = _c(kv_c, np.uint16)
    kv_tok = _c(kv_tok, np.uint16)
    N_cap, L_cap = kv_c.shape[1], kv_tok.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    kmax = 0
    if sel_idx is not None:
        sel_idx = _c(sel_idx, np.int32)
        kmax = sel_idx.shape[-1]
        sel_cnt = _c(sel_cnt, np.int32)
    out = np.empty((B, Q, H, D), np.float64)
    lse = np.empty((B, Q, H), np.float64)
    lib().orc_mqa(B, Q, H, D, m, W, rope_dim, rope_base, _p(rope_freq, C.c_double),
                  _p(q, C.c_uint16),
                  _p(_c(pos_q, np.int64), C.c_int64), _p(kv_c, C.c_uint16), N_cap,
                  _p(sel_idx, C.c_int32), _p(sel_cnt, C.c_int32), kmax,
                  _p(kv_tok, C.c_uint16), L_cap, tok_base, _p(_c(sink, np.float32), C.c_float),
                  _p(None if gamma_q is None else _c(gamma_q, np.float32), C.c_float),
                  _p(None if gamma_kv is None else _c(gamma_kv, np.float32), C.c_float),
                  eps, scale, _p(out, C.c_double), _p(lse, C.c_double), nthreads)
    return out, lse


# --------------------------------------------------------------- composites --
def compress_kv(tok, ctx_len, w_s, b_pos, gamma, m, first_block, n_blocks, N_cap, eps=1e-6,
                nthreads=0, rope_dim=0, rope_base=10000.0, rope_freq=None, overlap=0):
    """a1 for the KV stream with bfloat16 storage (entries stored rotated to
    their position when rope_dim > 0): returns (bf16 bits, written mask, fp64 values)."""
    vals, written = pool(tok, ctx_len, w_s, b_pos, gamma, m, first_block, n_blocks, N_cap,
                         eps, True, nthreads, rope_dim, rope_base, rope_freq, overlap)
    return bf16_encode(vals), written, vals


def compress_index(tok, ctx_len, w_s, b_pos, m, first_block, n_blocks, N_cap, eps=1e-6,
                   nthreads=0, overlap=0):
    """a1 for the indexer stream: pooled, RMSNorm'd, E4M3 rows (codes, scale, fp64 values, written)."""
    vals, written = pool(tok, ctx_len, w_s, b_pos, None, m, first_block, n_blocks, N_cap,
                         eps, True, nthreads, overlap=overlap)
    codes, scale = quant_rows_e4m3(vals)
    return codes, scale, vals, written


def csa_decode(q, q_idx, q_scale, w, pos_q, kv_c, idx_key, idx_scale, kv_tok, sink, m, k, W,
               rope_dim, gamma_q=None, gamma_kv=None, nthreads=0):
    """One CSA decode step after compression: indexer -> top-k -> sparse MQA.

    q [B,H,D] (one query per sequence).  Returns dict of intermediate and final results.
    """
    B = q.shape[0]
    pos = _c(pos_q, np.int64).reshape(B, 1)
    sc = index_scores(q_idx.reshape((B, 1) + q_idx.shape[-2:]), q_scale.reshape(B, 1, -1),
                      w.reshape(B, 1, -1), idx_key, idx_scale, pos, m, nthreads)
    n_vis = np.minimum((pos + 1) // m, idx_key.shape[1])
    idx, cnt = topk(sc, n_vis, k, nthreads)
    out, lse = mqa(q.reshape((B, 1) + q.shape[-2:]), pos, kv_c, kv_tok, sink, m, W, rope_dim,
                   idx, cnt, gamma_q, gamma_kv, nthreads=nthreads)
    return dict(scores=sc[:, 0], idx=idx[:, 0], cnt=cnt[:, 0], out=out[:, 0], lse=lse[:, 0],
                out_bf16=bf16_encode(out[:, 0]))


def hca_decode(q, pos_q, kv_c, kv_tok, sink, m, W, rope_dim, gamma_q=None, gamma_kv=None,
               nthreads=0):
    """One HCA decode step after compression: dense MQA over all visible entries."""
    B = q.shape[0]
    pos = _c(pos_q, np.int64).reshape(B, 1)
    out, lse = mqa(q.reshape((B, 1) + q.shape[-2:]), pos, kv_c, kv_tok, sink, m, W, rope_dim,
                   None, None, gamma_q, gamma_kv, nthreads=nthreads)
    return dict(out=out[:, 0], lse=lse[:, 0], out_bf16=bf16_encode(out[:, 0]))


def grouped_out_proj(o, w_g, w_o, y_bf16=True, y_in=None, nthreads=0):
    """Grouped output projection (f1) in fp64.

    o [T, H, D] bf16 bits (the attention output); w_g [g, d_g, H/g * D] and
    w_o [d, g * d_g] bf16 bits (rows = outputs).  y_bf16 rounds the
    intermediate y to bf16 (the library's storage); y_in [T, g * d_g] bf16
    bits replaces the first projection.  Returns (y fp64 [T, g*d_g], z fp64 [T, d])."""
    o = _c(o, np.uint16)
    T, H, D = o.shape
    w_g = _c(w_g, np.uint16)
    g, d_g, kin = w_g.shape
    if H % g or kin != (H // g) * D:
        raise ValueError("w_g must be [g, d_g, H/g * D] with g dividing H")
    w_o = _c(w_o, np.uint16)
    d_model = w_o.shape[0]
    if w_o.shape[1] != g * d_g:
        raise ValueError("w_o must be [d, g * d_g]")
    if y_in is not None:
        y_in = _c(y_in, np.uint16)
        if y_in.shape != (T, g * d_g):
            raise ValueError("y_in must be [T, g * d_g]")
    y = np.empty((T, g * d_g), np.float64)
    z = np.empty((T, d_model), np.float64)
    lib().orc_grouped_out_proj(T, H, D, g, d_g, d_model, _p(o, C.c_uint16), _p(w_g, C.c_uint16),
                               _p(w_o, C.c_uint16), 1 if y_bf16 else 0, _p(y_in, C.c_uint16),
                               _p(y, C.c_double), _p(z, C.c_double), nthreads)
    return y, z
