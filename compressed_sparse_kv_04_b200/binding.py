"""Thin ctypes binding of libcsa.so (include/csa.h), same entry-point names.

Argument marshalling only: every step runs in the library's CUDA kernels.
Tensors are torch tensors on the current CUDA device; the current torch
stream is passed as the `stream` argument.  Loading fails loudly when the
library has not been built: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

CSA_OK = 0
STATUS_NAMES = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED_SHAPE",
                3: "CSA_ERR_CAPACITY", 4: "CSA_ERR_WORKSPACE", 5: "CSA_ERR_CUDA",
                6: "CSA_ERR_DEVICE_TIMEOUT", 7: "CSA_ERR_DEVICE_INDEX"}
OP_INDEX_TOPK, OP_SPARSE_MQA, OP_DENSE_MQA, OP_PREFILL, OP_HCA_PREFILL = 1, 2, 3, 4, 5
OP_CSA_DECODE_STEP, OP_HCA_DECODE_STEP = 6, 7

EXPORTS = ["csa_version", "csa_last_error", "csa_workspace_bytes", "hca_compress",
           "csa_compress", "lightning_index_topk", "lightning_index_scores", "topk_select",
           "sparse_mqa_decode", "dense_mqa_decode", "csa_prefill_chunk",
           "lightning_index_topk_static", "csa_rope_yarn", "hca_prefill_chunk",
           "csa_decode_step", "hca_decode_step", "grouped_out_proj",
           "grouped_out_proj_workspace_bytes", "csa_shard_candidates", "csa_merge_candidates",
           "sparse_mqa_partials", "mqa_merge_partials", "csa_copy_async", "csa_copy_rows_async"]


class CsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class csa_params(C.Structure):
    _fields_ = [("B", C.c_int), ("d", C.c_int), ("H", C.c_int), ("H_I", C.c_int),
                ("D_I", C.c_int), ("k", C.c_int), ("window", C.c_int), ("rope_dim", C.c_int),
                ("m", C.c_int), ("eps", C.c_float), ("softmax_scale", C.c_float),
                ("rope_inv_freq", C.POINTER(C.c_double)), ("overlap", C.c_int),
                ("entry_offset", C.c_int64)]


_lib = None


def lib():
    """The loaded libcsa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libcsa.so not found at {LIB_PATH}; build it with "
                               "`python -m compressed_sparse_kv_04_b200.build`")
        L = C.CDLL(LIB_PATH)
        _declare(L)
        _lib = L
    return _lib


def _declare(L):
    vp, i32, i64, sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
    P = C.POINTER(csa_params)
    L.csa_version.restype = i32
    L.csa_last_error.restype = C.c_char_p
    L.csa_workspace_bytes.argtypes = [P, i32, i32, i64]
    L.csa_workspace_bytes.restype = sz
    L.hca_compress.argtypes = [P, vp, i64, vp, vp, vp, vp, i64, i64, vp, i64, vp, vp]
    L.csa_compress.argtypes = [P, vp, i64, vp, vp, vp, vp, i64, i64, vp, i64, vp, vp, vp, vp,
                               vp, vp, vp]
    L.lightning_index_topk.argtypes = [P, i32, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, sz,
                                       vp, vp]
    L.lightning_index_scores.argtypes = [P, i32, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp]
    L.topk_select.argtypes = [P, i32, vp, i64, vp, vp, vp, vp, vp]
    L.sparse_mqa_decode.argtypes = [P, vp, vp, vp, i64, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp,
                                    sz, vp, vp]
    L.dense_mqa_decode.argtypes = [P, vp, vp, vp, i64, vp, i64, vp, vp, vp, vp, vp, vp, sz, vp,
                                   vp]
    L.csa_prefill_chunk.argtypes = [P, i64, i32, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp,
                                    i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    L.lightning_index_topk_static.argtypes = [P, i32, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp,
                                              vp]
    L.hca_prefill_chunk.argtypes = [P, i64, i32, vp, i64, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp,
                                    vp, vp, sz, vp, vp]
    L.csa_decode_step.argtypes = [P, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, i64, vp, vp,
                                  vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]
    L.hca_decode_step.argtypes = [P, vp, vp, i64, vp, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp, vp,
                                  sz, vp, vp]
    L.csa_rope_yarn.argtypes = [i32, C.c_double, C.c_double, C.c_double, C.c_double,
                                C.c_double, i32, C.POINTER(C.c_double), C.POINTER(C.c_double),
                                C.POINTER(C.c_float)]
    L.grouped_out_proj.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp,
                                   vp]
    L.grouped_out_proj_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    L.grouped_out_proj_workspace_bytes.restype = sz
    L.csa_shard_candidates.argtypes = [P, i32, vp, i64, vp, vp, vp, vp, vp, vp]
    L.csa_merge_candidates.argtypes = [P, i32, i32, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp]
    L.sparse_mqa_partials.argtypes = [P, i32, vp, vp, vp, i64, vp, vp, vp, i64, vp, vp, vp, vp,
                                      vp, vp]
    L.mqa_merge_partials.argtypes = [P, i32, vp, vp, vp, vp, vp, vp, vp, vp]
    L.csa_copy_async.argtypes = [vp, vp, sz, vp]
    L.csa_copy_rows_async.argtypes = [vp, sz, vp, sz, sz, sz, vp]
    for name in EXPORTS[3:]:
        if name != "grouped_out_proj_workspace_bytes":
            getattr(L, name).restype = i32


def make_params(B, d, H=0, H_I=0, D_I=0, k=0, window=0, rope_dim=0, m=4, eps=1e-6,
                softmax_scale=0.0, rope_inv_freq=None, overlap=0, entry_offset=0):
    p = csa_params(B, d, H, H_I, D_I, k, window, rope_dim, m, eps, softmax_scale, None, overlap,
                   entry_offset)
    if rope_inv_freq is not None:
        arr = (C.c_double * len(rope_inv_freq))(*rope_inv_freq)
        p.rope_inv_freq = C.cast(arr, C.POINTER(C.c_double))
        p._keep = arr
    return p


def params_for(w, B=None, **kw):
    """csa_params for a Workload (compressed_sparse_kv_04_b200.configs).  A
    workload with YaRN settings gets the library's YaRN frequency table and
    logit scale (csa_rope_yarn), unless the caller passes its own."""
    if w.yarn is not None and w.rope_dim > 0 and "rope_inv_freq" not in kw:
        tab, _, scale = rope_yarn(w.rope_dim, *w.yarn, d=w.d)
        kw["rope_inv_freq"] = tab
        kw.setdefault("softmax_scale", scale)
    kw.setdefault("overlap", w.overlap)
    return make_params(B or w.B, w.d, w.H, w.H_I, w.D_I, w.k, w.W, w.rope_dim, w.m, **kw)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"expected a torch.Tensor, got {type(t)}")
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(status):
    if status != CSA_OK:
        raise CsaError(status, lib().csa_last_error().decode())


def version():
    return lib().csa_version()


def workspace_bytes(p, op, Q, N_cap):
    n = lib().csa_workspace_bytes(C.byref(p), op, Q, N_cap)
    if n == 0:
        raise CsaError(1, lib().csa_last_error().decode())
    return n


def workspace(p, op, Q, N_cap, device=None):
    """A zero-filled workspace (the decode step's score histogram starts
    cleared; each call leaves it so)."""
    return torch.zeros(workspace_bytes(p, op, Q, N_cap), dtype=torch.uint8,
                       device=device or torch.cuda.current_device())


def hca_compress(p, kv_tok, ctx_len, w_s, b_pos, gamma, first_block, n_blocks, kv_c,
                 dev_status=None, stream=None):
    _check(lib().hca_compress(C.byref(p), _ptr(kv_tok), kv_tok.shape[1], _ptr(ctx_len),
                              _ptr(w_s), _ptr(b_pos), _ptr(gamma), first_block, n_blocks,
                              _ptr(kv_c), kv_c.shape[1], _ptr(dev_status), _stream(stream)))


def csa_compress(p, kv_tok, ctx_len, w_s, b_pos, gamma, first_block, n_blocks, kv_c,
                 idx_tok=None, w_s_idx=None, b_pos_idx=None, idx_key=None, idx_scale=None,
                 dev_status=None, stream=None):
    _check(lib().csa_compress(C.byref(p), _ptr(kv_tok), kv_tok.shape[1], _ptr(ctx_len),
                              _ptr(w_s), _ptr(b_pos), _ptr(gamma), first_block, n_blocks,
                              _ptr(kv_c), kv_c.shape[1], _ptr(idx_tok), _ptr(w_s_idx),
                              _ptr(b_pos_idx), _ptr(idx_key), _ptr(idx_scale),
                              _ptr(dev_status), _stream(stream)))


def lightning_index_topk(p, Q, q_idx, q_scale, w, idx_key, idx_scale, pos_q, topk_idx,
                         topk_cnt, scores_out=None, ws=None, dev_status=None, stream=None):
    _check(lib().lightning_index_topk(
        C.byref(p), Q, _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(idx_key), _ptr(idx_scale),
        idx_key.shape[1], _ptr(pos_q), _ptr(topk_idx), _ptr(topk_cnt), _ptr(scores_out),
        _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(stream)))


def lightning_index_topk_static(p, Q, q_idx, q_scale, w, idx_key, idx_scale, pos_q, topk_idx,
                                topk_cnt, dev_status=None, stream=None):
    """lightning_index_topk with the scores in the library's own device array
    (no workspace; B*Q*N_cap <= 2**21)."""
    _check(lib().lightning_index_topk_static(
        C.byref(p), Q, _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(idx_key), _ptr(idx_scale),
        idx_key.shape[1], _ptr(pos_q), _ptr(topk_idx), _ptr(topk_cnt), _ptr(dev_status),
        _stream(stream)))


def rope_yarn(rope_dim, factor, beta_fast, beta_slow, original_len, base=10000.0, d=1):
    """YaRN frequency table, logit gain and logit scale for head dim d (host
    only, computed by the library): returns (list of rope_dim/2 frequencies
    for make_params(rope_inv_freq=...), logit gain, softmax_scale)."""
    tab = (C.c_double * max(1, rope_dim // 2))()
    gain = C.c_double()
    scale = C.c_float()
    _check(lib().csa_rope_yarn(rope_dim, base, factor, beta_fast, beta_slow, original_len, d, tab,
                               C.byref(gain), C.byref(scale)))
    return list(tab)[: rope_dim // 2], gain.value, scale.value


def lightning_index_scores(p, Q, q_idx, q_scale, w, idx_key, idx_scale, pos_q, scores,
                           dev_status=None, stream=None):
    _check(lib().lightning_index_scores(
        C.byref(p), Q, _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(idx_key), _ptr(idx_scale),
        idx_key.shape[1], _ptr(pos_q), _ptr(scores), _ptr(dev_status), _stream(stream)))


def topk_select(p, Q, scores, pos_q, topk_idx, topk_cnt, dev_status=None, stream=None):
    _check(lib().topk_select(C.byref(p), Q, _ptr(scores), scores.shape[-1], _ptr(pos_q),
                             _ptr(topk_idx), _ptr(topk_cnt), _ptr(dev_status), _stream(stream)))


def sparse_mqa_decode(p, q, pos_q, kv_c, topk_idx, topk_cnt, kv_tok, sink, out, gamma_q=None,
                      gamma_kv=None, lse=None, ws=None, dev_status=None, stream=None):
    _check(lib().sparse_mqa_decode(
        C.byref(p), _ptr(q), _ptr(pos_q), _ptr(kv_c), kv_c.shape[1], _ptr(topk_idx),
        _ptr(topk_cnt), _ptr(kv_tok), kv_tok.shape[1], _ptr(sink), _ptr(gamma_q),
        _ptr(gamma_kv), _ptr(out), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def dense_mqa_decode(p, q, pos_q, kv_c, kv_tok, sink, out, gamma_q=None, gamma_kv=None,
                     lse=None, ws=None, dev_status=None, stream=None):
    _check(lib().dense_mqa_decode(
        C.byref(p), _ptr(q), _ptr(pos_q), _ptr(kv_c), kv_c.shape[1], _ptr(kv_tok),
        kv_tok.shape[1], _ptr(sink), _ptr(gamma_q), _ptr(gamma_kv), _ptr(out), _ptr(lse),
        _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(stream)))


def csa_prefill_chunk(p, P, T, kv_tok, idx_tok, w_s, b_pos, gamma, w_s_idx, b_pos_idx, kv_c,
                      idx_key, idx_scale, q, q_idx, q_scale, w, sink, topk_idx, topk_cnt, out,
                      gamma_q=None, gamma_kv=None, ws=None, dev_status=None, stream=None):
    _check(lib().csa_prefill_chunk(
        C.byref(p), P, T, _ptr(kv_tok), _ptr(idx_tok), kv_tok.shape[1], _ptr(w_s), _ptr(b_pos),
        _ptr(gamma), _ptr(w_s_idx), _ptr(b_pos_idx), _ptr(kv_c), _ptr(idx_key), _ptr(idx_scale),
        kv_c.shape[1], _ptr(q), _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(sink), _ptr(gamma_q),
        _ptr(gamma_kv), _ptr(topk_idx), _ptr(topk_cnt), _ptr(out), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def hca_prefill_chunk(p, P, T, kv_tok, w_s, b_pos, gamma, kv_c, q, sink, out, gamma_q=None,
                      gamma_kv=None, lse=None, ws=None, dev_status=None, stream=None):
    """HCA prefill chunk (B = 1): compression of the chunk's blocks, then dense
    MQA per new query.  kv_tok [1, L_cap, d]; kv_c [1, N_cap, d]; q/out [T, H, d]."""
    _check(lib().hca_prefill_chunk(
        C.byref(p), P, T, _ptr(kv_tok), kv_tok.shape[1], _ptr(w_s), _ptr(b_pos), _ptr(gamma),
        _ptr(kv_c), kv_c.shape[1], _ptr(q), _ptr(sink), _ptr(gamma_q), _ptr(gamma_kv), _ptr(out),
        _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
        _ptr(dev_status), _stream(stream)))


def csa_decode_step(p, pos_q, kv_tok, idx_tok, w_s, b_pos, gamma, w_s_idx, b_pos_idx, kv_c,
                    idx_key, idx_scale, q, q_idx, q_scale, w, sink, topk_idx, topk_cnt, out,
                    gamma_q=None, gamma_kv=None, lse=None, ws=None, dev_status=None, stream=None):
    """One CSA decode step (newest-block compression, indexer, top-k, sparse
    MQA) for B sequences at positions pos_q [B]."""
    _check(lib().csa_decode_step(
        C.byref(p), _ptr(pos_q), _ptr(kv_tok), _ptr(idx_tok), kv_tok.shape[1], _ptr(w_s),
        _ptr(b_pos), _ptr(gamma), _ptr(w_s_idx), _ptr(b_pos_idx), _ptr(kv_c), _ptr(idx_key),
        _ptr(idx_scale), kv_c.shape[1], _ptr(q), _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(sink),
        _ptr(gamma_q), _ptr(gamma_kv), _ptr(topk_idx), _ptr(topk_cnt), _ptr(out), _ptr(lse),
        _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status),
        _stream(stream)))


class CsaDecodeStep:
    """csa_decode_step for a fixed set of sequences: the arguments that stay
    the same from step to step (token buffers, caches, weights, sink and
    gains, the selection outputs, workspace and status word) are checked and
    converted once; each call passes the step's positions, queries and
    outputs.  Same C entry point and the same device-side work as
    csa_decode_step (argument marshalling only)."""

    def __init__(self, p, kv_tok, idx_tok, w_s, b_pos, gamma, w_s_idx, b_pos_idx, kv_c, idx_key,
                 idx_scale, sink, topk_idx, topk_cnt, ws, gamma_q=None, gamma_kv=None,
                 dev_status=None):
        self._fn = lib().csa_decode_step
        self._keep = (p, kv_tok, idx_tok, w_s, b_pos, gamma, w_s_idx, b_pos_idx, kv_c, idx_key,
                      idx_scale, sink, topk_idx, topk_cnt, ws, gamma_q, gamma_kv, dev_status)
        self._head = (C.byref(p),)
        self._mid = (_ptr(kv_tok), _ptr(idx_tok), kv_tok.shape[1], _ptr(w_s), _ptr(b_pos),
                     _ptr(gamma), _ptr(w_s_idx), _ptr(b_pos_idx), _ptr(kv_c), _ptr(idx_key),
                     _ptr(idx_scale), kv_c.shape[1])
        self._sink = (_ptr(sink), _ptr(gamma_q), _ptr(gamma_kv), _ptr(topk_idx), _ptr(topk_cnt))
        self._tail = (_ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status))

    def _args(self, pos_q, q, q_idx, q_scale, w, out, lse, stream):
        return (*self._head, _ptr(pos_q), *self._mid, _ptr(q), _ptr(q_idx), _ptr(q_scale),
                _ptr(w), *self._sink, _ptr(out), _ptr(lse), *self._tail, _stream(stream))

    def __call__(self, pos_q, q, q_idx, q_scale, w, out, lse=None, stream=None):
        _check(self._fn(*self._args(pos_q, q, q_idx, q_scale, w, out, lse, stream)))

    def bind(self, pos_q, q, q_idx, q_scale, w, out, lse=None, stream=None):
        """The step with its per-step buffers fixed as well (a decode loop
        that writes each step's positions and queries into the same
        buffers): returns f() that runs one step on `stream`."""
        fn, args = self._fn, self._args(pos_q, q, q_idx, q_scale, w, out, lse, stream)
        keep = (self, pos_q, q, q_idx, q_scale, w, out, lse, stream)

        def run(_keep=keep):
            _check(fn(*args))
        return run


class HcaDecodeStep:
    """hca_decode_step for a fixed set of sequences (see CsaDecodeStep)."""

    def __init__(self, p, kv_tok, w_s, b_pos, gamma, kv_c, sink, ws, gamma_q=None, gamma_kv=None,
                 dev_status=None):
        self._fn = lib().hca_decode_step
        self._keep = (p, kv_tok, w_s, b_pos, gamma, kv_c, sink, ws, gamma_q, gamma_kv, dev_status)
        self._head = (C.byref(p),)
        self._mid = (_ptr(kv_tok), kv_tok.shape[1], _ptr(w_s), _ptr(b_pos), _ptr(gamma),
                     _ptr(kv_c), kv_c.shape[1])
        self._gains = (_ptr(sink), _ptr(gamma_q), _ptr(gamma_kv))
        self._tail = (_ptr(ws), ws.numel() * ws.element_size(), _ptr(dev_status))

    def _args(self, pos_q, q, out, lse, stream):
        return (*self._head, _ptr(pos_q), *self._mid, _ptr(q), *self._gains, _ptr(out),
                _ptr(lse), *self._tail, _stream(stream))

    def __call__(self, pos_q, q, out, lse=None, stream=None):
        _check(self._fn(*self._args(pos_q, q, out, lse, stream)))

    def bind(self, pos_q, q, out, lse=None, stream=None):
        """The step with its per-step buffers fixed (see CsaDecodeStep.bind)."""
        fn, args = self._fn, self._args(pos_q, q, out, lse, stream)
        keep = (self, pos_q, q, out, lse, stream)

        def run(_keep=keep):
            _check(fn(*args))
        return run


def _rows_of(t):
    """(rows, row_bytes, pitch_bytes) of a tensor whose first dimension
    strides over rows that are each contiguous."""
    if t.dim() == 0:
        return 1, t.element_size(), t.element_size()
    inner = t[0] if t.shape[0] > 0 else t
    if t.shape[0] > 0 and not inner.is_contiguous():
        raise ValueError("each row (first-dimension slice) must be contiguous")
    row = (t.numel() // max(1, t.shape[0])) * t.element_size()
    pitch = t.stride(0) * t.element_size() if t.shape[0] > 1 else row
    return t.shape[0], row, pitch


class PreparedCopy:
    """One asynchronous copy between two tensors of the same shape and dtype
    (page-locked host <-> device, either direction) with its addresses and
    stream fixed: csa_copy_async when both are contiguous, else
    csa_copy_rows_async over the first dimension (each row contiguous, e.g.
    kv_tok[:, pos:pos+1] of a [B, L_cap, d] token buffer).  f() enqueues it."""

    def __init__(self, dst, src, stream=None):
        if dst.shape != src.shape or dst.dtype != src.dtype:
            raise ValueError(f"copy between {tuple(src.shape)} {src.dtype} and "
                             f"{tuple(dst.shape)} {dst.dtype}")
        for t in (dst, src):
            if not t.is_cuda and not t.is_pinned():
                raise ValueError("host tensors of a prepared copy must be page-locked")
        self._keep = (dst, src, stream)
        L = lib()
        st = _stream(stream)
        if dst.is_contiguous() and src.is_contiguous():
            fn = L.csa_copy_async
            args = (C.c_void_p(dst.data_ptr()), C.c_void_p(src.data_ptr()),
                    dst.numel() * dst.element_size(), st)
        else:
            rows, row, dp = _rows_of(dst)
            _, srow, sp = _rows_of(src)
            fn = L.csa_copy_rows_async
            args = (C.c_void_p(dst.data_ptr()), dp, C.c_void_p(src.data_ptr()), sp, row, rows, st)
        self.bytes = dst.numel() * dst.element_size()
        self._fn, self._args = fn, args

    def __call__(self):
        _check(self._fn(*self._args))


def hca_decode_step(p, pos_q, kv_tok, w_s, b_pos, gamma, kv_c, q, sink, out, gamma_q=None,
                    gamma_kv=None, lse=None, ws=None, dev_status=None, stream=None):
    """One HCA decode step (newest-block compression, dense MQA) for B
    sequences at positions pos_q [B]."""
    _check(lib().hca_decode_step(
        C.byref(p), _ptr(pos_q), _ptr(kv_tok), kv_tok.shape[1], _ptr(w_s), _ptr(b_pos),
        _ptr(gamma), _ptr(kv_c), kv_c.shape[1], _ptr(q), _ptr(sink), _ptr(gamma_q),
        _ptr(gamma_kv), _ptr(out), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _ptr(dev_status), _stream(stream)))


def grouped_out_proj_workspace_bytes(T, H, D, g, d_g, d_model):
    n = lib().grouped_out_proj_workspace_bytes(T, H, D, g, d_g, d_model)
    if n == 0:
        raise CsaError(2, lib().csa_last_error().decode())
    return n


def grouped_out_proj(o, w_g, w_o, z, y=None, ws=None, dev_status=None, stream=None):
    """Grouped output projection: o [T, H, D] -> y [T, g*d_g] -> z [T, d_model]
    (w_g [g, d_g, H/g*D], w_o [d_model, g*d_g], all bf16).  The workspace is
    allocated here when not given."""
    T, H, D = o.shape
    g, d_g, _ = w_g.shape
    d_model = w_o.shape[0]
    if ws is None:
        ws = torch.empty(grouped_out_proj_workspace_bytes(T, H, D, g, d_g, d_model),
                         dtype=torch.uint8, device=o.device)
    _check(lib().grouped_out_proj(T, H, D, g, d_g, d_model, _ptr(o), _ptr(w_g), _ptr(w_o),
                                  _ptr(y), _ptr(z), _ptr(ws), ws.numel() * ws.element_size(),
                                  _ptr(dev_status), _stream(stream)))


# ------------------------------------------- context split over several devices --
def csa_shard_candidates(p, Q, scores, topk_idx, topk_cnt, cand_score, cand_idx,
                         dev_status=None, stream=None):
    _check(lib().csa_shard_candidates(C.byref(p), Q, _ptr(scores), scores.shape[-1],
                                      _ptr(topk_idx), _ptr(topk_cnt), _ptr(cand_score),
                                      _ptr(cand_idx), _ptr(dev_status), _stream(stream)))


def csa_merge_candidates(p, Q, G, cand_score, cand_idx, cand_cnt, N_cap, topk_idx, topk_cnt,
                         local_idx, local_cnt, dev_status=None, stream=None):
    _check(lib().csa_merge_candidates(C.byref(p), Q, G, _ptr(cand_score), _ptr(cand_idx),
                                      _ptr(cand_cnt), N_cap, _ptr(topk_idx), _ptr(topk_cnt),
                                      _ptr(local_idx), _ptr(local_cnt), _ptr(dev_status),
                                      _stream(stream)))


def sparse_mqa_partials(p, splits, q, pos_q, kv_c, topk_idx, topk_cnt, kv_tok, part_o, part_ml,
                        gamma_q=None, gamma_kv=None, dev_status=None, stream=None):
    _check(lib().sparse_mqa_partials(C.byref(p), splits, _ptr(q), _ptr(pos_q), _ptr(kv_c),
                                     kv_c.shape[1], _ptr(topk_idx), _ptr(topk_cnt), _ptr(kv_tok),
                                     kv_tok.shape[1], _ptr(gamma_q), _ptr(gamma_kv),
                                     _ptr(part_o), _ptr(part_ml), _ptr(dev_status),
                                     _stream(stream)))


def mqa_merge_partials(p, splits, part_o, part_ml, pos_q, sink, out, lse=None, dev_status=None,
                       stream=None):
    _check(lib().mqa_merge_partials(C.byref(p), splits, _ptr(part_o), _ptr(part_ml), _ptr(pos_q),
                                    _ptr(sink), _ptr(out), _ptr(lse), _ptr(dev_status),
                                    _stream(stream)))
