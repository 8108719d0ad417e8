// C ABI of libcsa.so: argument validation, workspace carving and launches.
// Every entry point is declared and documented in include/csa.h.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/csa.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

csa_status fail(csa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

constexpr int64_t kMaxIndexEntries = 262144;  // one 8-CTA cluster holds a score row
constexpr int kMaxTopk = 2048;                // entries kept per query

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQ_PTR(p)                                                                     \
  do {                                                                                 \
    if ((p) == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: %s is null", fn, #p);    \
    if (!aligned16(p)) return fail(CSA_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)
#define OPT_PTR(p)                                                                     \
  do {                                                                                 \
    if ((p) != nullptr && !aligned16(p))                                               \
      return fail(CSA_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, #p);      \
  } while (0)
// 4-byte alignment suffices for small fp32 parameter vectors.
#define REQ_PTR4(p)                                                                    \
  do {                                                                                 \
    if ((p) == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: %s is null", fn, #p);    \
    if ((reinterpret_cast<uintptr_t>(p) & 3u) != 0)                                    \
      return fail(CSA_ERR_INVALID_ARG, "%s: %s is not 4-byte aligned", fn, #p);       \
  } while (0)
#define OPT_PTR4(p)                                                                    \
  do {                                                                                 \
    if ((p) != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) != 0)                  \
      return fail(CSA_ERR_INVALID_ARG, "%s: %s is not 4-byte aligned", fn, #p);       \
  } while (0)

csa_status check_common(const char* fn, const csa_params* p) {
  if (!p) return fail(CSA_ERR_INVALID_ARG, "%s: params is null", fn);
  if (p->B < 1) return fail(CSA_ERR_INVALID_ARG, "%s: B=%d must be >= 1", fn, p->B);
  if (p->d != 128 && p->d != 512)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: d=%d (supported: 128, 512)", fn, p->d);
  if (p->m < 1 || p->m > 128)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: m=%d (supported: 1..128)", fn, p->m);
  if (p->entry_offset < 0 || p->entry_offset > ((int64_t)1 << 40))
    return fail(CSA_ERR_INVALID_ARG, "%s: entry_offset=%lld", fn, (long long)p->entry_offset);
  if (p->overlap < 0 || p->overlap > p->m || p->m + p->overlap > 128)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: overlap=%d (supported: 0..m, m + overlap <= 128)",
                fn, p->overlap);
  if (!(p->eps > 0.f) || !std::isfinite(p->eps))
    return fail(CSA_ERR_INVALID_ARG, "%s: eps must be finite and > 0", fn);
  return CSA_OK;
}

csa_status check_indexer(const char* fn, const csa_params* p) {
  if (p->D_I != 64 && p->D_I != 128)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: D_I=%d (supported: 64, 128)", fn, p->D_I);
  if (p->H_I < 1 || p->H_I > 64)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: H_I=%d (supported: 1..64)", fn, p->H_I);
  if (p->k < 1 || p->k > kMaxTopk)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: k=%d (supported: 1..%d)", fn, p->k, kMaxTopk);
  return CSA_OK;
}

csa_status check_attention(const char* fn, const csa_params* p) {
  if (p->H < 1 || p->H > 128)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: H=%d (supported: 1..128)", fn, p->H);
  if (p->window < 0 || p->window > 1024)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: window=%d (supported: 0..1024)", fn, p->window);
  if ((p->rope_dim != 0 && p->rope_dim != 32 && p->rope_dim != 64) || p->rope_dim > p->d / 4)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "%s: rope_dim=%d (supported: 0, 32, 64, and at most d/4)", fn, p->rope_dim);
  if (p->softmax_scale < 0.f || !std::isfinite(p->softmax_scale))
    return fail(CSA_ERR_INVALID_ARG, "%s: softmax_scale must be finite and >= 0", fn);
  return CSA_OK;
}

csa_status cuda_fail(const char* fn, cudaError_t e) {
  return fail(CSA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t scores_bytes(int64_t rows, int64_t N_cap) {
  return round_up((size_t)rows * (size_t)N_cap * sizeof(float), 256);
}

// The decode step's score histogram ([B, kScoreHistBins] u32, left zeroed by
// each call) and the top-k path word per sequence, after the scores.
size_t hist_bytes(int64_t B) {
  return (size_t)B * csa::kScoreHistBins * sizeof(uint32_t) + round_up((size_t)B * 4, 256);
}

void fill_inv_freq(const csa_params* p, double* out) {
  int half = p->rope_dim / 2;
  for (int j = 0; j < 64; ++j) out[j] = 0.0;
  for (int j = 0; j < half; ++j)
    out[j] = p->rope_inv_freq ? p->rope_inv_freq[j]
                              : std::pow(10000.0, -2.0 * j / (double)p->rope_dim);
}

float softmax_scale_of(const csa_params* p) {
  return p->softmax_scale > 0.f ? p->softmax_scale : (float)(1.0 / std::sqrt((double)p->d));
}

// reserve: SMs held by a kernel that runs alongside the attention (the
// compression of an HCA decode step, one CTA per sequence), left out so
// that every attention CTA is resident from the start.
int splits_for(const csa_params* p, csa_op op, int rows, int64_t N_cap, int reserve = 0) {
  const int64_t compressed_max = (op == CSA_OP_DENSE_MQA) ? N_cap : (int64_t)p->k;
  const int sms = csa::device_sm_count();
  return csa::mqa_choose_splits(rows, compressed_max, p->window,
                                sms - reserve >= 2 ? sms - reserve : sms, p->H);
}

// SMs the CSA decode step's attention leaves to its top-k.  The attention
// is launched while the top-k still runs; CTAs beyond the SMs the top-k
// leaves free start only when it ends.  Where every attention CTA fits
// beside the top-k at the cost of at most one more 64-entry tile per CTA,
// the splits are sized for the free SMs.
int decode_step_reserve(const csa_params* p, int64_t N_cap) {
  const int r = csa::topk_hist_ctas(p->B, N_cap);
  if (r <= 0) return 0;
  const int s0 = splits_for(p, CSA_OP_SPARSE_MQA, p->B, N_cap);
  const int s1 = splits_for(p, CSA_OP_SPARSE_MQA, p->B, N_cap, r);
  const int64_t tiles = ((int64_t)p->k + 63) / 64 + (p->window + 63) / 64;
  const int64_t t0 = (tiles + s0 - 1) / s0, t1 = (tiles + s1 - 1) / s1;
  return (s1 < s0 && t1 <= t0 + 1) ? r : 0;
}

}  // namespace

namespace csa {
// Records the message returned by csa_last_error (for entry points defined
// in other files of the library).
csa_status set_error(csa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}
}  // namespace csa

extern "C" {

int csa_version(void) { return 102; }

csa_status csa_rope_yarn(int rope_dim, double base, double factor, double beta_fast,
                         double beta_slow, double original_len, int d, double* inv_freq,
                         double* logit_gain, float* softmax_scale) {
  const char* fn = "csa_rope_yarn";
  if (rope_dim < 2 || rope_dim > 128 || rope_dim % 2)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: rope_dim=%d (supported: even, 2..128)", fn,
                rope_dim);
  if (!inv_freq) return fail(CSA_ERR_INVALID_ARG, "%s: inv_freq is NULL", fn);
  if (softmax_scale && d < 1)
    return fail(CSA_ERR_INVALID_ARG, "%s: d=%d must be >= 1 for softmax_scale", fn, d);
  if (!(base > 1.0) || !std::isfinite(base) || !(factor >= 1.0) || !std::isfinite(factor) ||
      !(beta_slow >= 0.0) || !(beta_fast > beta_slow) || !std::isfinite(beta_fast) ||
      !(original_len > 0.0) || !std::isfinite(original_len))
    return fail(CSA_ERR_INVALID_ARG,
                "%s: need base > 1, factor >= 1, 0 <= beta_slow < beta_fast, original_len > 0",
                fn);
  const double kTwoPi = 6.283185307179586;
  for (int j = 0; j < rope_dim / 2; ++j) {
    const double theta = std::pow(base, -2.0 * j / (double)rope_dim);
    // Turns of this pair over the original context place it on the ramp:
    // 1 keeps the frequency, 0 divides it by the factor.
    double ramp = (original_len * theta / kTwoPi - beta_slow) / (beta_fast - beta_slow);
    ramp = ramp < 0.0 ? 0.0 : (ramp > 1.0 ? 1.0 : ramp);
    inv_freq[j] = theta / factor + ramp * (theta - theta / factor);
  }
  // The method's attention temperature: q and k are each scaled by
  // 1 + 0.1 ln(factor), so the logits by its square.
  const double t = 1.0 + 0.1 * std::log(factor);
  if (logit_gain) *logit_gain = t * t;
  if (softmax_scale) *softmax_scale = (float)(t * t / std::sqrt((double)d));
  return CSA_OK;
}

const char* csa_last_error(void) { return g_err; }

csa_status csa_copy_async(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return CSA_OK;
  if (!dst || !src)
    return fail(CSA_ERR_INVALID_ARG, "csa_copy_async: NULL address for %zu bytes", bytes);
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return fail(CSA_ERR_CUDA, "csa_copy_async: %s", cudaGetErrorString(e));
  return CSA_OK;
}

csa_status csa_copy_rows_async(void* dst, size_t dst_pitch, const void* src, size_t src_pitch,
                               size_t row_bytes, size_t rows, void* stream) {
  const char* fn = "csa_copy_rows_async";
  if (row_bytes == 0 || rows == 0) return CSA_OK;
  if (!dst || !src) return fail(CSA_ERR_INVALID_ARG, "%s: NULL address", fn);
  if (dst_pitch < row_bytes || src_pitch < row_bytes)
    return fail(CSA_ERR_INVALID_ARG, "%s: pitches %zu / %zu below the row of %zu bytes", fn,
                dst_pitch, src_pitch, row_bytes);
  cudaError_t e = cudaMemcpy2DAsync(dst, dst_pitch, src, src_pitch, row_bytes, rows,
                                    cudaMemcpyDefault, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  return CSA_OK;
}

size_t csa_workspace_bytes(const csa_params* p, csa_op op, int Q, int64_t N_cap) {
  const char* fn = "csa_workspace_bytes";
  if (check_common(fn, p) != CSA_OK) return 0;
  if (Q < 1 || N_cap < 0) {
    fail(CSA_ERR_INVALID_ARG, "%s: Q=%d, N_cap=%lld", fn, Q, (long long)N_cap);
    return 0;
  }
  switch (op) {
    case CSA_OP_INDEX_TOPK:
      return scores_bytes((int64_t)p->B * Q, N_cap) + 256;
    case CSA_OP_SPARSE_MQA:
    case CSA_OP_DENSE_MQA: {
      int rows = p->B;
      return csa::mqa_workspace_bytes(rows, splits_for(p, op, rows, N_cap), p->H, p->d) + 256;
    }
    case CSA_OP_PREFILL: {
      int rows = Q;
      return scores_bytes(rows, N_cap) +
             csa::mqa_workspace_bytes(rows, splits_for(p, CSA_OP_SPARSE_MQA, rows, N_cap), p->H,
                                      p->d) +
             512;
    }
    case CSA_OP_CSA_DECODE_STEP:
      return scores_bytes(p->B, N_cap) + hist_bytes(p->B) +
             csa::mqa_workspace_bytes(p->B,
                                      splits_for(p, CSA_OP_SPARSE_MQA, p->B, N_cap,
                                                 decode_step_reserve(p, N_cap)),
                                      p->H, p->d) +
             512;
    case CSA_OP_HCA_DECODE_STEP:
      return csa::mqa_workspace_bytes(p->B, splits_for(p, CSA_OP_DENSE_MQA, p->B, N_cap, p->B),
                                      p->H, p->d) +
             256;
    case CSA_OP_HCA_PREFILL: {
      int rows = Q;
      return csa::mqa_workspace_bytes(rows, splits_for(p, CSA_OP_DENSE_MQA, rows, N_cap), p->H,
                                      p->d) +
             256;
    }
  }
  fail(CSA_ERR_INVALID_ARG, "%s: unknown op %d", fn, (int)op);
  return 0;
}

static csa_status compress_common(const char* fn, const csa_params* p, const void* kv_tok,
                                  int64_t L_cap, const int64_t* ctx_len, int64_t ctx_len_value,
                                  const float* w_s, const float* b_pos, const float* gamma,
                                  int64_t first_block, int64_t n_blocks, void* kv_c,
                                  int64_t N_cap, const void* idx_tok, const float* w_s_idx,
                                  const float* b_pos_idx, uint8_t* idx_key, float* idx_scale,
                                  int32_t* dev_status, void* stream,
                                  const int64_t* pos_newest = nullptr, int pdl_head = 0,
                                  int* ctas = nullptr) {
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  REQ_PTR(kv_tok);
  REQ_PTR(kv_c);
  REQ_PTR4(w_s);
  REQ_PTR4(b_pos);
  OPT_PTR4(gamma);
  OPT_PTR4(dev_status);
  if (ctx_len) OPT_PTR(ctx_len);
  if (L_cap < 1 || N_cap < 1)
    return fail(CSA_ERR_INVALID_ARG, "%s: L_cap=%lld N_cap=%lld", fn, (long long)L_cap,
                (long long)N_cap);
  if (first_block < 0 || n_blocks < 0 || first_block + n_blocks > N_cap)
    return fail(CSA_ERR_CAPACITY, "%s: blocks [%lld, %lld) outside N_cap=%lld", fn,
                (long long)first_block, (long long)(first_block + n_blocks), (long long)N_cap);
  if ((p->rope_dim != 0 && p->rope_dim != 32 && p->rope_dim != 64) || p->rope_dim > p->d / 4)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "%s: rope_dim=%d (supported: 0, 32, 64, and at most d/4)", fn, p->rope_dim);
  if (idx_tok) {
    st = check_indexer(fn, p);
    if (st != CSA_OK) return st;
    REQ_PTR(idx_tok);
    REQ_PTR4(w_s_idx);
    REQ_PTR4(b_pos_idx);
    REQ_PTR(idx_key);
    REQ_PTR4(idx_scale);
  }
  csa::CompressLaunch c{};
  c.B = p->B;
  c.d = p->d;
  c.D_I = p->D_I;
  c.m = p->m;
  c.overlap = p->overlap;
  c.entry_offset = p->entry_offset;
  c.L_cap = L_cap;
  c.N_cap = N_cap;
  c.kv_tok = kv_tok;
  c.idx_tok = idx_tok;
  c.ctx_len = ctx_len;
  c.ctx_len_value = ctx_len_value;
  c.w_s = w_s;
  c.b_pos = b_pos;
  c.gamma = gamma;
  c.w_s_idx = w_s_idx;
  c.b_pos_idx = b_pos_idx;
  c.first_block = first_block;
  c.n_blocks = n_blocks;
  c.pos_newest = pos_newest;
  c.kv_c = kv_c;
  c.idx_key = idx_key;
  c.idx_scale = idx_scale;
  c.eps = p->eps;
  c.rope_dim = p->rope_dim;
  fill_inv_freq(p, c.inv_freq);
  c.status = dev_status;
  c.pdl_head = pdl_head;
  if (ctas) *ctas = csa::compress_ctas(c);
  cudaError_t e = csa::launch_compress(c, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

csa_status hca_compress(const csa_params* p, const void* kv_tok, int64_t L_cap,
                        const int64_t* ctx_len, const float* w_s, const float* b_pos,
                        const float* gamma, int64_t first_block, int64_t n_blocks, void* kv_c,
                        int64_t N_cap, int32_t* dev_status, void* stream) {
  const char* fn = "hca_compress";
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  REQ_PTR(ctx_len);
  return compress_common(fn, p, kv_tok, L_cap, ctx_len, 0, w_s, b_pos, gamma, first_block,
                         n_blocks, kv_c, N_cap, nullptr, nullptr, nullptr, nullptr, nullptr,
                         dev_status, stream);
}

csa_status csa_compress(const csa_params* p, const void* kv_tok, int64_t L_cap,
                        const int64_t* ctx_len, const float* w_s, const float* b_pos,
                        const float* gamma, int64_t first_block, int64_t n_blocks, void* kv_c,
                        int64_t N_cap, const void* idx_tok, const float* w_s_idx,
                        const float* b_pos_idx, uint8_t* idx_key, float* idx_scale,
                        int32_t* dev_status, void* stream) {
  const char* fn = "csa_compress";
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  REQ_PTR(ctx_len);
  return compress_common(fn, p, kv_tok, L_cap, ctx_len, 0, w_s, b_pos, gamma, first_block,
                         n_blocks, kv_c, N_cap, idx_tok, w_s_idx, b_pos_idx, idx_key,
                         idx_scale, dev_status, stream);
}

static csa_status index_common(const char* fn, const csa_params* p, int Q,
                               const uint8_t* q_idx, const float* q_scale, const float* w,
                               const uint8_t* idx_key, const float* idx_scale, int64_t N_cap,
                               const int64_t* pos_q, int64_t pos_base, float* scores,
                               int32_t* dev_status, cudaStream_t stream, int chained,
                               const int64_t* safe_pos = nullptr,
                               int64_t safe_fixed = INT64_MAX, uint32_t* hist = nullptr,
                               int reserve_slots = 0) {
  csa::IndexLaunch a{};
  a.chained = chained;
  a.hist = hist;
  a.reserve_slots = reserve_slots;
  a.safe_pos = safe_pos;
  a.safe_fixed = safe_fixed;
  a.B = p->B;
  a.Q = Q;
  a.H_I = p->H_I;
  a.D_I = p->D_I;
  a.m = p->m;
  a.N_cap = N_cap;
  a.q_idx = q_idx;
  a.q_scale = q_scale;
  a.w = w;
  a.key = idx_key;
  a.key_scale = idx_scale;
  a.pos_q = pos_q;
  a.pos_base = pos_base;
  a.scores = scores;
  a.status = dev_status;
  a.num_sms = csa::device_sm_count();
  a.entry_offset = p->entry_offset;
  cudaError_t e = csa::launch_index_scores(a, stream);
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

static csa_status topk_common(const char* fn, const csa_params* p, int Q, const float* scores,
                              int64_t N_cap, const int64_t* pos_q, int64_t pos_base,
                              int32_t* topk_idx, int32_t* topk_cnt, int32_t* dev_status,
                              cudaStream_t stream, int chained, uint32_t* hist = nullptr,
                              int32_t* path = nullptr) {
  csa::TopkLaunch t{};
  t.chained = chained;
  t.hist = hist;
  t.path = path;
  t.rows = p->B * Q;
  t.Q = Q;
  t.m = p->m;
  t.N_cap = N_cap;
  t.scores = scores;
  t.pos_q = pos_q;
  t.pos_base = pos_base;
  t.k = p->k;
  t.idx = topk_idx;
  t.cnt = topk_cnt;
  t.status = dev_status;
  t.entry_offset = p->entry_offset;
  cudaError_t e = csa::launch_topk(t, stream);
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

static csa_status index_topk_common(const char* fn, const csa_params* p, int Q,
                                    const uint8_t* q_idx, const float* q_scale, const float* w,
                                    const uint8_t* idx_key, const float* idx_scale,
                                    int64_t N_cap, const int64_t* pos_q, int64_t pos_base,
                                    int32_t* topk_idx, int32_t* topk_cnt, float* scores,
                                    int32_t* dev_status, cudaStream_t stream, int chained,
                                    const int64_t* safe_pos = nullptr,
                                    int64_t safe_fixed = INT64_MAX, uint32_t* hist = nullptr,
                                    int32_t* path = nullptr, int reserve_slots = 0) {
  csa_status st = index_common(fn, p, Q, q_idx, q_scale, w, idx_key, idx_scale, N_cap, pos_q,
                               pos_base, scores, dev_status, stream, chained, safe_pos,
                               safe_fixed, hist, reserve_slots);
  if (st != CSA_OK) return st;
  return topk_common(fn, p, Q, scores, N_cap, pos_q, pos_base, topk_idx, topk_cnt, dev_status,
                     stream, 1, hist, path);
}

static csa_status check_index_args(const char* fn, const csa_params* p, int Q, int64_t N_cap) {
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  st = check_indexer(fn, p);
  if (st != CSA_OK) return st;
  if (Q < 1) return fail(CSA_ERR_INVALID_ARG, "%s: Q=%d", fn, Q);
  if (N_cap < 1 || N_cap > kMaxIndexEntries)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: N_cap=%lld (supported: 1..%lld)", fn,
                (long long)N_cap, (long long)kMaxIndexEntries);
  if ((int64_t)p->B * Q > 65535)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: B*Q=%lld (supported: <= 65535)", fn,
                (long long)p->B * Q);
  return CSA_OK;
}

csa_status lightning_index_topk(const csa_params* p, int Q, const uint8_t* q_idx,
                                const float* q_scale, const float* w, const uint8_t* idx_key,
                                const float* idx_scale, int64_t N_cap, const int64_t* pos_q,
                                int32_t* topk_idx, int32_t* topk_cnt, float* scores_out,
                                void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  const char* fn = "lightning_index_topk";
  csa_status st = check_index_args(fn, p, Q, N_cap);
  if (st != CSA_OK) return st;
  REQ_PTR(q_idx);
  REQ_PTR4(q_scale);
  REQ_PTR4(w);
  REQ_PTR(idx_key);
  REQ_PTR4(idx_scale);
  REQ_PTR(pos_q);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  OPT_PTR(scores_out);
  OPT_PTR4(dev_status);
  float* scores = scores_out;
  if (!scores) {
    size_t need = csa_workspace_bytes(p, CSA_OP_INDEX_TOPK, Q, N_cap);
    if (!ws || ws_bytes < need)
      return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                  ws ? ws_bytes : (size_t)0);
    if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
    scores = static_cast<float*>(ws);
  }
  return index_topk_common(fn, p, Q, q_idx, q_scale, w, idx_key, idx_scale, N_cap, pos_q, 0,
                           topk_idx, topk_cnt, scores, dev_status,
                           static_cast<cudaStream_t>(stream), 0);
}

csa_status lightning_index_scores(const csa_params* p, int Q, const uint8_t* q_idx,
                                  const float* q_scale, const float* w, const uint8_t* idx_key,
                                  const float* idx_scale, int64_t N_cap, const int64_t* pos_q,
                                  float* scores, int32_t* dev_status, void* stream) {
  const char* fn = "lightning_index_scores";
  csa_status st = check_index_args(fn, p, Q, N_cap);
  if (st != CSA_OK) return st;
  REQ_PTR(q_idx);
  REQ_PTR4(q_scale);
  REQ_PTR4(w);
  REQ_PTR(idx_key);
  REQ_PTR4(idx_scale);
  REQ_PTR(pos_q);
  REQ_PTR(scores);
  OPT_PTR4(dev_status);
  return index_common(fn, p, Q, q_idx, q_scale, w, idx_key, idx_scale, N_cap, pos_q, 0, scores,
                      dev_status, static_cast<cudaStream_t>(stream), 0);
}

csa_status topk_select(const csa_params* p, int Q, const float* scores, int64_t N_cap,
                       const int64_t* pos_q, int32_t* topk_idx, int32_t* topk_cnt,
                       int32_t* dev_status, void* stream) {
  const char* fn = "topk_select";
  csa_status st = check_index_args(fn, p, Q, N_cap);
  if (st != CSA_OK) return st;
  REQ_PTR(scores);
  REQ_PTR(pos_q);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  OPT_PTR4(dev_status);
  return topk_common(fn, p, Q, scores, N_cap, pos_q, 0, topk_idx, topk_cnt, dev_status,
                     static_cast<cudaStream_t>(stream), 0);
}

static csa_status mqa_common(const char* fn, const csa_params* p, csa_op op, int rows, int Q,
                             const void* q, const int64_t* pos_q, int64_t pos_base,
                             const void* kv_c, int64_t N_cap, const int32_t* sel_idx,
                             const int32_t* sel_cnt, const void* kv_tok, int64_t L_cap,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             void* out, float* lse, void* ws, size_t ws_bytes,
                             int32_t* dev_status, cudaStream_t stream, int chained,
                             const int64_t* safe_pos = nullptr, int64_t safe_fixed = 0,
                             int reserve = 0) {
  int splits = splits_for(p, op, rows, N_cap, reserve);
  size_t need = csa::mqa_workspace_bytes(rows, splits, p->H, p->d);
  if (!ws || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                ws ? ws_bytes : (size_t)0);
  if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
  csa::MqaLaunch a{};
  a.B = p->B;
  a.Q = Q;
  a.H = p->H;
  a.D = p->d;
  a.m = p->m;
  a.W = p->window;
  a.rope_dim = p->rope_dim;
  a.N_cap = N_cap;
  a.L_cap = L_cap;
  a.q = q;
  a.pos_q = pos_q;
  a.pos_base = pos_base;
  a.kv_c = kv_c;
  a.sel_idx = sel_idx;
  a.sel_cnt = sel_cnt;
  a.kmax = p->k;
  a.kv_tok = kv_tok;
  a.sink = sink;
  a.gamma_q = gamma_q;
  a.gamma_kv = gamma_kv;
  a.eps = p->eps;
  a.scale = softmax_scale_of(p);
  fill_inv_freq(p, a.inv_freq);
  a.out = out;
  a.lse = lse;
  a.splits = splits;
  a.part_o = ws;
  a.part_ml = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                       round_up((size_t)rows * splits * p->H * p->d * 2, 256));
  a.status = dev_status;
  a.chained = chained;
  a.entry_offset = p->entry_offset;
  a.safe_pos = safe_pos;
  a.safe_fixed = safe_fixed;
  cudaError_t e = csa::launch_mqa(a, stream);
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

static csa_status check_mqa_args(const char* fn, const csa_params* p, const void* q,
                                 const int64_t* pos_q, const void* kv_c, int64_t N_cap,
                                 const void* kv_tok, int64_t L_cap, const float* sink,
                                 const float* gamma_q, const float* gamma_kv, void* out,
                                 float* lse, int32_t* dev_status) {
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  st = check_attention(fn, p);
  if (st != CSA_OK) return st;
  REQ_PTR(q);
  REQ_PTR(pos_q);
  REQ_PTR(kv_c);
  REQ_PTR(kv_tok);
  REQ_PTR4(sink);
  OPT_PTR4(gamma_q);
  OPT_PTR4(gamma_kv);
  REQ_PTR(out);
  OPT_PTR4(lse);
  OPT_PTR4(dev_status);
  if (N_cap < 1 || L_cap < 1 || N_cap > ((int64_t)1 << 31) - 1 || L_cap > ((int64_t)1 << 31) - 1)
    return fail(CSA_ERR_INVALID_ARG, "%s: N_cap=%lld L_cap=%lld", fn, (long long)N_cap,
                (long long)L_cap);
  if ((int64_t)p->B * N_cap > ((int64_t)1 << 31) - 1 || (int64_t)p->B * L_cap > ((int64_t)1 << 31) - 1)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: B*N_cap and B*L_cap must fit in int32 rows", fn);
  return CSA_OK;
}

csa_status sparse_mqa_decode(const csa_params* p, const void* q, const int64_t* pos_q,
                             const void* kv_c, int64_t N_cap, const int32_t* topk_idx,
                             const int32_t* topk_cnt, const void* kv_tok, int64_t L_cap,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             void* out, float* lse, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream) {
  const char* fn = "sparse_mqa_decode";
  csa_status st = check_mqa_args(fn, p, q, pos_q, kv_c, N_cap, kv_tok, L_cap, sink, gamma_q,
                                 gamma_kv, out, lse, dev_status);
  if (st != CSA_OK) return st;
  if (p->k < 1 || p->k > kMaxTopk)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: k=%d (supported: 1..%d)", fn, p->k, kMaxTopk);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  return mqa_common(fn, p, CSA_OP_SPARSE_MQA, p->B, 1, q, pos_q, 0, kv_c, N_cap, topk_idx,
                    topk_cnt, kv_tok, L_cap, sink, gamma_q, gamma_kv, out, lse, ws, ws_bytes,
                    dev_status, static_cast<cudaStream_t>(stream), 0);
}

csa_status dense_mqa_decode(const csa_params* p, const void* q, const int64_t* pos_q,
                            const void* kv_c, int64_t N_cap, const void* kv_tok, int64_t L_cap,
                            const float* sink, const float* gamma_q, const float* gamma_kv,
                            void* out, float* lse, void* ws, size_t ws_bytes,
                            int32_t* dev_status, void* stream) {
  const char* fn = "dense_mqa_decode";
  csa_status st = check_mqa_args(fn, p, q, pos_q, kv_c, N_cap, kv_tok, L_cap, sink, gamma_q,
                                 gamma_kv, out, lse, dev_status);
  if (st != CSA_OK) return st;
  return mqa_common(fn, p, CSA_OP_DENSE_MQA, p->B, 1, q, pos_q, 0, kv_c, N_cap, nullptr,
                    nullptr, kv_tok, L_cap, sink, gamma_q, gamma_kv, out, lse, ws, ws_bytes,
                    dev_status, static_cast<cudaStream_t>(stream), 0);
}

csa_status csa_prefill_chunk(const csa_params* p, int64_t P, int T, const void* kv_tok,
                             const void* idx_tok, int64_t L_cap, const float* w_s,
                             const float* b_pos, const float* gamma, const float* w_s_idx,
                             const float* b_pos_idx, void* kv_c, uint8_t* idx_key,
                             float* idx_scale, int64_t N_cap, const void* q,
                             const uint8_t* q_idx, const float* q_scale, const float* w,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             int32_t* topk_idx, int32_t* topk_cnt, void* out, void* ws,
                             size_t ws_bytes, int32_t* dev_status, void* stream) {
  const char* fn = "csa_prefill_chunk";
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  if (p->B != 1) return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: B=%d (supported: 1)", fn, p->B);
  if (p->entry_offset != 0)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: entry_offset=%lld (supported: 0)", fn,
                (long long)p->entry_offset);
  st = check_indexer(fn, p);
  if (st != CSA_OK) return st;
  st = check_attention(fn, p);
  if (st != CSA_OK) return st;
  if (P < 0 || T < 1 || P % p->m != 0)
    return fail(CSA_ERR_INVALID_ARG, "%s: P=%lld must be a multiple of m=%d, T=%d >= 1", fn,
                (long long)P, p->m, T);
  if (P + T > L_cap)
    return fail(CSA_ERR_CAPACITY, "%s: P+T=%lld exceeds L_cap=%lld", fn, (long long)(P + T),
                (long long)L_cap);
  int64_t nblk_total = (P + T + p->m - 1) / p->m;
  if (nblk_total > N_cap)
    return fail(CSA_ERR_CAPACITY, "%s: %lld compressed entries exceed N_cap=%lld", fn,
                (long long)nblk_total, (long long)N_cap);
  REQ_PTR(q);
  REQ_PTR(q_idx);
  REQ_PTR4(q_scale);
  REQ_PTR4(w);
  REQ_PTR4(sink);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  REQ_PTR(out);
  REQ_PTR(kv_c);
  REQ_PTR(kv_tok);
  size_t need = csa_workspace_bytes(p, CSA_OP_PREFILL, T, N_cap);
  if (!ws || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                ws ? ws_bytes : (size_t)0);
  if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. Compress the blocks the new tokens touch.
  int64_t b0 = P / p->m;
  st = compress_common(fn, p, kv_tok, L_cap, nullptr, P + T, w_s, b_pos, gamma, b0,
                       nblk_total - b0, kv_c, N_cap, idx_tok, w_s_idx, b_pos_idx, idx_key,
                       idx_scale, dev_status, stream);
  if (st != CSA_OK) return st;
  // 2-3. Causal indexer and top-k for the T queries at positions P .. P+T-1.
  float* scores = static_cast<float*>(ws);
  csa_params p1 = *p;
  // The keys of blocks before P/m were written before this call.
  st = index_topk_common(fn, &p1, T, q_idx, q_scale, w, idx_key, idx_scale, N_cap, nullptr, P,
                         topk_idx, topk_cnt, scores, dev_status, s, 1, nullptr, b0);
  if (st != CSA_OK) return st;
  // 4. Sparse MQA per query, each with its own causal window.
  char* rest = static_cast<char*>(ws) + scores_bytes(T, N_cap);
  size_t rest_bytes = ws_bytes - scores_bytes(T, N_cap);
  return mqa_common(fn, p, CSA_OP_SPARSE_MQA, T, T, q, nullptr, P, kv_c, N_cap, topk_idx,
                    topk_cnt, kv_tok, L_cap, sink, gamma_q, gamma_kv, out, nullptr, rest,
                    rest_bytes, dev_status, s, 1);
}

csa_status csa_decode_step(const csa_params* p, const int64_t* pos_q, const void* kv_tok,
                           const void* idx_tok, int64_t L_cap, const float* w_s,
                           const float* b_pos, const float* gamma, const float* w_s_idx,
                           const float* b_pos_idx, void* kv_c, uint8_t* idx_key,
                           float* idx_scale, int64_t N_cap, const void* q, const uint8_t* q_idx,
                           const float* q_scale, const float* w, const float* sink,
                           const float* gamma_q, const float* gamma_kv, int32_t* topk_idx,
                           int32_t* topk_cnt, void* out, float* lse, void* ws, size_t ws_bytes,
                           int32_t* dev_status, void* stream) {
  const char* fn = "csa_decode_step";
  csa_status st = check_index_args(fn, p, 1, N_cap);
  if (st != CSA_OK) return st;
  st = check_mqa_args(fn, p, q, pos_q, kv_c, N_cap, kv_tok, L_cap, sink, gamma_q, gamma_kv, out,
                      lse, dev_status);
  if (st != CSA_OK) return st;
  if (p->k < 1 || p->k > kMaxTopk)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: k=%d (supported: 1..%d)", fn, p->k, kMaxTopk);
  REQ_PTR(idx_tok);
  REQ_PTR(q_idx);
  REQ_PTR4(q_scale);
  REQ_PTR4(w);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  size_t need = csa_workspace_bytes(p, CSA_OP_CSA_DECODE_STEP, 1, N_cap);
  if (!ws || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                ws ? ws_bytes : (size_t)0);
  if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. Each sequence's newest block: the one holding its query token,
  // pooled over the tokens up to it.
  int compress_ctas = 0;
  st = compress_common(fn, p, kv_tok, L_cap, nullptr, 0, w_s, b_pos, gamma, 0, 1, kv_c, N_cap,
                       idx_tok, w_s_idx, b_pos_idx, idx_key, idx_scale, dev_status, stream, pos_q,
                       1, &compress_ctas);
  if (st != CSA_OK) return st;
  // 2-3. Indexer and top-k over each sequence's visible entries (the indexer
  // grid leaves out the slots the compression CTAs hold).  Where the
  // top-k spreads a row over a cluster, the indexer also counts the scores
  // by their top key bits, which seeds the selection.
  float* scores = static_cast<float*>(ws);
  char* hist_at = static_cast<char*>(ws) + scores_bytes(p->B, N_cap);
  uint32_t* hist = csa::topk_uses_hist(p->B, N_cap) ? reinterpret_cast<uint32_t*>(hist_at) : nullptr;
  int32_t* path = hist ? reinterpret_cast<int32_t*>(hist + (size_t)p->B * csa::kScoreHistBins)
                       : nullptr;
  // Only each sequence's newest block is written by this call.
  st = index_topk_common(fn, p, 1, q_idx, q_scale, w, idx_key, idx_scale, N_cap, pos_q, 0,
                         topk_idx, topk_cnt, scores, dev_status, s, 1, pos_q, INT64_MAX, hist,
                         path, compress_ctas);
  if (st != CSA_OK) return st;
  // 4. Sparse MQA over the selection, the window and the sink.
  const size_t head = scores_bytes(p->B, N_cap) + hist_bytes(p->B);
  char* rest = static_cast<char*>(ws) + head;
  return mqa_common(fn, p, CSA_OP_SPARSE_MQA, p->B, 1, q, pos_q, 0, kv_c, N_cap, topk_idx,
                    topk_cnt, kv_tok, L_cap, sink, gamma_q, gamma_kv, out, lse, rest,
                    ws_bytes - head, dev_status, s, 1, nullptr, 0,
                    decode_step_reserve(p, N_cap));
}

csa_status hca_decode_step(const csa_params* p, const int64_t* pos_q, const void* kv_tok,
                           int64_t L_cap, const float* w_s, const float* b_pos,
                           const float* gamma, void* kv_c, int64_t N_cap, const void* q,
                           const float* sink, const float* gamma_q, const float* gamma_kv,
                           void* out, float* lse, void* ws, size_t ws_bytes,
                           int32_t* dev_status, void* stream) {
  const char* fn = "hca_decode_step";
  csa_status st = check_mqa_args(fn, p, q, pos_q, kv_c, N_cap, kv_tok, L_cap, sink, gamma_q,
                                 gamma_kv, out, lse, dev_status);
  if (st != CSA_OK) return st;
  size_t need = csa_workspace_bytes(p, CSA_OP_HCA_DECODE_STEP, 1, N_cap);
  if (!ws || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                ws ? ws_bytes : (size_t)0);
  if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
  // 1. Each sequence's newest block, then 2. dense MQA with window and sink.
  st = compress_common(fn, p, kv_tok, L_cap, nullptr, 0, w_s, b_pos, gamma, 0, 1, kv_c, N_cap,
                       nullptr, nullptr, nullptr, nullptr, nullptr, dev_status, stream, pos_q, 1);
  if (st != CSA_OK) return st;
  // Only each sequence's newest block is written by this call: the older
  // entries stream in while it is compressed.
  return mqa_common(fn, p, CSA_OP_DENSE_MQA, p->B, 1, q, pos_q, 0, kv_c, N_cap, nullptr, nullptr,
                    kv_tok, L_cap, sink, gamma_q, gamma_kv, out, lse, ws, ws_bytes, dev_status,
                    static_cast<cudaStream_t>(stream), 1, pos_q, 0, p->B);
}

csa_status hca_prefill_chunk(const csa_params* p, int64_t P, int T, const void* kv_tok,
                             int64_t L_cap, const float* w_s, const float* b_pos,
                             const float* gamma, void* kv_c, int64_t N_cap, const void* q,
                             const float* sink, const float* gamma_q, const float* gamma_kv,
                             void* out, float* lse, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream) {
  const char* fn = "hca_prefill_chunk";
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  if (p->B != 1) return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: B=%d (supported: 1)", fn, p->B);
  if (p->entry_offset != 0)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: entry_offset=%lld (supported: 0)", fn,
                (long long)p->entry_offset);
  st = check_attention(fn, p);
  if (st != CSA_OK) return st;
  if (P < 0 || T < 1 || P % p->m != 0)
    return fail(CSA_ERR_INVALID_ARG, "%s: P=%lld must be a multiple of m=%d, T=%d >= 1", fn,
                (long long)P, p->m, T);
  if (T > 65535) return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: T=%d (supported: <= 65535)", fn, T);
  if (P + T > L_cap)
    return fail(CSA_ERR_CAPACITY, "%s: P+T=%lld exceeds L_cap=%lld", fn, (long long)(P + T),
                (long long)L_cap);
  if (L_cap > ((int64_t)1 << 31) - 1 || N_cap > ((int64_t)1 << 31) - 1)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: N_cap and L_cap must fit in int32 rows", fn);
  const int64_t nblk_total = (P + T + p->m - 1) / p->m;
  if (nblk_total > N_cap)
    return fail(CSA_ERR_CAPACITY, "%s: %lld compressed entries exceed N_cap=%lld", fn,
                (long long)nblk_total, (long long)N_cap);
  REQ_PTR(q);
  REQ_PTR4(sink);
  OPT_PTR4(gamma_q);
  OPT_PTR4(gamma_kv);
  REQ_PTR(out);
  OPT_PTR4(lse);
  size_t need = csa_workspace_bytes(p, CSA_OP_HCA_PREFILL, T, N_cap);
  if (!ws || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                ws ? ws_bytes : (size_t)0);
  if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
  // 1. Compress the blocks the new tokens touch (ctx_len = P+T for all).
  const int64_t b0 = P / p->m;
  st = compress_common(fn, p, kv_tok, L_cap, nullptr, P + T, w_s, b_pos, gamma, b0,
                       nblk_total - b0, kv_c, N_cap, nullptr, nullptr, nullptr, nullptr, nullptr,
                       dev_status, stream);
  if (st != CSA_OK) return st;
  // 2. Dense MQA per query over its visible entries and its causal window
  // (entries below b0 were written before the call).
  return mqa_common(fn, p, CSA_OP_DENSE_MQA, T, T, q, nullptr, P, kv_c, N_cap, nullptr, nullptr,
                    kv_tok, L_cap, sink, gamma_q, gamma_kv, out, lse, ws, ws_bytes, dev_status,
                    static_cast<cudaStream_t>(stream), 1, nullptr, b0);
}

// ------------------------------------------------- grouped output projection --
static csa_status check_proj(const char* fn, int T, int H, int D, int g, int d_g, int d_model) {
  if (T < 1 || H < 1 || D < 1 || g < 1 || d_g < 1 || d_model < 1)
    return fail(CSA_ERR_INVALID_ARG, "%s: T=%d H=%d D=%d g=%d d_g=%d d=%d must be >= 1", fn, T, H, D,
                g, d_g, d_model);
  if (H % g)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: g=%d must divide H=%d", fn, g, H);
  const int64_t k1 = (int64_t)(H / g) * D, k2 = (int64_t)g * d_g;
  if (k1 % 64 || k2 % 64 || d_g % 128 || d_model % 128 || k1 > (1 << 20) || k2 > (1 << 20) ||
      (int64_t)H * D > ((int64_t)1 << 24) || d_model > (1 << 20))
    return fail(CSA_ERR_UNSUPPORTED_SHAPE,
                "%s: need (H/g)*D and g*d_g multiples of 64, d_g and d multiples of 128", fn);
  if ((int64_t)T > (int64_t)65535 * 256)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: T=%d too large", fn, T);
  return CSA_OK;
}

struct ProjPlan {
  int64_t k1, n1, k2;
  int s1, s2;
  size_t y_bytes, part_bytes;
};

static ProjPlan proj_plan(int T, int H, int D, int g, int d_g, int d_model) {
  ProjPlan pl{};
  pl.k1 = (int64_t)(H / g) * D;
  pl.n1 = (int64_t)g * d_g;
  pl.k2 = pl.n1;
  const int sms = csa::device_sm_count();
  pl.s1 = csa::proj_choose_splits(T, d_g, g, (int)pl.k1, sms);
  pl.s2 = csa::proj_choose_splits(T, d_model, 1, (int)pl.k2, sms);
  pl.y_bytes = round_up((size_t)T * pl.n1 * 2, 256);
  size_t p1 = pl.s1 > 1 ? (size_t)pl.s1 * T * pl.n1 * 4 : 0;
  size_t p2 = pl.s2 > 1 ? (size_t)pl.s2 * T * d_model * 4 : 0;
  pl.part_bytes = round_up(p1 > p2 ? p1 : p2, 256);
  return pl;
}

size_t grouped_out_proj_workspace_bytes(int T, int H, int D, int g, int d_g, int d_model) {
  if (check_proj("grouped_out_proj_workspace_bytes", T, H, D, g, d_g, d_model) != CSA_OK) return 0;
  const ProjPlan pl = proj_plan(T, H, D, g, d_g, d_model);
  return pl.y_bytes + pl.part_bytes + 256;
}

csa_status grouped_out_proj(int T, int H, int D, int g, int d_g, int d_model, const void* o,
                            const void* w_g, const void* w_o, void* y, void* z, void* ws,
                            size_t ws_bytes, int32_t* dev_status, void* stream) {
  const char* fn = "grouped_out_proj";
  csa_status st = check_proj(fn, T, H, D, g, d_g, d_model);
  if (st != CSA_OK) return st;
  REQ_PTR(o);
  REQ_PTR(w_g);
  REQ_PTR(w_o);
  OPT_PTR(y);
  REQ_PTR(z);
  OPT_PTR4(dev_status);
  const ProjPlan pl = proj_plan(T, H, D, g, d_g, d_model);
  const size_t need = pl.y_bytes + pl.part_bytes + 256;
  if (!ws || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                ws ? ws_bytes : (size_t)0);
  if (!aligned16(ws)) return fail(CSA_ERR_INVALID_ARG, "%s: ws is not 16-byte aligned", fn);
  char* wsb = static_cast<char*>(ws);
  void* ybuf = y ? y : static_cast<void*>(wsb);
  float* part = reinterpret_cast<float*>(wsb + pl.y_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. Per group j: y[:, j*d_g .. ] = x_j W_g[j]^T, x_j = heads j*H/g .. of o.
  csa::ProjGemm a{};
  a.a = o;
  a.lda = (int64_t)H * D;
  a.w = w_g;
  a.w_rows = pl.n1;
  a.K = (int)pl.k1;
  a.N = d_g;
  a.groups = g;
  a.T = T;
  a.splits = pl.s1;
  a.c = ybuf;
  a.ldc = (int)pl.n1;
  a.part = part;
  a.status = dev_status;
  a.chained = 0;
  cudaError_t e = csa::launch_proj_gemm(a, s);
  if (e != cudaSuccess) return cuda_fail(fn, e);
  // 2. z = y W_o^T.
  csa::ProjGemm b{};
  b.a = ybuf;
  b.lda = pl.n1;
  b.w = w_o;
  b.w_rows = d_model;
  b.K = (int)pl.k2;
  b.N = d_model;
  b.groups = 1;
  b.T = T;
  b.splits = pl.s2;
  b.c = z;
  b.ldc = d_model;
  b.part = part;
  b.status = dev_status;
  b.chained = 1;
  e = csa::launch_proj_gemm(b, s);
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

// ----------------------------------------- context split over several devices --
csa_status csa_shard_candidates(const csa_params* p, int Q, const float* scores, int64_t N_cap,
                                const int32_t* topk_idx, const int32_t* topk_cnt,
                                float* cand_score, int32_t* cand_idx, int32_t* dev_status,
                                void* stream) {
  const char* fn = "csa_shard_candidates";
  csa_status st = check_index_args(fn, p, Q, N_cap);
  if (st != CSA_OK) return st;
  REQ_PTR(scores);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  REQ_PTR4(cand_score);
  REQ_PTR4(cand_idx);
  OPT_PTR4(dev_status);
  if (p->entry_offset + N_cap > 0x7FFFFFFF)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: sequence indices must fit in int32", fn);
  cudaError_t e = csa::launch_shard_candidates(scores, N_cap, topk_idx, topk_cnt, p->B * Q, p->k,
                                               p->entry_offset, cand_score, cand_idx,
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

csa_status csa_merge_candidates(const csa_params* p, int Q, int G, const float* cand_score,
                                const int32_t* cand_idx, const int32_t* cand_cnt, int64_t N_cap,
                                int32_t* topk_idx, int32_t* topk_cnt, int32_t* local_idx,
                                int32_t* local_cnt, int32_t* dev_status, void* stream) {
  const char* fn = "csa_merge_candidates";
  csa_status st = check_index_args(fn, p, Q, N_cap);
  if (st != CSA_OK) return st;
  if (G < 1 || G > 64 || (size_t)G * p->k * 8 > 190 * 1024)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: G=%d (supported: 1..64 with G*k <= 24320)", fn, G);
  REQ_PTR4(cand_score);
  REQ_PTR4(cand_idx);
  REQ_PTR4(cand_cnt);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  REQ_PTR(local_idx);
  REQ_PTR4(local_cnt);
  OPT_PTR4(dev_status);
  csa::MergeLaunch a{};
  a.G = G;
  a.rows = p->B * Q;
  a.k = p->k;
  a.cand_s = cand_score;
  a.cand_i = cand_idx;
  a.cand_c = cand_cnt;
  a.idx = topk_idx;
  a.cnt = topk_cnt;
  a.lo = p->entry_offset;
  a.hi = p->entry_offset + N_cap;
  a.local_idx = local_idx;
  a.local_cnt = local_cnt;
  a.status = dev_status;
  a.chained = 0;
  cudaError_t e = csa::launch_merge_candidates(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

csa_status sparse_mqa_partials(const csa_params* p, int splits, const void* q, const int64_t* pos_q,
                               const void* kv_c, int64_t N_cap, const int32_t* topk_idx,
                               const int32_t* topk_cnt, const void* kv_tok, int64_t L_cap,
                               const float* gamma_q, const float* gamma_kv, void* part_o,
                               float* part_ml, int32_t* dev_status, void* stream) {
  const char* fn = "sparse_mqa_partials";
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  st = check_attention(fn, p);
  if (st != CSA_OK) return st;
  if (p->k < 1 || p->k > kMaxTopk)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: k=%d (supported: 1..%d)", fn, p->k, kMaxTopk);
  if (splits < 1 || splits > 64)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: splits=%d (supported: 1..64)", fn, splits);
  REQ_PTR(q);
  REQ_PTR(pos_q);
  REQ_PTR(kv_c);
  REQ_PTR(kv_tok);
  REQ_PTR(topk_idx);
  REQ_PTR4(topk_cnt);
  OPT_PTR4(gamma_q);
  OPT_PTR4(gamma_kv);
  REQ_PTR(part_o);
  REQ_PTR4(part_ml);
  OPT_PTR4(dev_status);
  if (N_cap < 1 || L_cap < 1 || (int64_t)p->B * N_cap > ((int64_t)1 << 31) - 1 ||
      (int64_t)p->B * L_cap > ((int64_t)1 << 31) - 1)
    return fail(CSA_ERR_INVALID_ARG, "%s: N_cap=%lld L_cap=%lld", fn, (long long)N_cap,
                (long long)L_cap);
  csa::MqaLaunch a{};
  a.B = p->B;
  a.Q = 1;
  a.H = p->H;
  a.D = p->d;
  a.m = p->m;
  a.W = p->window;
  a.rope_dim = p->rope_dim;
  a.N_cap = N_cap;
  a.L_cap = L_cap;
  a.q = q;
  a.pos_q = pos_q;
  a.kv_c = kv_c;
  a.sel_idx = topk_idx;
  a.sel_cnt = topk_cnt;
  a.kmax = p->k;
  a.kv_tok = kv_tok;
  a.sink = nullptr;
  a.gamma_q = gamma_q;
  a.gamma_kv = gamma_kv;
  a.eps = p->eps;
  a.scale = softmax_scale_of(p);
  fill_inv_freq(p, a.inv_freq);
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.splits = splits;
  a.status = dev_status;
  a.entry_offset = p->entry_offset;
  a.emit_partials = 1;
  cudaError_t e = csa::launch_mqa(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

csa_status mqa_merge_partials(const csa_params* p, int splits, const void* part_o,
                              const float* part_ml, const int64_t* pos_q, const float* sink,
                              void* out, float* lse, int32_t* dev_status, void* stream) {
  const char* fn = "mqa_merge_partials";
  csa_status st = check_common(fn, p);
  if (st != CSA_OK) return st;
  st = check_attention(fn, p);
  if (st != CSA_OK) return st;
  if (splits < 1 || splits > 4096)
    return fail(CSA_ERR_UNSUPPORTED_SHAPE, "%s: splits=%d (supported: 1..4096)", fn, splits);
  REQ_PTR(part_o);
  REQ_PTR4(part_ml);
  REQ_PTR(pos_q);
  REQ_PTR4(sink);
  REQ_PTR(out);
  OPT_PTR4(lse);
  OPT_PTR4(dev_status);
  csa::MqaLaunch a{};
  a.B = p->B;
  a.Q = 1;
  a.H = p->H;
  a.D = p->d;
  a.rope_dim = p->rope_dim;
  a.pos_q = pos_q;
  a.sink = sink;
  fill_inv_freq(p, a.inv_freq);
  a.out = out;
  a.lse = lse;
  a.part_o = const_cast<void*>(part_o);
  a.part_ml = const_cast<float*>(part_ml);
  a.splits = splits;
  a.status = dev_status;
  a.chained = 0;
  cudaError_t e = csa::launch_mqa_merge(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(fn, e);
  return CSA_OK;
}

}  // extern "C"
