// Reference oracle for the DeepSeek-V4 hybrid-attention hot path (CSA / HCA).
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
// this file: only the test suite, the smoke check and the benchmark's CPU
// baseline leg do.  It is a plain, slow, fp64 restatement of the method, kept
// deliberately free of blocking, fusion or reordering, so that each function
// can be checked against the source pages by eye.  It shares no code, header,
// table or constant with the CUDA library.
//
// Sources (pages are cited by title and section):
//   [P2]  agentupdate.ai, "DeepSeek V4 technical report ..." (Chinese),
//         section "混合注意力机制" (hybrid attention), CSA steps 1-4 and HCA.
//   [P3]  webconsulting.at, "DeepSeek V4-Pro Architecture: KV Cache
//         Compression and Hyper-Connections Visualised", "Key points" and
//         "Dual Compression and Indexing".
//   [P5]  lizeman.github.io llm-arch-kb, "DeepSeek V4-Pro", section
//         "What's new in V4 / 1. Hybrid attention: CSA + HCA replace MLA".
//
// Where the pages leave a form open, the reading used is stated beside the
// code (pooling weight form, indexer score form, tie rule, RoPE layout and
// base, entry position, joint window+compressed softmax, eps and scale).
//
// Parity status: every function below is pinned by tests/test_oracle_pins.py
// against closed forms, library routines, invariants or brute force.  The
// literal DeepSeek numerics (trained weights) are not available anywhere, so
// what is pinned is this specification, not the production model.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- threads ---
// Static split of [0, n) over worker threads.  The work per index is
// independent, so results do not depend on the thread count.
void parallel_for(int64_t n, int nthreads, const std::function<void(int64_t)>& fn) {
  if (n <= 0) return;
  int t = nthreads > 0 ? nthreads : (int)std::thread::hardware_concurrency();
  if (t < 1) t = 1;
  if (t > n) t = (int)n;
  if (t == 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  for (int w = 0; w < t; ++w) {
    pool.emplace_back([&]() {
      for (;;) {
        int64_t i = next.fetch_add(1);
        if (i >= n) break;
        fn(i);
      }
    });
  }
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------- number formats ---
// bfloat16: the upper 16 bits of an IEEE binary32.  Decoding is exact.
double bf16_decode(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Round an fp64 value to the nearest bfloat16 (ties to even), directly from
// fp64 (no intermediate fp32 rounding).  8 significant bits, exponent range
// of binary32, subnormals down to 2^-133, overflow to infinity.
uint16_t bf16_encode(double x) {
  if (std::isnan(x)) return 0x7FC0;
  uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  double a = std::fabs(x);
  if (a == 0.0) return sign;
  int e;
  std::frexp(a, &e);          // a = f * 2^e, f in [0.5, 1)  ->  a in [2^(e-1), 2^e)
  int ex = e - 1;             // a in [2^ex, 2^(ex+1))
  if (ex < -126) ex = -126;   // subnormal range has the spacing of 2^-126 binade
  double ulp = std::ldexp(1.0, ex - 7);
  double n = std::nearbyint(a / ulp);  // exact scaling; default mode is ties-to-even
  double r = n * ulp;
  const double maxv = std::ldexp(255.0, 127 - 7);  // (2 - 2^-7) * 2^127
  if (r > maxv) return sign | 0x7F80;              // +-inf
  float rf = (float)r;                             // exact: r has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &rf, 4);
  return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

// OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits;
// no infinities; S.1111.111 is NaN; largest finite magnitude 448.
double e4m3_decode(uint8_t c) {
  int s = (c >> 7) & 1, E = (c >> 3) & 15, M = c & 7;
  double v;
  if (E == 15 && M == 7) return std::numeric_limits<double>::quiet_NaN();
  if (E == 0) v = std::ldexp((double)M, -9);            // M/8 * 2^-6
  else v = std::ldexp(8.0 + M, E - 10);                 // (1 + M/8) * 2^(E-7)
  return s ? -v : v;
}

// Round a binary32 value to E4M3 with ties to even and saturation to +-448
// (the "satfinite" rule).  NaN maps to the NaN code.
uint8_t e4m3_encode(float xf) {
  double x = (double)xf;
  if (std::isnan(x)) return 0x7F;
  uint8_t s = std::signbit(x) ? 0x80 : 0;
  double a = std::fabs(x);
  if (a >= 448.0) return s | 0x7E;                      // saturate
  // Grid spacing: 2^-9 below the smallest normal 2^-6, else 2^(ex-3).
  int ex = -6;
  if (a >= std::ldexp(1.0, -6)) {
    int e;
    std::frexp(a, &e);
    ex = e - 1;
  }
  double ulp = std::ldexp(1.0, ex - 3);
  double n = std::nearbyint(a / ulp);
  double r = n * ulp;
  if (r >= 448.0) return s | 0x7E;
  // Re-encode r exactly.
  uint8_t code = 0;
  if (r < std::ldexp(1.0, -6)) {
    code = (uint8_t)std::lround(r / std::ldexp(1.0, -9));  // subnormal: M * 2^-9
  } else {
    int e;
    std::frexp(r, &e);
    int E = (e - 1) + 7;
    int M = (int)std::lround((r / std::ldexp(1.0, e - 1) - 1.0) * 8.0);
    code = (uint8_t)((E << 3) | M);
  }
  return s | code;
}

// ------------------------------------------------------------------- RoPE ---
// [P5] rotates only the last 64 dimensions of query, KV and output.
// Reading: rotate-half pairing over the last r dimensions, (D-r+j, D-r+j+r/2) for
// j < r/2, frequency theta_j = base^(-2j/r), angle = position * theta_j.
// The pages give neither the pairing nor the base; 10000 is used.  A
// caller-given table freq[j] replaces base^(-2j/r) (a context-extension
// rescaling such as YaRN changes only these per-pair frequencies).
void rope_apply(double* v, int D, int r, double base, const double* freq, double pos,
                double sign) {
  if (r <= 0) return;
  int b0 = D - r, half = r / 2;
  for (int j = 0; j < half; ++j) {
    double theta = freq ? freq[j] : std::pow(base, -2.0 * j / (double)r);
    double ang = sign * pos * theta;
    double c = std::cos(ang), s = std::sin(ang);
    double x1 = v[b0 + j], x2 = v[b0 + j + half];
    v[b0 + j] = x1 * c - x2 * s;
    v[b0 + j + half] = x2 * c + x1 * s;
  }
}

void rms_norm(double* v, int D, const float* gamma, double eps) {
  double ss = 0.0;
  for (int d = 0; d < D; ++d) ss += v[d] * v[d];
  double inv = 1.0 / std::sqrt(ss / D + eps);
  for (int d = 0; d < D; ++d) v[d] = v[d] * inv * (gamma ? (double)gamma[d] : 1.0);
}

}  // namespace

extern "C" {

int orc_abi_version(void) { return 4; }

double orc_bf16_decode(uint16_t h) { return bf16_decode(h); }
uint16_t orc_bf16_encode(double x) { return bf16_encode(x); }
double orc_e4m3_decode(uint8_t c) { return e4m3_decode(c); }
uint8_t orc_e4m3_encode(float x) { return e4m3_encode(x); }

void orc_bf16_encode_array(int64_t n, const double* x, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_encode(x[i]);
}

// --------------------------------------------------------- a1: compression ---
// [P2] CSA step 1 merges each run of m token KV vectors into one entry with
// learned, attention-like weights; [P2] HCA uses m' = 128 with no overlap
// between blocks; [P3] describes the merge as a learned weighted average;
// [P5] gives m = 4 for CSA and m' = 128 for HCA.
//
// Reading (weight form not given by the pages): for block i the present
// tokens t = i*m - overlap + j (j < m + overlap, 0 <= t < ctx_len) get scores
// s_j = c_t . w_s + b_pos[j]; the weights are the softmax of s over the
// present j; the pooled vector is the weighted sum, followed by RMSNorm with
// gain gamma (this is the KV side of the QK-Norm that [P5] places on the one
// shared compressed KV head).  overlap = 0: blocks do not overlap ([P2] says
// so for HCA).  overlap > 0 (a CSA variant: [P2] states "no overlap" for HCA
// only, and gives no overlap rule): entry i also pools the last `overlap`
// tokens of block i-1, i.e. a window of m + overlap tokens at stride m,
// clipped at the sequence start.  A block with no present token of its own
// range is not written.  `normalize` = 0 skips the RMSNorm (a test hook only).
//
// Storage reading for the KV stream ([P5] puts RoPE on the last dimensions
// of the KV; where it is applied is not fixed): the entry is stored already
// rotated to its own position (i+1)*m - 1, the last token of the block, so
// that attention uses it as stored.  rope_dim = 0 stores it unrotated (the
// indexer stream, which the pages do not rotate).
void orc_pool(int B, int64_t L_cap, int d, int m, int overlap, const uint16_t* tok,
              const int64_t* ctx_len, const float* w_s, const float* b_pos, const float* gamma,
              double eps, int normalize, int rope_dim, double rope_base, const double* rope_freq,
              int64_t first_block, int64_t n_blocks, int64_t N_cap, double* out,
              uint8_t* written, int nthreads) {
  parallel_for((int64_t)B * n_blocks, nthreads, [&](int64_t w) {
    int64_t b = w / n_blocks, i = first_block + w % n_blocks;
    if (i < 0 || i >= N_cap) return;
    int64_t L = std::min<int64_t>(ctx_len[b], L_cap);
    if (L <= i * m) return;  // no token of the block's own range yet
    // Window positions j = 0 .. m+overlap-1 hold token t = i*m - overlap + j.
    int64_t t0 = i * m - overlap;
    std::vector<int> js;
    for (int j = 0; j < m + overlap; ++j)
      if (t0 + j >= 0 && t0 + j < L) js.push_back(j);
    std::vector<double> s(js.size());
    double smax = -std::numeric_limits<double>::infinity();
    for (size_t q = 0; q < js.size(); ++q) {
      const uint16_t* row = tok + ((int64_t)b * L_cap + t0 + js[q]) * d;
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += bf16_decode(row[k]) * (double)w_s[k];
      s[q] = acc + (double)b_pos[js[q]];
      smax = std::max(smax, s[q]);
    }
    double z = 0.0;
    for (size_t q = 0; q < js.size(); ++q) z += std::exp(s[q] - smax);
    std::vector<double> p(d, 0.0);
    for (size_t q = 0; q < js.size(); ++q) {
      double a = std::exp(s[q] - smax) / z;
      const uint16_t* row = tok + ((int64_t)b * L_cap + t0 + js[q]) * d;
      for (int k = 0; k < d; ++k) p[k] += a * bf16_decode(row[k]);
    }
    if (normalize) rms_norm(p.data(), d, gamma, eps);
    rope_apply(p.data(), d, rope_dim, rope_base, rope_freq, (double)((i + 1) * m - 1), +1.0);
    double* o = out + ((int64_t)b * N_cap + i) * d;
    for (int k = 0; k < d; ++k) o[k] = p[k];
    if (written) written[(int64_t)b * N_cap + i] = 1;
  });
}

// Indexer-key storage ([P3]: the indexer runs in low precision): each row is
// scaled by amax/448 and rounded to E4M3.  The decision is taken in binary32,
// as the kernel takes it: x32 = (float)x, amax over the row in binary32,
// scale = amax / 448 in binary32 (1 when amax is 0), code = E4M3(x32 / scale).
void orc_quant_rows_e4m3(int64_t rows, int dim, const double* x, uint8_t* codes, float* scale) {
  for (int64_t r = 0; r < rows; ++r) {
    const double* xr = x + r * dim;
    float amax = 0.0f;
    for (int k = 0; k < dim; ++k) amax = std::max(amax, std::fabs((float)xr[k]));
    float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int k = 0; k < dim; ++k) codes[r * dim + k] = e4m3_encode((float)xr[k] / sc);
    scale[r] = sc;
  }
}

// ------------------------------------------------------- a2: indexer score ---
// [P2] CSA step 2 / [P5] (64 indexer heads of dimension 128): a light scorer
// of each query against every compressed entry.  Reading (the DSA form
// the pages cite): score_i = sum_h w_h * ReLU(q_h . k_i), with q and k the
// dequantised E4M3 values (code * scale).  Only entries visible to the query
// are scored: i < floor((pos+1)/m), because [P5] notes that compressed
// attention cannot see into the block still being filled.  Other entries get
// -inf.
void orc_index_scores(int B, int Q, int H_I, int D_I, int m, const uint8_t* q_idx,
                      const float* q_scale, const float* w, const uint8_t* key,
                      const float* key_scale, int64_t N_cap, const int64_t* pos_q,
                      double* scores, int nthreads) {
  double lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = e4m3_decode((uint8_t)c);
  const int64_t CH = 4096;
  int64_t nch = (N_cap + CH - 1) / CH;
  parallel_for((int64_t)B * Q * nch, nthreads, [&](int64_t w_) {
    int64_t bq = w_ / nch, ch = w_ % nch;
    int64_t b = bq / Q;
    int64_t nvis = (pos_q[bq] + 1) / m;
    std::vector<double> qf((size_t)H_I * D_I);
    for (int h = 0; h < H_I; ++h)
      for (int k = 0; k < D_I; ++k)
        qf[(size_t)h * D_I + k] =
            lut[q_idx[(bq * H_I + h) * D_I + k]] * (double)q_scale[bq * H_I + h];
    std::vector<double> kf(D_I);
    for (int64_t i = ch * CH; i < std::min(N_cap, (ch + 1) * CH); ++i) {
      double* out = scores + bq * N_cap + i;
      if (i >= nvis) {
        *out = -std::numeric_limits<double>::infinity();
        continue;
      }
      const uint8_t* kr = key + (b * N_cap + i) * D_I;
      for (int k = 0; k < D_I; ++k) kf[k] = lut[kr[k]] * (double)key_scale[b * N_cap + i];
      double sc = 0.0;
      for (int h = 0; h < H_I; ++h) {
        double dot = 0.0;
        for (int k = 0; k < D_I; ++k) dot += qf[(size_t)h * D_I + k] * kf[k];
        sc += (double)w[bq * H_I + h] * std::max(0.0, dot);
      }
      *out = sc;
    }
  });
}

// --------------------------------------------------------------- a3: top-k ---
// [P2] CSA step 2 keeps the k best-scoring blocks per query; [P5] sets
// k = 1024.  Tie rule (not on the pages): rank by score descending,
// then index ascending; NaN ranks below every number; -0 equals +0.  The
// first min(k, n_vis) ranked entries are returned as ascending indices,
// padded with -1.  n_vis[bq] bounds the candidates (entries 0..n_vis-1).
void orc_topk(int64_t BQ, int64_t N_cap, const double* scores, const int64_t* n_vis, int k,
              int32_t* idx, int32_t* cnt, int nthreads) {
  parallel_for(BQ, nthreads, [&](int64_t bq) {
    int64_t n = std::min<int64_t>(std::max<int64_t>(n_vis[bq], 0), N_cap);
    const double* s = scores + bq * N_cap;
    std::vector<int64_t> order(n);
    for (int64_t i = 0; i < n; ++i) order[i] = i;
    auto before = [&](int64_t a, int64_t b) {
      double sa = s[a], sb = s[b];
      bool na = std::isnan(sa), nb = std::isnan(sb);
      if (na != nb) return nb;            // the number ranks above the NaN
      if (!na && sa != sb) return sa > sb;
      return a < b;
    };
    std::sort(order.begin(), order.end(), before);
    int64_t c = std::min<int64_t>(k, n);
    std::vector<int64_t> sel(order.begin(), order.begin() + c);
    std::sort(sel.begin(), sel.end());
    for (int j = 0; j < k; ++j) idx[bq * k + j] = j < c ? (int32_t)sel[j] : -1;
    cnt[bq] = (int32_t)c;
  });
}

// --------------------------------------------- a4/a5: shared-KV MQA + sink ---
// [P2] CSA step 3: multi-query attention over the selected compressed
// entries; [P2]/[P5] HCA: dense attention over all compressed entries.
// [P5] supplementary mechanisms: a sliding-window branch of the n_win most
// recent uncompressed tokens, and a learnable per-head sink logit added to
// the softmax denominator.  [P5] QK-Norm: RMSNorm on each query head and on
// the KV head before the dot product.  [P5] RoPE on the last r dimensions of
// query, KV and output, with inverse RoPE on the output.
//
// Readings: window and compressed entries share one softmax and are not
// de-duplicated; the window holds tokens max(0, pos-W+1) .. pos (the query
// token itself included); compressed entries are used as stored: their
// pooling RMSNorm is the KV norm and they are stored already rotated to
// their position (i+1)*m - 1 (see orc_pool); window tokens get RMSNorm with
// gamma_kv and the rotation to their position t; the logit scale is `scale`
// (1/sqrt(D) in the library); K = V = the roped vector; the output is
// RoPE(-pos) of the normalised weighted sum.  A sink of -inf drops out; a
// sink of +inf gives a zero output.
//
// sel_idx == nullptr selects the dense form (entries 0..n_vis-1); otherwise
// entries sel_idx[bq, 0..sel_cnt[bq]) are used (negative ones are skipped).
// kv_tok holds token rows tok_base .. tok_base+L_cap-1 (a window of a long
// stream; pure storage offset, no effect on the arithmetic).
void orc_mqa(int B, int Q, int H, int D, int m, int W, int rope_dim, double rope_base,
             const double* rope_freq, const uint16_t* q, const int64_t* pos_q, const uint16_t* kv_c, int64_t N_cap,
             const int32_t* sel_idx, const int32_t* sel_cnt, int kmax, const uint16_t* kv_tok,
             int64_t L_cap, int64_t tok_base, const float* sink, const float* gamma_q,
             const float* gamma_kv, double eps, double scale, double* out, double* lse,
             int nthreads) {
  const double inf = std::numeric_limits<double>::infinity();
  for (int64_t bq = 0; bq < (int64_t)B * Q; ++bq) {
    int64_t b = bq / Q;
    int64_t pos = pos_q[bq];
    int64_t nvis = std::min<int64_t>((pos + 1) / m, N_cap);
    // Gather the KV set once per query (shared by all heads).
    std::vector<int64_t> ent;
    if (sel_idx == nullptr) {
      for (int64_t i = 0; i < nvis; ++i) ent.push_back(i);
    } else {
      for (int j = 0; j < sel_cnt[bq]; ++j) {
        int64_t i = sel_idx[bq * kmax + j];
        if (i >= 0 && i < nvis) ent.push_back(i);
      }
    }
    int64_t w0 = std::max<int64_t>(0, pos - W + 1);
    int64_t nwin = W > 0 ? pos - w0 + 1 : 0;
    int64_t T = (int64_t)ent.size() + nwin;
    std::vector<double> kv((size_t)T * D);
    for (int64_t j = 0; j < T; ++j) {
      double* v = kv.data() + j * D;
      if (j < (int64_t)ent.size()) {
        int64_t i = ent[j];
        const uint16_t* row = kv_c + (b * N_cap + i) * D;
        for (int d = 0; d < D; ++d) v[d] = bf16_decode(row[d]);  // stored rotated
      } else {
        int64_t t = w0 + (j - (int64_t)ent.size());
        const uint16_t* row = kv_tok + (b * L_cap + (t - tok_base)) * D;
        for (int d = 0; d < D; ++d) v[d] = bf16_decode(row[d]);
        rms_norm(v, D, gamma_kv, eps);
        rope_apply(v, D, rope_dim, rope_base, rope_freq, (double)t, +1.0);
      }
    }
    parallel_for(H, nthreads, [&](int64_t h) {
      std::vector<double> qh(D);
      const uint16_t* qr = q + (bq * H + h) * D;
      for (int d = 0; d < D; ++d) qh[d] = bf16_decode(qr[d]);
      rms_norm(qh.data(), D, gamma_q, eps);
      rope_apply(qh.data(), D, rope_dim, rope_base, rope_freq, (double)pos, +1.0);
      std::vector<double> s(T);
      double smax = -inf;
      for (int64_t j = 0; j < T; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qh[d] * kv[j * D + d];
        s[j] = acc * scale;
        smax = std::max(smax, s[j]);
      }
      double z = (double)sink[h];
      double* o = out + (bq * H + h) * D;
      if (z == inf) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (lse) lse[bq * H + h] = inf;
        return;
      }
      double M = std::max(smax, z);
      if (M == -inf) {  // empty KV set and a sink of -inf
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (lse) lse[bq * H + h] = -inf;
        return;
      }
      double L = (z == -inf) ? 0.0 : std::exp(z - M);
      std::vector<double> acc(D, 0.0);
      for (int64_t j = 0; j < T; ++j) {
        double p = std::exp(s[j] - M);
        L += p;
        for (int d = 0; d < D; ++d) acc[d] += p * kv[j * D + d];
      }
      for (int d = 0; d < D; ++d) acc[d] /= L;
      rope_apply(acc.data(), D, rope_dim, rope_base, rope_freq, (double)pos, -1.0);
      for (int d = 0; d < D; ++d) o[d] = acc[d];
      if (lse) lse[bq * H + h] = M + std::log(L);
    });
  }
}

// ------------------------------------------- f1: grouped output projection ---
// "DeepSeek V4 technical report" (agentupdate.ai), 混合注意力机制, item
// 分组输出投影 (grouped output projection): with head dim 512, projecting all
// head outputs straight back to the model dim d is costly, so the n_h heads
// are split into g groups, each group is first projected to an intermediate
// dim d_g, and the results are then projected together back to d.  "DeepSeek
// V4-Pro" (llm-arch-kb), "1. Hybrid attention": g = 16, d_g = 1024.
//
// Reading (the pages give the two projections only): for token t and group
// j, x_j = the concatenation of the outputs of heads j*H/g .. (j+1)*H/g - 1
// (H/g * D values, head-major); y_j = W_g[j] x_j (W_g[j]: [d_g, H/g * D],
// rows = outputs); y = concat_j y_j ([g * d_g]); z = W_o y (W_o: [d, g * d_g]).
// No bias and no nonlinearity between the two.  The library stores y in
// bfloat16, so y_bf16 != 0 rounds y to bfloat16 before the second
// projection, as the storage contract does; y_in != nullptr replaces the
// first projection by the given bfloat16 y (a step-chained check).
void orc_grouped_out_proj(int64_t T, int H, int D, int g, int d_g, int d_model,
                          const uint16_t* o, const uint16_t* w_g, const uint16_t* w_o,
                          int y_bf16, const uint16_t* y_in, double* y_out, double* z_out,
                          int nthreads) {
  const int hpg = H / g;             // heads per group
  const int64_t kin = (int64_t)hpg * D;  // inputs of one group
  const int64_t ny = (int64_t)g * d_g;
  parallel_for(T, nthreads, [&](int64_t t) {
    std::vector<double> y(ny);
    if (y_in) {
      for (int64_t i = 0; i < ny; ++i) y[i] = bf16_decode(y_in[t * ny + i]);
    } else {
      for (int j = 0; j < g; ++j) {
        const uint16_t* x = o + (t * H + (int64_t)j * hpg) * D;  // heads of group j, contiguous
        for (int r = 0; r < d_g; ++r) {
          const uint16_t* wr = w_g + ((int64_t)j * d_g + r) * kin;
          double acc = 0.0;
          for (int64_t c = 0; c < kin; ++c) acc += bf16_decode(wr[c]) * bf16_decode(x[c]);
          y[(int64_t)j * d_g + r] = acc;
        }
      }
      if (y_bf16)
        for (int64_t i = 0; i < ny; ++i) y[i] = bf16_decode(bf16_encode(y[i]));
    }
    if (y_out)
      for (int64_t i = 0; i < ny; ++i) y_out[t * ny + i] = y[i];
    for (int n = 0; n < d_model; ++n) {
      const uint16_t* wr = w_o + (int64_t)n * ny;
      double acc = 0.0;
      for (int64_t i = 0; i < ny; ++i) acc += bf16_decode(wr[i]) * y[i];
      z_out[t * d_model + n] = acc;
    }
  });
}

}  // extern "C"
