// Internal launch interface between the C ABI (abi.cu) and the kernels.
// Host-side only types: plain pointers and sizes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

struct CompressLaunch {
  int B, d, D_I, m;
  int overlap;              // tokens of block i-1 that entry i also pools (b_pos has m + overlap)
  int64_t entry_offset;     // local entry i is block entry_offset + i of the sequence
  // First kernel of a call, launched with programmatic serialization: it
  // waits for the previous kernel before any global read and lets its
  // dependents start only after that (so they may read the call's inputs).
  int pdl_head;
  int64_t L_cap, N_cap;
  const void* kv_tok;
  const void* idx_tok;  // null: KV stream only
  const int64_t* ctx_len;
  int64_t ctx_len_value;  // used when ctx_len is null
  const float *w_s, *b_pos, *gamma, *w_s_idx, *b_pos_idx;
  int64_t first_block, n_blocks;
  const int64_t* pos_newest;  // [B] or null: one block per sequence, the one holding pos
  void* kv_c;
  uint8_t* idx_key;
  float* idx_scale;
  float eps;
  int rope_dim;             // KV entries are stored rotated to (i+1)*m - 1
  double inv_freq[64];      // rope_dim/2 entries
  int32_t* status;
  int chained;              // see launch_pdl
};
cudaError_t launch_compress(const CompressLaunch& c, cudaStream_t stream);
// CTAs of launch_compress for these arguments.
int compress_ctas(const CompressLaunch& c);

// Lightning Indexer scores (tcgen05 kind::f8f6f4) over every (query, entry
// tile).  Queries are grouped G per MMA (N = G * H_I <= 256).
struct IndexLaunch {
  int B, Q, H_I, D_I, m;
  int64_t N_cap;
  const uint8_t* q_idx;     // [B, Q, H_I, D_I]
  const float* q_scale;     // [B, Q, H_I]
  const float* w;           // [B, Q, H_I]
  const uint8_t* key;       // [B, N_cap, D_I]
  const float* key_scale;   // [B, N_cap]
  const int64_t* pos_q;     // [B, Q] or null -> pos_base + q
  int64_t pos_base;
  float* scores;            // [B, Q, N_cap]
  int32_t* status;
  int num_sms;
  int64_t entry_offset;     // the cache holds entries entry_offset .. N_cap-1+entry_offset
  // Keys of entries below the bound were written before the call and are
  // read before waiting on the previous kernel: safe_pos[b] / m (per
  // sequence, the block holding that position is being written) when given,
  // else safe_fixed.
  const int64_t* safe_pos;
  int64_t safe_fixed;
  int chained;              // see launch_pdl
  // One query per sequence only (Q == 1): adds, per sequence, the count of
  // its visible scores by the top kScoreHistBits bits of their keys
  // (score_key) to hist[b * kScoreHistBins ..].  Null: no histogram.
  uint32_t* hist = nullptr;
  // Slots (CTAs of this kernel's size) that the call's previous kernel keeps
  // busy while this one starts: the grid leaves them out.
  int reserve_slots = 0;
};
cudaError_t launch_index_scores(const IndexLaunch& a, cudaStream_t stream);

// Score histogram of the decode chain: bins of the top 12 key bits.
constexpr int kScoreHistBits = 12;
constexpr int kScoreHistBins = 1 << kScoreHistBits;

// Exact top-k over fp32 scores, one cluster of CTAs per query row.
struct TopkLaunch {
  int rows;                 // B * Q
  int Q, m;
  int64_t N_cap;
  const float* scores;      // [rows, N_cap]
  const int64_t* pos_q;     // [rows] or null -> pos_base + (row % Q)
  int64_t pos_base;
  int k;
  int32_t* idx;             // [rows, k]
  int32_t* cnt;             // [rows]
  int32_t* status;
  int64_t entry_offset;     // score j is entry entry_offset + j of the sequence
  int chained;              // see launch_pdl
  // [rows, kScoreHistBins] histogram of each row's visible scores, written
  // by the indexer kernel (IndexLaunch::hist), or null.  Used as a guess of
  // the threshold bin; the selection is exact whatever it holds.  Every bin
  // is zero when the kernel ends.
  uint32_t* hist = nullptr;
  int32_t* path = nullptr;  // [rows] or null: 0 all kept, 1 histogram, 2 radix rounds
};
cudaError_t launch_topk(const TopkLaunch& a, cudaStream_t stream);
// True when launch_topk takes the histogram path for these rows (one
// cluster of CTAs per row): only then should the indexer build one.
bool topk_uses_hist(int rows, int64_t N_cap);
// CTAs (one SM each) of the histogram top-k for these rows; 0 when it does
// not run.
int topk_hist_ctas(int rows, int64_t N_cap);

// Context split over ranks: a shard's candidates (score, sequence index) and
// the global top-k over all ranks' candidates.
cudaError_t launch_shard_candidates(const float* scores, int64_t N_cap, const int32_t* idx,
                                    const int32_t* cnt, int rows, int k, int64_t offset,
                                    float* cand_s, int32_t* cand_i, cudaStream_t stream);
struct MergeLaunch {
  int G, rows, k;
  const float* cand_s;      // [G, rows, k]
  const int32_t* cand_i;    // [G, rows, k]
  const int32_t* cand_c;    // [G, rows]
  int32_t* idx;             // [rows, k]
  int32_t* cnt;             // [rows]
  int64_t lo, hi;           // this rank's entries
  int32_t* local_idx;       // [rows, k]
  int32_t* local_cnt;       // [rows]
  int32_t* status;
  int chained;
};
cudaError_t launch_merge_candidates(const MergeLaunch& a, cudaStream_t stream);

// Shared-KV MQA decode (sparse or dense) with window and sink: one CTA per
// (query row, split) for H <= 64, two for H > 64 (64 heads each), at the
// full head dim;
// split partials (fp16 O/l plus max and sum) are merged by the combine
// kernel.
struct MqaLaunch {
  int B, Q, H, D, m, W, rope_dim;
  int64_t N_cap, L_cap;
  const void* q;            // [B*Q, H, D] bf16
  const int64_t* pos_q;     // [B*Q] or null -> pos_base + (row % Q)
  int64_t pos_base;
  const void* kv_c;         // [B, N_cap, D]
  const int32_t* sel_idx;   // [B*Q, kmax] or null (dense)
  const int32_t* sel_cnt;   // [B*Q]
  int kmax;
  const void* kv_tok;       // [B, L_cap, D]
  const float* sink;        // [H]
  const float* gamma_q;     // [D] or null
  const float* gamma_kv;    // [D] or null
  float eps, scale;
  double inv_freq[64];      // rope_dim/2 entries
  void* out;                // [B*Q, H, D] bf16
  float* lse;               // [B*Q, H] or null
  void* part_o;             // workspace [rows, S, H, D] fp16: split output / split sum
  float* part_ml;           // workspace [rows, S, 2, H] fp32
  int splits;               // S
  int32_t* status;
  int64_t entry_offset;     // the cache holds entries entry_offset .. of the sequence
  int chained;              // see launch_pdl (the merge kernel is always chained)
  int emit_partials;        // write the split partials only (no merge, no output)
  // Without a selection, cached entries below the bound were written before
  // the call and are read before waiting on the previous kernel:
  // safe_pos[b] / m (per sequence, the block holding that position is being
  // written) when given, else safe_fixed (0: every cached entry waits).
  // Window tokens are caller inputs and never wait; a selection always does.
  const int64_t* safe_pos = nullptr;
  int64_t safe_fixed = 0;
};
size_t mqa_workspace_bytes(int rows, int splits, int H, int D);
int mqa_choose_splits(int rows, int64_t compressed_max, int window, int num_sms, int H);
cudaError_t launch_mqa(const MqaLaunch& a, cudaStream_t stream);
// The split merge alone (part_o / part_ml with a.splits splits per row).
cudaError_t launch_mqa_merge(const MqaLaunch& a, cudaStream_t stream);

// One projection GEMM of the grouped output projection: for each group j,
// C[t, j*N + n] = sum_k A[t, j*K + k] * W[j*N + n, k] (bf16 in, fp32
// accumulate, bf16 out), or fp32 split-K partials reduced by a second kernel.
struct ProjGemm {
  const void* a;      // [T, lda] bf16 (lda >= groups * K)
  int64_t lda;
  const void* w;      // [w_rows, K] bf16, w_rows = groups * N
  int64_t w_rows;
  int K, N, groups, T;
  int splits;         // split-K factor (partials in `part` when > 1)
  void* c;            // [T, ldc] bf16
  int ldc;
  float* part;        // [splits, T, ldc] fp32 workspace (splits > 1)
  int32_t* status;
  int chained;        // see launch_pdl
};
cudaError_t launch_proj_gemm(const ProjGemm& g, cudaStream_t stream);
int proj_token_tile(int T);
int proj_choose_splits(int T, int N, int groups, int K, int num_sms);

int device_sm_count();

// Launches `kern` and, when cluster_x > 0, as (cluster_x, 1, 1) clusters.
//
// chained != 0: with programmatic stream serialization, so the kernel may
// start while its predecessor in the stream still runs, up to its
// pdl_wait().  Only the second and later kernels of one entry point are
// launched this way: their predecessor is a kernel of the same call, which
// itself started only after everything before the call had completed.  So
// their reads of caller inputs before pdl_wait() are safe, and their reads
// of data written by an earlier kernel of the call come after pdl_wait().
// chained == 0 (the first kernel of an entry point): an ordinary launch,
// which starts after all earlier work in the stream has completed, whatever
// that work is (a caller's kernel that lets its dependents start early
// included).  The decode steps' first kernel (compression) instead runs in
// a head mode: launched with programmatic serialization, it waits for the
// previous kernel before it reads anything and triggers its dependents only
// after that wait, which gives the same guarantee while its launch overlaps
// the previous kernel.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, int cluster_x, int chained, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (chained) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Sets the message that csa_last_error returns and passes `s` through.
csa_status set_error(csa_status s, const char* fmt, ...);

// Sets the dynamic shared-memory limit of `func` once per device (the call
// is then skipped, which keeps launches legal inside CUDA-graph capture).
// `slot` (0..31) identifies the kernel: each kernel instance has its own
// (indexer 0-1, 15-16 and 19-20, top-k 2, 8-9 and 17, attention 3-7, projection 10-14).
cudaError_t ensure_smem_attr(const void* func, int slot, size_t bytes);

}  // namespace csa
