// Shared-KV multi-query attention for decode (CSA sparse / HCA dense) with
// the sliding window and per-head sink, on the 5th-generation tensor cores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), hybrid attention: CSA step
// 3 (multi-query attention over the selected compressed entries) and the HCA
// paragraph (dense attention over every compressed entry); "DeepSeek V4-Pro"
// (llm-arch-kb), "Hybrid attention": 128 query heads of dim 512 sharing one
// KV head, a 128-token uncompressed window branch, a learnable sink logit per
// head in the softmax denominator, RMSNorm on queries and KV, RoPE on the
// last 64 dims of query / KV / output with the inverse rotation on the output.
//
// Design.  The 128 x 512 fp32 output accumulator alone would fill the whole
// tensor memory of an SM, so a pair of CTAs (a cluster of 2) shares every
// (query, split): CTA r owns head-dim half r.  Per 64-entry tile:
//   - the producer warp gathers the tile's rows with TMA tile::gather4 (only
//     this CTA's half of each row; 128-byte swizzle), K = V = that tile;
//   - transform warps RoPE the rotated dims in place (the half that holds
//     them) and, for window tokens, compute the half-row sum of squares that
//     the token RMSNorm needs;
//   - the MMA warp issues S_r = Qhat_r . K_r^T (A = this CTA's half of the
//     normalised, roped query, resident in TMEM; B = the tile, K-major) into
//     one of two TMEM S buffers, then P . V_r into the O half (A = P in TMEM,
//     B = the same tile read MN-major);
//   - softmax warps (thread = head) exchange the partial S rows with the peer
//     through distributed shared memory, sum them in a fixed order (so both
//     CTAs hold bit-identical logits), apply the window-token norm factors,
//     run an online softmax with lazy rescaling (O is rescaled in TMEM only
//     when the running max grows by more than 8), and write P (bf16) back
//     into the S buffer for the P.V MMA.
// Splits of the KV list run on different pairs; their (m, l, O) partials are
// merged by mqa_combine_kernel, which also folds in the sink and applies the
// inverse RoPE.  Every wait is bounded and reports CSA_ERR_DEVICE_TIMEOUT.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma.h"

namespace csa {

size_t mqa_workspace_bytes(int rows, int splits, int H, int D) {
  size_t o = (size_t)rows * splits * H * D * 4;
  o = (o + 255) / 256 * 256;
  return o + (size_t)rows * splits * 2 * H * 4;
}

// Splits of each row's KV list over CTA pairs: at most one wave of pairs
// (rows * splits <= SMs / 2), no split left without a tile.
int mqa_choose_splits(int rows, int64_t compressed_max, int window, int num_sms) {
  const int64_t tiles = (compressed_max + 63) / 64 + (window + 63) / 64;
  const int64_t pairs = std::max(1, num_sms / 2);
  int64_t s = std::max<int64_t>(1, pairs / std::max(1, rows));
  s = std::min<int64_t>(s, std::max<int64_t>(1, tiles));
  const int64_t tps = (tiles + s - 1) / s;
  s = std::max<int64_t>(1, (tiles + tps - 1) / tps);
  return (int)s;
}

namespace {

constexpr int TN = 64;           // KV rows per tile
constexpr int kThreads = 320;    // 10 warps
constexpr int kXRow = TN;        // floats per head row in an exchange slot
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct MCfg {
  static constexpr int Dh = D / 2;             // head-dim half per CTA
  static constexpr int NC = Dh / 64;           // 128-byte chunks per half row
  static constexpr int kChunkBytes = TN * 128;
  static constexpr int kStageBytes = NC * kChunkBytes;
  static constexpr int kStages = D == 512 ? 2 : 4;
  static constexpr int kQCols = Dh / 2;        // bf16 pairs
  static constexpr int kSCol0 = kQCols;        // two S buffers of TN columns
  static constexpr int kOCol = kQCols + 2 * TN;
  static constexpr int kCols = kOCol + Dh;     // 512 for D = 512
  static constexpr uint32_t kAlloc = kCols <= 256 ? 256 : 512;
};

struct Meta {
  int32_t grow[TN];   // row coordinate in the tensor map
  int32_t pos[TN];    // RoPE position
  float ss[TN];       // half-row sum of squares (window tiles)
  uint32_t valid[2];  // bit r: row r holds a real KV vector
  int32_t window;     // 1: window tokens; 0: compressed entries
  int32_t pad;
};

// One tile's partial logits of all 128 heads (+ the window half-row sums),
// as staged locally and as received from the peer.  Within a row the 16-byte
// chunks are XOR-swizzled by the row index so that the 128 threads' vector
// stores and loads hit distinct banks.
struct XSlot {
  float s[128 * kXRow];
  float ss[TN];
};
CSA_DEV int xoff(int h, int j) {  // float offset of (head h, column j)
  return h * kXRow + ((((j >> 2) ^ (h & 15)) << 2) | (j & 3));
}

struct Params {
  int Q, H, m, W, R, splits;
  int64_t N_cap, L_cap;
  const __nv_bfloat16* q;
  const int64_t* pos_q;
  int64_t pos_base;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  int kmax;
  const float* gamma_q;
  const float* gamma_kv;
  float eps, scale_log2;  // softmax scale * log2(e)
  float* part_o;
  float* part_ml;
  int32_t* status;
  double inv_freq[64];
};

// Byte offset of (row r, local dim d) inside a stage (128B-swizzled chunks).
CSA_DEV uint32_t tile_off(int r, int d) {
  uint32_t lin = (uint32_t)r * 128u + (uint32_t)(d & 63) * 2u;
  return (uint32_t)(d >> 6) * (TN * 128u) + (lin ^ (((lin >> 7) & 7u) << 4));
}

CSA_DEV uint64_t desc_k(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }
template <int D>
CSA_DEV uint64_t desc_mn(uint32_t saddr) {
  return sdesc_sw128(saddr, MCfg<D>::kChunkBytes, 1024);
}

CSA_DEV int64_t row_pos(const Params& p, int row) {
  return p.pos_q ? p.pos_q[row] : p.pos_base + row % p.Q;
}

template <bool kCluster = false>
CSA_DEV bool wait_all(uint64_t* bar, uint32_t parity, const Params& p, volatile int* abort_flag) {
  bool ok = mbar_wait<kCluster>(bar, parity, p.status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}


// Query prologue: qhat = RoPE(RMSNorm(q) * gamma_q), this CTA's half of every
// head row, into TMEM (bf16 pairs, the A operand of S = Qhat K^T).  Two
// threads share a head row: part 0 (a transform-warp thread) takes the first
// quarter of the row, part 1 (a softmax-warp thread, which also owns the
// rotated dims) the second; both sit in warps of the head's TMEM lane
// quarter.  All loads of a thread are in flight at once.  The half-row sums
// of squares are combined in the CTA (part 0 + part 1) and then with the peer
// CTA through distributed shared memory, always in rank order, so both CTAs
// normalise with the same bits.
template <int D, int R>
CSA_DEV void q_prologue(const Params& p, int part, int h, int row, uint32_t rank, uint32_t peer,
                        int64_t pos, uint32_t t_q, float* pss, float* qss_in, uint64_t* qssbar,
                        uint64_t* qready, volatile int* abort_flag) {
  using C = MCfg<D>;
  constexpr int NU = C::Dh / 16;  // 16-byte units per quarter row
  const bool head_ok = h < p.H;
  const int e0 = part * (C::Dh / 2);  // first element of this thread's quarter
  const __nv_bfloat16* qr =
      p.q + ((int64_t)row * p.H + (head_ok ? h : 0)) * D + rank * C::Dh + e0;
  uint4 u[NU];
#pragma unroll
  for (int c = 0; c < NU; ++c) u[c] = __ldg(reinterpret_cast<const uint4*>(qr) + c);
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < NU; ++c) {
    const uint32_t w4[4] = {u[c].x, u[c].y, u[c].z, u[c].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = bf16_lo(w4[q]), hi = bf16_hi(w4[q]);
      ss = fmaf(lo, lo, fmaf(hi, hi, ss));
    }
  }
  pss[part * 128 + h] = ss;
  named_barrier_sync(2, 256);  // the 128 part-0 and 128 part-1 threads
  const float half_ss = pss[h] + pss[128 + h];
  if (part == 1) {
    const uint32_t dst = mapa(smem_u32(&qss_in[h]), peer);
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(dst), "f"(half_ss) : "memory");
    mbar_arrive_remote(mapa(smem_u32(qssbar), peer));
  }
  mbar_wait<true>(qssbar, 0, p.status, abort_flag);
  const float other = qss_in[h];
  const float tot = rank == 0 ? half_ss + other : other + half_ss;
  const float inv = head_ok ? 1.0f / sqrtf(tot / (float)D + p.eps) : 0.f;
  const int dbase = rank * C::Dh + e0;
  const uint32_t lane_base = (uint32_t)(h & ~31) << 16;
  const float* gq = p.gamma_q ? p.gamma_q + dbase : nullptr;
  // 8 normalised elements of unit c (re-read: the lines are in L1 by now).
  auto unit8 = [&](int c, float (&x)[8]) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(qr) + c);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      x[2 * q] = bf16_lo(w4[q]) * inv;
      x[2 * q + 1] = bf16_hi(w4[q]) * inv;
    }
    if (gq) {
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(gq + 8 * c));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(gq + 8 * c + 4));
      x[0] *= g0.x; x[1] *= g0.y; x[2] *= g0.z; x[3] *= g0.w;
      x[4] *= g1.x; x[5] *= g1.y; x[6] *= g1.z; x[7] *= g1.w;
    }
  };
  constexpr int Qn = C::Dh / 2;                         // elements per quarter row
  const bool roped = R > 0 && rank == 1 && part == 1;  // rotated dims: end of the half
  const int plain_end = roped ? Qn - R : Qn;
#pragma unroll 1
  for (int c0 = 0; c0 < plain_end; c0 += 32) {
    uint32_t pk[16];
#pragma unroll
    for (int u4 = 0; u4 < 4; ++u4) {
      float x[8];
      unit8(c0 / 8 + u4, x);
#pragma unroll
      for (int q = 0; q < 4; ++q) pk[u4 * 4 + q] = pack_bf16(x[2 * q], x[2 * q + 1]);
    }
    tmem_st16(t_q + lane_base + (e0 + c0) / 2, pk);
  }
  if constexpr (R > 0) {
    if (roped) {
      constexpr int half = R / 2;
      constexpr int b0 = Qn - R;
#pragma unroll 1
      for (int j0 = 0; j0 < half; j0 += 16) {
        float a[16], b[16];
        unit8((b0 + j0) / 8, *reinterpret_cast<float(*)[8]>(a));
        unit8((b0 + j0) / 8 + 1, *reinterpret_cast<float(*)[8]>(a + 8));
        unit8((b0 + half + j0) / 8, *reinterpret_cast<float(*)[8]>(b));
        unit8((b0 + half + j0) / 8 + 1, *reinterpret_cast<float(*)[8]>(b + 8));
        uint32_t pk1[8], pk2[8];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          float s0, c0, s1, c1;
          sincos_reduced((double)pos * p.inv_freq[j0 + j], &s0, &c0);
          sincos_reduced((double)pos * p.inv_freq[j0 + j + 1], &s1, &c1);
          pk1[j / 2] = pack_bf16(a[j] * c0 - b[j] * s0, a[j + 1] * c1 - b[j + 1] * s1);
          pk2[j / 2] = pack_bf16(b[j] * c0 + a[j] * s0, b[j + 1] * c1 + a[j + 1] * s1);
        }
        // Columns hold bf16 pairs: local dim d -> column d/2 (8 columns each).
        tmem_st8(t_q + lane_base + (e0 + b0 + j0) / 2, pk1);
        tmem_st8(t_q + lane_base + (e0 + b0 + half + j0) / 2, pk2);
      }
    }
  }
  tmem_wait_st();
  tc_fence_before();
  mbar_arrive(qready);
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 1)
    mqa_pair_kernel(const __grid_constant__ CUtensorMap map_c,
                    const __grid_constant__ CUtensorMap map_t,
                    const __grid_constant__ CUtensorMap box_c,
                    const __grid_constant__ CUtensorMap box_t, const Params p) {
  using C = MCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  XSlot* xs = reinterpret_cast<XSlot*>(stages + C::kStages * C::kStageBytes);
  XSlot* xst = xs + 2;  // [2] local staging of this CTA's partial logits
  Meta* meta = reinterpret_cast<Meta*>(xs + 4);
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta + C::kStages);
  uint64_t* full = bars;
  uint64_t* ready = full + C::kStages;
  uint64_t* empty = ready + C::kStages;
  uint64_t* sfull = empty + C::kStages;
  uint64_t* pready = sfull + 2;
  uint64_t* xfull = pready + 2;
  uint64_t* xempty = xfull + 2;
  uint64_t* pvdone = xempty + 2;
  uint64_t* qready = pvdone + 1;
  uint64_t* drain = qready + 1;
  uint64_t* staged = drain + 1;
  uint64_t* qssbar = staged + 1;
  float* qss_in = reinterpret_cast<float*>(qssbar + 1);  // [128] peer's half-row sums
  float* pss = qss_in + 128;                               // [2][128] quarter-row sums
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pss + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int split = blockIdx.x >> 1;
  const int row = blockIdx.y;
  const int b = row / p.Q;

  // The KV list of this query row: n_c compressed entries, then the window.
  const int64_t pos = row_pos(p, row);
  int64_t n_vis = pos < 0 ? 0 : (pos + 1) / p.m;
  if (n_vis > p.N_cap) n_vis = p.N_cap;
  int n_c;
  if (p.sel_idx) {
    int c = p.sel_cnt[row];
    n_c = c < 0 ? 0 : (c > p.kmax ? p.kmax : c);
  } else {
    n_c = (int)n_vis;
  }
  const int64_t w0 = pos - p.W + 1 < 0 ? 0 : pos - p.W + 1;
  const int nwin = (p.W > 0 && pos >= 0) ? (int)(pos - w0 + 1) : 0;
  const int tiles_c = (n_c + TN - 1) / TN;
  const int tiles_all = tiles_c + (nwin + TN - 1) / TN;
  const int tps = (tiles_all + p.splits - 1) / p.splits;
  const int t0 = std::min(split * tps, tiles_all);
  const int t1 = std::min(t0 + tps, tiles_all);
  const int ntile = t1 - t0;

  float* po = p.part_o + (((int64_t)row * p.splits + split) * p.H) * D + rank * C::Dh;
  float* pml = p.part_ml + ((int64_t)row * p.splits + split) * 2 * p.H;
  if (ntile <= 0) {  // empty split: an empty partial (uniform over the pair)
    if (rank == 0)
      for (int h = threadIdx.x; h < p.H; h += kThreads) {
        pml[h] = -INFINITY;
        pml[p.H + h] = 0.f;
      }
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&pready[a], 128);
      mbar_init(&xfull[a], 1);    // own expect_tx + the peer's bulk copy
      mbar_init(&xempty[a], 128); // the peer's softmax threads
    }
    mbar_init(pvdone, 1);
    mbar_init(qready, 256);
    mbar_init(drain, 1);
    mbar_init(qssbar, 128);
    mbar_init(staged, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the peer's barriers are initialised before any remote arrive
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_q = tmem, t_s = tmem + C::kSCol0, t_o = tmem + C::kOCol;

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    // Contiguous tiles (dense entries, window tokens) are fetched with four
    // 64-row box copies; selected entries with row gathers (tile::gather4),
    // two per lane so the whole warp issues them.
    int it = 0;
    for (int t = t0; t < t1; ++t, ++it) {
      const int s = it % C::kStages;
      const uint32_t ph = (it / C::kStages) & 1;
      const bool win = t >= tiles_c;
      const bool gathered = !win && p.sel_idx != nullptr;
      // Row metadata (loads issued before the slot wait so they overlap it).
      int32_t grow[2], rpos[2];
      bool valid[2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = lane + 32 * hh;
        if (!win) {
          const int j = t * TN + r;
          valid[hh] = j < n_c;
          int64_t i = j;
          if (valid[hh] && gathered) {
            i = p.sel_idx[(int64_t)row * p.kmax + j];
            if (i < 0 || i >= n_vis) {
              report(p.status, CSA_ERR_DEVICE_INDEX);
              valid[hh] = false;
            }
          }
          if (!valid[hh] && gathered) i = 0;
          grow[hh] = (int32_t)((int64_t)b * p.N_cap + i);
          rpos[hh] = (int32_t)((i + 1) * p.m - 1);
        } else {
          const int j = (t - tiles_c) * TN + r;
          valid[hh] = j < nwin;
          if (valid[hh] && w0 + j >= p.L_cap) {  // query position beyond the token buffer
            report(p.status, CSA_ERR_CAPACITY);
            valid[hh] = false;
          }
          const int64_t tok = w0 + j;
          grow[hh] = (int32_t)((int64_t)b * p.L_cap + tok);
          rpos[hh] = (int32_t)tok;
        }
      }
      const uint32_t vb0 = __ballot_sync(0xffffffffu, valid[0]);
      const uint32_t vb1 = __ballot_sync(0xffffffffu, valid[1]);
      if (!wait_all(&empty[s], ph ^ 1, p, abort_flag)) break;
      Meta& M = meta[s];
      M.grow[lane] = grow[0];
      M.grow[lane + 32] = grow[1];
      M.pos[lane] = rpos[0];
      M.pos[lane + 32] = rpos[1];
      if (lane == 0) {
        M.valid[0] = vb0;
        M.valid[1] = vb1;
        M.window = win ? 1 : 0;
        mbar_expect_tx(&full[s], C::kStageBytes);
      }
      __syncwarp();
      uint8_t* dst = stages + s * C::kStageBytes;
      if (!gathered) {
        // Rows grow[0] .. grow[0]+63 are consecutive (rows past the list are
        // fetched too and masked; rows past the tensor are zero-filled).
        const int32_t y0 = __shfl_sync(0xffffffffu, grow[0], 0);
        if (lane < C::NC)
          tma_load_2d(dst + lane * C::kChunkBytes, win ? &box_t : &box_c, &full[s],
                      (int32_t)(rank * C::Dh + lane * 64), y0);
      } else {
        // 16 groups of 4 rows per 128-byte chunk: lane -> (chunk, 2 groups).
        constexpr int kGroups = C::NC * (TN / 4);
        for (int q = lane; q < kGroups; q += 32) {
          const int c = q / (TN / 4), g = q % (TN / 4);
          tma_gather4(dst + c * C::kChunkBytes + g * 4 * 128, &map_c, &full[s],
                      (int32_t)(rank * C::Dh + c * 64), M.grow[4 * g], M.grow[4 * g + 1],
                      M.grow[4 * g + 2], M.grow[4 * g + 3]);
        }
      }
    }
    if (*abort_flag && lane == 0) {  // copies still in flight must land first
      for (int j = std::max(0, it - C::kStages); j < it; ++j)
        mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.status);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    const uint32_t idesc_s = idesc_bf16(128, TN, 0, 0);
    const uint32_t idesc_pv = idesc_bf16(128, C::Dh, 0, 1);
    bool ok = wait_all(qready, 0, p, abort_flag);
    tc_fence_after();
    bool issued = false;
    auto issue_pv = [&](int jt) -> bool {
      const int a = jt & 1, s = jt % C::kStages;
      if (!wait_all(&pready[a], (jt >> 1) & 1, p, abort_flag)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t base = smem_u32(stages + s * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk)
          mma_bf16_ts(t_o, t_s + a * TN + kk * 8, desc_mn<D>(base + kk * 16 * 128), idesc_pv,
                      (jt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(pvdone);
      }
      __syncwarp();
      return true;
    };
    int it = 0;
    for (; ok && it < ntile; ++it) {
      const int s = it % C::kStages, a = it & 1;
      if (!wait_all(&ready[s], (it / C::kStages) & 1, p, abort_flag)) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t base = smem_u32(stages + s * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < C::Dh / 16; ++kk)
          mma_bf16_ts(t_s + a * TN, t_q + kk * 8,
                      desc_k(base + (kk >> 2) * C::kChunkBytes + (kk & 3) * 32), idesc_s,
                      kk > 0 ? 1u : 0u);
        mma_commit(&sfull[a]);
      }
      __syncwarp();
      issued = true;
      if (it > 0 && !issue_pv(it - 1)) break;
    }
    if (it == ntile && ntile > 0 && !*abort_flag) issue_pv(ntile - 1);
    if (*abort_flag && issued) {
      if (elect_one()) mma_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, p.status);
    }
  } else if (warp < 6) {
    // ----------------------------------------------------------- transform --
    // Two threads per tile row: `half` 0 takes the window-norm sum and the
    // first half of the rotated pairs, `half` 1 the second half.
    const int tid = threadIdx.x - 64;  // 0..127
    q_prologue<D, R>(p, 0, (warp & 3) * 32 + lane, row, rank, peer, pos, tmem, pss, qss_in,
                     qssbar, qready, abort_flag);
    const int r = tid >> 1, hf = tid & 1;
    const bool rope_here = (R > 0) && rank == 1;
    for (int it = 0; it < ntile; ++it) {
      const int s = it % C::kStages;
      if (!wait_all(&full[s], (it / C::kStages) & 1, p, abort_flag)) break;
      const Meta& M = meta[s];
      uint8_t* st = stages + s * C::kStageBytes;
      const bool valid = (M.valid[r >> 5] >> (r & 31)) & 1u;
      float ss = 0.f;
      if (valid && M.window) {
        for (int c = hf; c < C::Dh / 8; c += 2) {  // 16-byte units
          uint4 u = *reinterpret_cast<const uint4*>(st + tile_off(r, c * 8));
          uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float lo = bf16_lo(w4[q]), hi = bf16_hi(w4[q]);
            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
          }
          if (p.gamma_kv) {
            const float* g = p.gamma_kv + rank * C::Dh + c * 8;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              w4[q] = pack_bf16(bf16_lo(w4[q]) * __ldg(g + 2 * q),
                                bf16_hi(w4[q]) * __ldg(g + 2 * q + 1));
            *reinterpret_cast<uint4*>(st + tile_off(r, c * 8)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      if (hf == 0) meta[s].ss[r] = ss;
      __syncwarp();  // gain-scaled values are in place before the rotation reads them
      if (valid && rope_here) {
        // The rotated dims are the last R of this half row: pairs (j, j+R/2).
        // Thread half hf rotates pairs [hf*R/4, hf*R/4 + R/4) with 16-byte
        // shared-memory accesses (8 bf16 per access).
        constexpr int half = R / 2;
        constexpr int d0 = C::Dh - R;
        const double ppos = (double)M.pos[r];
#pragma unroll
        for (int q = 0; q < R / 32; ++q) {  // R/4 pairs per thread, 8 per access
          const int j0 = hf * (half / 2) + q * 8;
          uint4* pa = reinterpret_cast<uint4*>(st + tile_off(r, d0 + j0));
          uint4* pb = reinterpret_cast<uint4*>(st + tile_off(r, d0 + half + j0));
          uint4 ua = *pa, ub = *pb;
          uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float s0, c0, s1, c1;
            sincos_reduced(ppos * p.inv_freq[j0 + 2 * e], &s0, &c0);
            sincos_reduced(ppos * p.inv_freq[j0 + 2 * e + 1], &s1, &c1);
            const float x10 = bf16_lo(wa[e]), x11 = bf16_hi(wa[e]);
            const float x20 = bf16_lo(wb[e]), x21 = bf16_hi(wb[e]);
            wa[e] = pack_bf16(x10 * c0 - x20 * s0, x11 * c1 - x21 * s1);
            wb[e] = pack_bf16(x20 * c0 + x10 * s0, x21 * c1 + x11 * s1);
          }
          *pa = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          *pb = make_uint4(wb[0], wb[1], wb[2], wb[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[s]);
    }
  } else {
    // ------------------------------------------------- softmax / epilogue --
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;  // head == TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const bool head_ok = h < p.H;
    q_prologue<D, R>(p, 1, h, row, rank, peer, pos, t_q, pss, qss_in, qssbar, qready,
                     abort_flag);

    float m_run = -INFINITY, l_run = 0.f;
    const uint32_t xs_peer = mapa(smem_u32(&xs[0]), peer);
    const uint32_t xfull_peer = mapa(smem_u32(&xfull[0]), peer);
    const uint32_t xempty_peer = mapa(smem_u32(&xempty[0]), peer);
    const bool leader = h == 0;  // issues the bulk copies of the staged logits
    // Software pipeline with a lag of one tile: iteration it sends tile it's
    // partial logits to the peer, then computes the softmax of tile it-1,
    // whose exchange has had a whole iteration to land.
    //
    // send(it): S(it) from TMEM -> local staging slot a -> one bulk copy into
    // the peer's receive slot a (completes on the peer's xfull[a]).  Staging
    // slot a and the peer's receive slot a are both free once the peer has
    // consumed tile it-2 (its xempty[a] arrivals).
    auto send = [&](int it) -> bool {
      const int s = it % C::kStages, a = it & 1;
      if (!wait_all(&sfull[a], (it >> 1) & 1, p, abort_flag)) return false;
      tc_fence_after();
      float sv[TN];
      {
        uint32_t v[4][16];
        const uint32_t t_sa = t_s + lane_base + a * TN;
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(t_sa + 16 * c, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < 16; ++j) sv[16 * c + j] = __uint_as_float(v[c][j]);
      }
      if (!wait_all(&ready[s], (it / C::kStages) & 1, p, abort_flag)) return false;
      if (!wait_all<true>(&xempty[a], ((it >> 1) & 1) ^ 1, p, abort_flag)) return false;
      XSlot& st = xst[a];
#pragma unroll
      for (int j = 0; j < TN; j += 4)
        *reinterpret_cast<float4*>(st.s + xoff(h, j)) =
            make_float4(sv[j], sv[j + 1], sv[j + 2], sv[j + 3]);
      if (h < TN) st.ss[h] = meta[s].ss[h];
      fence_proxy_async_smem();
      mbar_arrive(staged);
      if (leader) {
        mbar_expect_tx(&xfull[a], (uint32_t)sizeof(XSlot));  // own receive slot
        if (mbar_wait(staged, it & 1, p.status, abort_flag))
          asm volatile(
              "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes"
              " [%0], [%1], %2, [%3];" ::"r"(xs_peer + (uint32_t)(a * sizeof(XSlot))),
              "r"(smem_u32(&st)), "r"((uint32_t)sizeof(XSlot)), "r"(xfull_peer + a * 8)
              : "memory");
      }
      return true;
    };
    // compute(it): logits, online softmax (lazy rescale), P into TMEM.
    auto compute = [&](int it) -> bool {
      const int s = it % C::kStages, a = it & 1;
      const uint32_t t_sa = t_s + lane_base + a * TN;
      if (!wait_all<true>(&xfull[a], (it >> 1) & 1, p, abort_flag)) return false;
      const Meta& M = meta[s];
      const bool win = M.window != 0;
      const uint32_t vw0 = M.valid[0], vw1 = M.valid[1];
      const XSlot& X = xs[a];
      const XSlot& Y = xst[a];
      // Logit of column j: the two partial sums added in rank order (bit-
      // identical in both CTAs); window tokens scaled by 1/rms(c_t) from the
      // two half sums of squares, also in rank order.
      auto logit4 = [&](int j, float (&v)[4]) {
        const float4 mine = *reinterpret_cast<const float4*>(Y.s + xoff(h, j));
        const float4 theirs = *reinterpret_cast<const float4*>(X.s + xoff(h, j));
        const float a4[4] = {mine.x, mine.y, mine.z, mine.w};
        const float b4[4] = {theirs.x, theirs.y, theirs.z, theirs.w};
        const uint32_t vw = j < 32 ? vw0 : vw1;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x = rank == 0 ? __fadd_rn(a4[e], b4[e]) : __fadd_rn(b4[e], a4[e]);
          if (win) {
            const float ssum = rank == 0 ? __fadd_rn(Y.ss[j + e], X.ss[j + e])
                                         : __fadd_rn(X.ss[j + e], Y.ss[j + e]);
            x = __fmul_rn(x, rsqrtf(__fadd_rn(__fmul_rn(ssum, 1.0f / (float)D), p.eps)));
          }
          v[e] = ((vw >> ((j + e) & 31)) & 1u) ? __fmul_rn(x, p.scale_log2) : -INFINITY;
        }
      };
      float mt;
      {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll 1
        for (int j = 0; j < TN; j += 16) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v[4];
            logit4(j + 4 * q, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) m4[e] = fmaxf(m4[e], v[e]);
          }
        }
        mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      // Online softmax with lazy rescaling (log2 domain).
      const bool grow = mt > m_run + kRescaleThreshold * 1.4426950408889634f || m_run == -INFINITY;
      const float m_new = grow ? fmaxf(mt, m_run) : m_run;
      const bool need = grow && m_run != -INFINITY;
      // P.V of the previous tile must be complete before O may be rescaled.
      // This wait happens on every tile, before pready(it) is released, so
      // the pvdone phase can never run two phases ahead of this check.
      if (it > 0) {
        if (!wait_all(pvdone, (it - 1) & 1, p, abort_flag)) return false;
        tc_fence_after();
      }
      if (__any_sync(0xffffffffu, need) && it > 0) {
        const float f = need ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < C::Dh; c += 16) {
          uint32_t v[16];
          tmem_ld16(t_o + lane_base + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
          tmem_st16(t_o + lane_base + c, v);
        }
        tmem_wait_st();
      }
      if (need) l_run *= fast_exp2(m_run - m_new);
      m_run = m_new;
      // P = 2^(logit - m) in bf16, times the window norm (V = norm * the
      // stored row), written over the consumed S columns.
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      const bool live = m_run != -INFINITY;
#pragma unroll 1
      for (int j = 0; j < TN; j += 16) {
        uint32_t pk[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[4];
          logit4(j + 4 * q, v);
          float pe[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            pe[e] = live ? fast_exp2(v[e] - m_run) : 0.f;
            l4[e] += pe[e];
            if (win) {
              const int jj = j + 4 * q + e;
              const float ssum = rank == 0 ? __fadd_rn(Y.ss[jj], X.ss[jj])
                                           : __fadd_rn(X.ss[jj], Y.ss[jj]);
              pe[e] *= rsqrtf(__fadd_rn(__fmul_rn(ssum, 1.0f / (float)D), p.eps));
            }
          }
          pk[2 * q] = pack_bf16(pe[0], pe[1]);
          pk[2 * q + 1] = pack_bf16(pe[2], pe[3]);
        }
        tmem_st8(t_sa + j / 2, pk);  // columns j/2 .. j/2+7 (S there is consumed)
      }
      l_run += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      mbar_arrive_remote(xempty_peer + a * 8);  // receive slot a consumed
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pready[a]);
      return true;
    };
    bool alive = ntile > 0 && send(0);
    for (int it = 1; alive && it < ntile; ++it) alive = send(it) && compute(it - 1);
    if (alive) compute(ntile - 1);
    // Epilogue: the O half and (rank 0) the running max / sum.
    if (!*abort_flag && wait_all(pvdone, (ntile - 1) & 1, p, abort_flag)) {
      tc_fence_after();
      float* dst = po + (int64_t)h * D;
      for (int c = 0; c < C::Dh; c += 32) {
        uint32_t v[32];
        tmem_ld32(t_o + lane_base + c, v);
        tmem_wait_ld();
        if (head_ok)
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dst + c + j) =
                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                            __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
      }
      if (rank == 0 && head_ok) {
        pml[h] = m_run;  // log2 domain
        pml[p.H + h] = l_run;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kAlloc);
  }
}

// Merge the split partials of one (row, head), fold in the sink, normalise,
// apply the inverse rotation, store bf16 (and the log-sum-exp).
__global__ void mqa_combine_kernel(const Params p, int D, const float* __restrict__ sink,
                                   __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ float so[];  // D floats
  const int row = blockIdx.x, h = blockIdx.y;
  const float* ml = p.part_ml + (int64_t)row * p.splits * 2 * p.H;
  const float LOG2E = 1.4426950408889634f;
  const float z = sink[h];
  __nv_bfloat16* o = out + ((int64_t)row * p.H + h) * D;
  if (z == INFINITY) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) o[d] = __float2bfloat16_rn(0.f);
    if (lse && threadIdx.x == 0) lse[(int64_t)row * p.H + h] = INFINITY;
    return;
  }
  const float z2 = z * LOG2E;  // log2 domain
  float M = z2;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, ml[(int64_t)s * 2 * p.H + h]);
  if (M == -INFINITY) {
    for (int d = threadIdx.x; d < D; d += blockDim.x) o[d] = __float2bfloat16_rn(0.f);
    if (lse && threadIdx.x == 0) lse[(int64_t)row * p.H + h] = -INFINITY;
    return;
  }
  float L = z2 == -INFINITY ? 0.f : exp2f(z2 - M);
  for (int s = 0; s < p.splits; ++s) {
    const float ms = ml[(int64_t)s * 2 * p.H + h];
    if (ms != -INFINITY) L += ml[(int64_t)s * 2 * p.H + p.H + h] * exp2f(ms - M);
  }
  const float invL = 1.0f / L;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      const float ms = ml[(int64_t)s * 2 * p.H + h];
      if (ms == -INFINITY) continue;
      acc = fmaf(p.part_o[(((int64_t)row * p.splits + s) * p.H + h) * D + d], exp2f(ms - M), acc);
    }
    so[d] = acc * invL;
  }
  __syncthreads();
  const int64_t pos = row_pos(p, row);
  const int half = p.R / 2, d0 = D - p.R;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float v = so[d];
    if (d >= d0 && p.R > 0) {
      const int j = (d - d0) % half;
      float sn, cs;
      sincos_reduced((double)pos * p.inv_freq[j], &sn, &cs);
      if (d - d0 < half)
        v = so[d] * cs + so[d + half] * sn;  // rotation by -angle
      else
        v = so[d] * cs - so[d - half] * sn;
    }
    o[d] = __float2bfloat16_rn(v);
  }
  if (lse && threadIdx.x == 0) lse[(int64_t)row * p.H + h] = (M + log2f(L)) / LOG2E;
}

template <int D, int R>
cudaError_t launch_impl(const MqaLaunch& a, cudaStream_t stream) {
  using C = MCfg<D>;
  Params p{};
  p.Q = a.Q;
  p.H = a.H;
  p.m = a.m;
  p.W = a.W;
  p.R = a.rope_dim;
  p.splits = a.splits;
  p.N_cap = a.N_cap;
  p.L_cap = a.L_cap;
  p.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  p.pos_q = a.pos_q;
  p.pos_base = a.pos_base;
  p.sel_idx = a.sel_idx;
  p.sel_cnt = a.sel_cnt;
  p.kmax = a.kmax;
  p.gamma_q = a.gamma_q;
  p.gamma_kv = a.gamma_kv;
  p.eps = a.eps;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.part_o = a.part_o;
  p.part_ml = a.part_ml;
  p.status = a.status;
  for (int j = 0; j < 64; ++j) p.inv_freq[j] = a.inv_freq[j];
  const int rows = a.B * a.Q;
  if (rows > 65535 || a.splits * 2 > 65535) return cudaErrorInvalidConfiguration;

  // Row-gather maps (one-row boxes) and 64-row box maps, 128-byte swizzle.
  CUtensorMap map_c, map_t, box_c, box_t;
  cudaError_t e = make_tmap_2d(&map_c, a.kv_c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                               (uint64_t)a.B * a.N_cap, D, 1, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&map_t, a.kv_tok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.B * a.L_cap,
                   D, 1, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&box_c, a.kv_c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.B * a.N_cap,
                   D, TN, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&box_t, a.kv_tok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.B * a.L_cap,
                   D, TN, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;

  const size_t smem = 1024 + (size_t)C::kStages * C::kStageBytes + 4 * sizeof(XSlot) +
                      C::kStages * sizeof(Meta) + 40 * 8 + 384 * 4 + 16;
  auto kern = mqa_pair_kernel<D, R>;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), 3 + (D == 512 ? 0 : 3) + R / 32, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * a.splits, rows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, map_c, map_t, box_c, box_t, p);
  if (e != cudaSuccess) return e;
  mqa_combine_kernel<<<dim3(rows, a.H), 128, D * sizeof(float), stream>>>(
      p, D, a.sink, reinterpret_cast<__nv_bfloat16*>(a.out), a.lse);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mqa(const MqaLaunch& a, cudaStream_t stream) {
  if (a.D == 512) {
    if (a.rope_dim == 64) return launch_impl<512, 64>(a, stream);
    if (a.rope_dim == 32) return launch_impl<512, 32>(a, stream);
    if (a.rope_dim == 0) return launch_impl<512, 0>(a, stream);
  } else if (a.D == 128) {
    if (a.rope_dim == 32) return launch_impl<128, 32>(a, stream);
    if (a.rope_dim == 0) return launch_impl<128, 0>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace csa
