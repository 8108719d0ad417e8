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
// Design.  The 128 x 512 fp32 output accumulator alone would fill the
// tensor memory of an SM, so the heads of a (query, split) are shared by two
// independent CTAs: CTA g owns heads [64g, 64g+64) with the full head dim
// and issues M = 64 MMAs.  An M = 64 accumulator occupies one 16-lane half of
// each TMEM sub-partition, so per CTA
//     O    (64 heads x D fp32)         lane half 0, columns 0 .. D-1
//     S    (64 heads x 64 fp32, x2)    lane half 1, columns 0 .. 127
//     Qhat (64 heads x D bf16 pairs)   lane half 1, columns 128 .. 128+D/2-1
// (the A operand of S = Qhat K^T is read from TMEM in the same lane half as
// the accumulator it feeds).  Per 64-entry tile:
//   - contiguous tiles (dense entries, window tokens) arrive by TMA boxes
//     issued by the producer warp; selected entries are gathered by the four
//     transform warps with 16-byte cp.async (two threads per row, a few
//     tiles ahead), which keeps many more rows in flight than per-row TMA
//     gathers; 128-byte swizzle either way, K = V = that tile;
//   - transform warps zero masked rows and, for window tokens, compute
//     1/rms(c_t), apply the KV gain and rotate the last R dims to the token
//     position (compressed entries are stored already rotated to theirs);
//   - the MMA warp issues S = Qhat K^T (TS form) into one of two S buffers,
//     then P V into O (P from shared memory, V = the same tile read
//     MN-major, in N <= 256 pieces);
//   - softmax warps (two threads per head row, 32 columns each, through the
//     16x32bx2 TMEM access) run an online softmax with lazy rescaling (O is
//     rescaled in TMEM only when the running max grows by more than 8) and
//     write P (bf16) to shared memory in the MMA's K-major layout.
// Splits of the KV list run on different CTAs; their (m, l, O) partials are
// merged, with the sink folded in and the inverse RoPE applied, by the CTAs
// themselves when the S splits of a head group form one thread-block
// cluster and all clusters of the launch fit at once (S <= 16: a cluster
// barrier, then each CTA merges a share of the heads from L2), else by
// mqa_combine_kernel.  With one split per row the
// attention CTA finishes its rows directly.  Every wait is bounded and
// reports CSA_ERR_DEVICE_TIMEOUT.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma.h"

namespace csa {

size_t mqa_workspace_bytes(int rows, int splits, int H, int D) {
  size_t o = (size_t)rows * splits * H * D * 2;  // fp16 partial outputs
  o = (o + 255) / 256 * 256;
  return o + (size_t)rows * splits * 2 * H * 4;
}

// Splits of each row's KV list over CTA pairs: at most one wave of pairs
// (rows * splits <= SMs / 2), no split left without a tile.
int mqa_choose_splits(int rows, int64_t compressed_max, int window, int num_sms, int H) {
  const int64_t tiles = (compressed_max + 63) / 64 + (window + 63) / 64;
  // One CTA per (row, split) owns up to 64 heads: H > 64 takes two.
  const int64_t units = std::max(1, num_sms / (H > 64 ? 2 : 1));
  int64_t s = std::max<int64_t>(1, units / std::max(1, rows));
  s = std::min<int64_t>(s, std::max<int64_t>(1, tiles));
  const int64_t tps = (tiles + s - 1) / s;
  s = std::max<int64_t>(1, (tiles + tps - 1) / tps);
  return (int)s;
}

namespace {

constexpr int TN = 64;         // KV rows per tile
constexpr int HC = 64;         // heads per CTA
constexpr int kThreads = 320;  // 10 warps
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct MCfg {
  static constexpr int NC = D / 64;                // 128-byte chunks per row
  static constexpr int kChunkBytes = TN * 128;     // one chunk of a tile
  static constexpr int kStageBytes = NC * kChunkBytes;
  static constexpr int kStages = D == 512 ? 3 : 4;
  static constexpr int kPBytes = HC * TN * 2;      // P tile, bf16
  static constexpr uint32_t kHalf1 = 16u << 16;    // TMEM lane offset of lane half 1
  static constexpr int kQCol = 2 * TN;             // Qhat columns start (half 1)
  static constexpr uint32_t kAlloc = (D <= 256 && kQCol + D / 2 <= 256) ? 256 : 512;
};

struct Meta {
  int32_t grow[TN];   // row coordinate in the tensor map
  int32_t pos[TN];    // RoPE position
  float rn[TN];       // window tokens: 1/rms(c_t); compressed entries: 1
  uint32_t valid[2];  // bit r: row r holds a real KV vector
  int32_t window;     // 1: window tokens; 0: compressed entries
  int32_t pad;
};

struct Params {
  int Q, H, m, W, R, splits;
  int64_t N_cap, L_cap;
  int64_t entry_offset;  // the cache holds entries entry_offset .. of the sequence
  // Cached entries below this bound were written before the call and are
  // read before pdl_wait(); see MqaLaunch.
  const int64_t* safe_pos;
  int64_t safe_fixed;
  const __nv_bfloat16* q;
  const int64_t* pos_q;
  int64_t pos_base;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  int kmax;
  const __nv_bfloat16* kv_c;
  const float* gamma_q;
  const float* gamma_kv;
  float eps, scale_log2;  // softmax scale * log2(e)
  __half* part_o;  // [rows, S, H, D]: the split's output divided by its sum
  float* part_ml;
  int32_t* status;
  // One split per row: the attention kernel finishes the rows itself (sink,
  // normalisation, inverse rotation, bf16 output and log-sum-exp) and no
  // merge runs.
  int fused;
  // Several splits per row, launched as one cluster per (row, head group):
  // after every CTA of the cluster has written its partial, the CTAs merge
  // them themselves (each a share of the group's heads) and no merge kernel
  // runs.
  int cluster_merge;
  const float* sink;
  __nv_bfloat16* out;
  float* lse;
  double inv_freq[64];
};

// Byte offset of (row r, dim d) inside a tile (128B-swizzled 64-dim chunks).
CSA_DEV uint32_t tile_off(int r, int d) {
  uint32_t lin = (uint32_t)r * 128u + (uint32_t)(d & 63) * 2u;
  return (uint32_t)(d >> 6) * (TN * 128u) + (lin ^ (((lin >> 7) & 7u) << 4));
}

CSA_DEV uint64_t desc_k(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }
CSA_DEV uint64_t desc_mn(uint32_t saddr) { return sdesc_sw128(saddr, TN * 128, 1024); }

CSA_DEV int64_t row_pos(const Params& p, int row) {
  return p.pos_q ? p.pos_q[row] : p.pos_base + row % p.Q;
}

template <bool kCluster = false>
CSA_DEV bool wait_all(uint64_t* bar, uint32_t parity, const Params& p, volatile int* abort_flag) {
  bool ok = mbar_wait<kCluster>(bar, parity, p.status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// Merge of the split partials of one (row, head) by one warp: fold in the
// sink, normalise, apply the inverse rotation, store bf16 (and the
// log-sum-exp).  Lane l owns dims [l*VPL, (l+1)*VPL) (VPL = D/32), so the
// output row leaves as one coalesced 32-lane store and the rotated pairs
// (d, d + R/2) sit in lanes l and l ^ (R/2/VPL).  The S (max, sum) pairs
// become one weight per split (wsplit: S floats of this warp's shared
// memory).  The first G splits' partials are loaded together with the
// (max, sum) pairs, so that with S <= G the warp waits on one round of L2
// reads; further groups of G follow one round each.
// kLdg: the partials come from an earlier kernel (read-only path); otherwise
// they were written during this kernel by other CTAs and are read from L2.
template <int D, int R, int G, bool kLdg>
CSA_DEV void merge_head(const Params& p, int row, int h, int lane, float* wsplit) {
  constexpr int VPL = D / 32;     // dims per lane: 16 (D = 512) or 4 (D = 128)
  constexpr int NW = VPL / 2;     // 32-bit words (fp16 pairs) per lane and split
  static_assert(VPL == 16 || VPL == 4, "D must be 512 or 128");
  const int S = p.splits;
  const float* ml = p.part_ml + (int64_t)row * S * 2 * p.H;
  const __half* src = p.part_o + ((int64_t)row * S * p.H + h) * D + lane * VPL;
  const int64_t stride = (int64_t)p.H * D;
  auto ld4 = [](const uint4* a) -> uint4 { return kLdg ? __ldg(a) : __ldcg(a); };
  auto ld2 = [](const uint2* a) -> uint2 { return kLdg ? __ldg(a) : __ldcg(a); };
  auto ldf = [](const float* a) -> float { return kLdg ? __ldg(a) : __ldcg(a); };
  auto load = [&](int s, uint32_t (&v)[NW]) {
    const __half* a = src + (int64_t)s * stride;
    if constexpr (VPL == 16) {
      *reinterpret_cast<uint4*>(&v[0]) = ld4(reinterpret_cast<const uint4*>(a));
      *reinterpret_cast<uint4*>(&v[4]) = ld4(reinterpret_cast<const uint4*>(a) + 1);
    } else {
      *reinterpret_cast<uint2*>(&v[0]) = ld2(reinterpret_cast<const uint2*>(a));
    }
  };
  uint32_t buf[G][NW];
#pragma unroll
  for (int u = 0; u < G; ++u)
    if (u < S) load(u, buf[u]);
  // Split `lane`'s (max, sum) pair, in flight with the partials.
  float m0 = -INFINITY, l0 = 0.f;
  if (lane < S) {
    m0 = ldf(ml + (int64_t)lane * 2 * p.H + h);
    l0 = ldf(ml + (int64_t)lane * 2 * p.H + p.H + h);
  }
  const float LOG2E = 1.4426950408889634f;
  const float z = p.sink[h];
  const float z2 = z * LOG2E;  // log2 domain
  float M = fmaxf(z2, m0);
  for (int s = lane + 32; s < S; s += 32) M = fmaxf(M, ldf(ml + (int64_t)s * 2 * p.H + h));
  M = warp_max(M);
  const bool zero = z == INFINITY || M == -INFINITY;  // +inf sink, or nothing to attend
  float L = 0.f;
  if (!zero) {
    for (int s = lane; s < S; s += 32) {
      const float ms = s == lane ? m0 : ldf(ml + (int64_t)s * 2 * p.H + h);
      const float ls = s == lane ? l0 : ldf(ml + (int64_t)s * 2 * p.H + p.H + h);
      const float w = ms == -INFINITY ? 0.f : ls * exp2f(ms - M);
      wsplit[s] = w;  // the split's stored output is O / l
      L += w;
    }
    L = warp_sum(L);
    if (z2 != -INFINITY) L += exp2f(z2 - M);
  }
  __syncwarp();
  __nv_bfloat16* o = p.out + ((int64_t)row * p.H + h) * D + lane * VPL;
  float acc[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
  if (!zero) {
    for (int s0 = 0; s0 < S; s0 += G) {
      if (s0 > 0) {
#pragma unroll
        for (int u = 0; u < G; ++u)
          if (s0 + u < S) load(s0 + u, buf[u]);
      }
#pragma unroll
      for (int u = 0; u < G; ++u) {
        if (s0 + u >= S) break;
        const float w = wsplit[s0 + u];
        if (w == 0.f) continue;  // empty split: its partial was never written
#pragma unroll
        for (int i = 0; i < NW; ++i) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&buf[u][i]));
          acc[2 * i] = fmaf(f.x, w, acc[2 * i]);
          acc[2 * i + 1] = fmaf(f.y, w, acc[2 * i + 1]);
        }
      }
    }
    const float invL = 1.0f / L;
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] *= invL;
    if constexpr (R > 0) {
      // Rotation by -pos: pair j of the last R dims is (d0 + j, d0 + j + R/2).
      constexpr int K = R / 2 / VPL;  // lanes per rotated half
      constexpr int L0 = 32 - 2 * K;  // first lane holding rotated dims
      static_assert(K >= 1 && (K & (K - 1)) == 0, "rotated halves must span whole lanes");
      const int64_t pos = row_pos(p, row);
      float sn = 0.f, cs = 1.f;
      if (lane < R / 2) sincos_reduced((double)pos * p.inv_freq[lane], &sn, &cs);
      const bool rot = lane >= L0;
      const bool first = rot && lane - L0 < K;
      const int jb = rot ? ((lane - L0) % K) * VPL : 0;
#pragma unroll
      for (int e = 0; e < VPL; ++e) {
        const float c = __shfl_sync(0xffffffffu, cs, jb + e);
        const float sj = __shfl_sync(0xffffffffu, sn, jb + e);
        const float other = __shfl_xor_sync(0xffffffffu, acc[e], K);
        if (rot) acc[e] = first ? acc[e] * c + other * sj : acc[e] * c - other * sj;
      }
    }
  }
  uint32_t packed[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) packed[i] = pack_bf16(acc[2 * i], acc[2 * i + 1]);
  if constexpr (VPL == 16) {
    reinterpret_cast<uint4*>(o)[0] = *reinterpret_cast<const uint4*>(&packed[0]);
    reinterpret_cast<uint4*>(o)[1] = *reinterpret_cast<const uint4*>(&packed[4]);
  } else {
    *reinterpret_cast<uint2*>(o) = *reinterpret_cast<const uint2*>(&packed[0]);
  }
  if (p.lse && lane == 0)
    p.lse[(int64_t)row * p.H + h] =
        zero ? (z == INFINITY ? INFINITY : -INFINITY) : (M + log2f(L)) / LOG2E;
}

// The split merge as its own kernel (several splits per row when the
// in-cluster merge is not available): one warp per (row, head), four per CTA.
template <int D, int R, int G>
__global__ void __launch_bounds__(128) mqa_combine_kernel(const Params p, int rows) {
  extern __shared__ float wsm[];  // [4 warps][S] split weights
  pdl_trigger();
  pdl_wait();  // the partials come from the attention kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * 4 + warp;
  if (gw >= (int64_t)rows * p.H) return;
  merge_head<D, R, G, true>(p, (int)(gw / p.H), (int)(gw % p.H), lane, wsm + warp * p.splits);
}

template <int D, int R>
__global__ void __launch_bounds__(kThreads, 1)
    mqa_heads_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap box_c,
                     const __grid_constant__ CUtensorMap box_t, const Params p) {
  using C = MCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* pbuf = stages + C::kStages * C::kStageBytes;  // [2] P tiles
  Meta* meta = reinterpret_cast<Meta*>(pbuf + 2 * C::kPBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta + C::kStages);
  uint64_t* full = bars;
  uint64_t* ready = full + C::kStages;
  uint64_t* empty = ready + C::kStages;
  uint64_t* sfull = empty + C::kStages;
  uint64_t* pfull = sfull + 2;
  uint64_t* pvdone = pfull + 2;  // [2]: P.V of tiles with parity 0 / 1
  uint64_t* qready = pvdone + 2;
  uint64_t* drain = qready + 1;
  uint64_t* done = drain + 1;  // one arrival per warp when its role is over
  uint64_t* qfull = done + 1;  // the query block landed in the last stage
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // The gains, staged once by the warps that use them: [0, D) gamma_q,
  // [D, 2D) gamma_kv (ones where not given).
  float* gam_s = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(abort_flag + 1) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  pdl_trigger();
  // H > 64: CTA g*S + s (g = 0, 1) owns heads [64g, 64g+64) of split s, so
  // the S splits of one head group are consecutive (one cluster when the
  // partials are merged in-cluster).
  const bool pair = p.H > HC;
  // Sparse decode without the in-cluster merge: the CTAs of every head
  // group's last split (the window tiles, which wait for no other kernel of
  // the call) come first in launch order, so CTAs that start late, on SMs the
  // top-k frees, hold only selected tiles.
  int gx = (int)blockIdx.x, gy = (int)blockIdx.y;
  if (p.Q == 1 && p.sel_idx != nullptr && !p.cluster_merge && p.splits > 1) {
    const int64_t G = (int64_t)gridDim.x / p.splits;  // head groups per row
    const int64_t ng = G * gridDim.y;
    const int64_t L = (int64_t)blockIdx.x + (int64_t)gridDim.x * blockIdx.y;
    const int64_t grp = L < ng ? L : (L - ng) / (p.splits - 1);
    const int64_t sp = L < ng ? p.splits - 1 : (L - ng) % (p.splits - 1);
    gy = (int)(grp / G);
    gx = (int)((grp % G) * p.splits + sp);
  }
  const int hg0 = pair ? (gx / p.splits) * HC : 0;  // first head of this CTA
  const int split = gx % p.splits;
  const int row = gy;
  const int b = row / p.Q;

  // The KV list of this query row: n_c compressed entries, then the window.
  const int64_t pos = row_pos(p, row);
  int64_t n_vis = pos < 0 ? 0 : (pos + 1) / p.m - p.entry_offset;
  if (n_vis < 0) n_vis = 0;
  if (n_vis > p.N_cap) n_vis = p.N_cap;
  const int64_t w0 = pos - p.W + 1 < 0 ? 0 : pos - p.W + 1;
  const int nwin = (p.W > 0 && pos >= 0) ? (int)(pos - w0 + 1) : 0;
  // This split's tiles [t0, t1) of the list; the selection count comes from
  // the top-k kernel, so every role calls this after pdl_wait().
  // With a selection the list is laid out for kmax entries (the tiles past
  // the selection count hold only masked rows), so the tile range does not
  // wait for the count; the count is read after pdl_wait() where needed.
  const int n_list = p.sel_idx ? p.kmax : (int)n_vis;
  const int tiles_c = (n_list + TN - 1) / TN;
  const int tiles_all = tiles_c + (nwin + TN - 1) / TN;
  const int tps = (tiles_all + p.splits - 1) / p.splits;
  const int t0 = std::min(split * tps, tiles_all);
  const int t1 = std::min(t0 + tps, tiles_all);
  const int ntile = t1 - t0;
  auto sel_count = [&]() -> int {
    if (!p.sel_idx) return (int)n_vis;
    const int c = p.sel_cnt[row];
    return c < 0 ? 0 : (c > p.kmax ? p.kmax : c);
  };
  // Tiles that read nothing the previous kernel of the call writes: window
  // tokens (caller inputs) and, without a selection, tiles whose visible
  // entries all lie below the safe bound (written before the call).  Only
  // the roles that read cached entries or the selection wait, just before
  // the first tile that is not safe; a selection is never safe.
  int64_t safe_e = 0;
  if (!p.sel_idx) {
    if (p.safe_pos) {
      const int64_t sp = p.safe_pos[b];
      safe_e = (sp < 0 ? 0 : sp / p.m) - p.entry_offset;
    } else {
      safe_e = p.safe_fixed;
    }
  }
  auto tile_safe = [&](int t) -> bool {
    if (t >= tiles_c) return true;
    if (p.sel_idx) return false;
    const int64_t end = (int64_t)(t + 1) * TN < n_vis ? (int64_t)(t + 1) * TN : n_vis;
    return end <= safe_e;
  };
  // The selection count is read only by CTAs with selected tiles (after
  // their wait).
  const bool sel_tiles = p.sel_idx != nullptr && t0 < tiles_c;

  float* pml = p.part_ml + ((int64_t)row * p.splits + split) * 2 * p.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1 + 128);  // producer + the transform threads
      mbar_init(&ready[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&pfull[a], 128);
    }
    mbar_init(&pvdone[0], 1);
    mbar_init(&pvdone[1], 1);
    mbar_init(qready, 128);
    mbar_init(drain, 1);
    mbar_init(done, kThreads / 32);
    mbar_init(qfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem + C::kHalf1;             // S buffers (lane half 1)
  const uint32_t t_q = tmem + C::kHalf1 + C::kQCol;  // Qhat (lane half 1)
  const uint32_t t_o = tmem;                         // O (lane half 0)

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    // Contiguous tiles (dense entries, window tokens): one 64-row box per
    // 128-byte chunk.  Selected entries: this warp only writes the row
    // metadata; the transform warps gather the rows.
    // The query block first (a caller input: no need to wait for the
    // previous kernel): 64 heads x D into the last stage, freed by qready.
    if (lane == 0) {
      mbar_expect_tx(qfull, C::kStageBytes);
      for (int c = 0; c < C::NC; ++c)
        tma_load_2d(stages + (C::kStages - 1) * C::kStageBytes + c * C::kChunkBytes, &map_q, qfull,
                    c * 64, row * p.H + hg0);
    }
    bool waited = false;
    auto ensure = [&](int t) {
      if (!waited && !tile_safe(t)) {
        pdl_wait();
        waited = true;
      }
    };
    // Selected indices of the next tile are loaded one tile ahead, and
    // independently of the selection count (both round trips overlap).
    auto load_idx = [&](int t, int hh) -> int64_t {
      const int j = t * TN + lane + 32 * hh;
      return (p.sel_idx && t < tiles_c && j < p.kmax) ? (int64_t)p.sel_idx[(int64_t)row * p.kmax + j]
                                                       : 0;
    };
    if (t0 < t1) ensure(t0);
    int64_t nxt0 = t0 < t1 ? load_idx(t0, 0) : 0, nxt1 = t0 < t1 ? load_idx(t0, 1) : 0;
    const int n_c = sel_tiles ? sel_count() : (p.sel_idx ? 0 : (int)n_vis);
    int it = 0;
    for (int t = t0; t < t1; ++t, ++it) {
      const int64_t cur[2] = {nxt0, nxt1};
      if (t + 1 < t1) {
        ensure(t + 1);
        nxt0 = load_idx(t + 1, 0);
        nxt1 = load_idx(t + 1, 1);
      }
      const int s = it % C::kStages;
      const uint32_t ph = (it / C::kStages) & 1;
      // The last stage holds the query block until the prologue is done.
      if (it == C::kStages - 1 && !wait_all(qready, 0, p, abort_flag)) break;
      const bool win = t >= tiles_c;
      const bool gathered = !win && p.sel_idx != nullptr;
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
            i = cur[hh];
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
        if (gathered)
          mbar_arrive(&full[s]);  // the transform warps gather the rows
        else
          mbar_expect_tx(&full[s], C::kStageBytes);
      }
      __syncwarp();
      if (!gathered) {
        // Rows grow[0] .. grow[0]+63 are consecutive (rows past the list are
        // fetched too and masked; rows past the tensor are zero-filled).
        uint8_t* dst = stages + s * C::kStageBytes;
        const int32_t y0 = __shfl_sync(0xffffffffu, grow[0], 0);
        if (lane < C::NC)
          tma_load_2d(dst + lane * C::kChunkBytes, win ? &box_t : &box_c, &full[s],
                      (int32_t)(lane * 64), y0);
      }
    }
    if (*abort_flag && lane == 0) {  // box copies still in flight must land first
      for (int j = std::max(0, it - C::kStages); j < it; ++j)
        if (t0 + j >= tiles_c || p.sel_idx == nullptr)
          mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.status);
    }
    // A CTA whose tiles were all safe still waits once, so that the grid
    // does not complete before the previous kernel.
    if (!waited) pdl_wait();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    constexpr int kPvN = D >= 256 ? 256 : D;  // N of one P.V instruction
    const uint32_t idesc_s = idesc_bf16(64, TN, 0, 0);
    const uint32_t idesc_pv = idesc_bf16(64, kPvN, 0, 1);
    const bool ok = wait_all(qready, 0, p, abort_flag);
    tc_fence_after();
    bool issued = false;
    auto issue_pv = [&](int jt) -> bool {
      const int a = jt & 1, s = jt % C::kStages;
      if (!wait_all(&pfull[a], (jt >> 1) & 1, p, abort_flag)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t vbase = smem_u32(stages + s * C::kStageBytes);
        const uint32_t pb = smem_u32(pbuf + a * C::kPBytes);
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk)
#pragma unroll
          for (int n = 0; n < D / kPvN; ++n)
            mma_bf16_ss(t_o + n * kPvN, desc_k(pb + kk * 32),
                        desc_mn(vbase + (n * kPvN / 64) * C::kChunkBytes + kk * 16 * 128),
                        idesc_pv, (jt > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&pvdone[jt & 1]);
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
        for (int kk = 0; kk < D / 16; ++kk)
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
    // Two threads per tile row.  Window tokens: 1/rms(c_t) over the full row
    // and the KV gain in place.  Every real row: RoPE on the rotated dims.
    const int tid = threadIdx.x - 64;  // 0..127
    const int r = tid >> 1, hf = tid & 1;
    for (int i = tid; i < D; i += 128) gam_s[D + i] = p.gamma_kv ? __ldg(p.gamma_kv + i) : 1.f;
    named_barrier_sync(2, 128);  // the transform warps
    if (sel_tiles) pdl_wait();  // selected rows are gathered here
    const int n_c = sel_tiles ? sel_count() : (p.sel_idx ? 0 : (int)n_vis);
    // Tile `it`: selected entries are fetched here (thread pair r gathers
    // row r, half hf each, 16 bytes per cp.async) once the stage is free;
    // every thread then arrives on full[s] (after its copies land).
    // Gathers: transform warp tw copies rows tw, tw+4, ..., tw+60 of the
    // tile, a whole row per pair of instructions (lane l: 16 bytes at
    // 16*l and 512+16*l), so each instruction reads 512 contiguous bytes.
    // Lane l (< 16) holds the index of row tw + 4*l, loaded ahead.
    const int tw = tid >> 5, tl = tid & 31;
    auto row_index = [&](int it) -> int64_t {
      const int t = t0 + it, j = t * TN + tw + 4 * (tl & 15);
      return (p.sel_idx && t < tiles_c && j < p.kmax) ? (int64_t)p.sel_idx[(int64_t)row * p.kmax + j]
                                                       : 0;
    };
    auto fetch = [&](int it, int64_t i) -> bool {
      const int s = it % C::kStages;
      const int t = t0 + it;
      if (p.sel_idx != nullptr && t < tiles_c) {
        const int j = t * TN + tw + 4 * (tl & 15);
        if (j >= n_c || i < 0 || i >= n_vis) i = -1;  // masked row: not fetched (zeroed later)
        if (!wait_all(&empty[s], ((it / C::kStages) & 1) ^ 1, p, abort_flag)) return false;
        if (it == C::kStages - 1 && !wait_all(qready, 0, p, abort_flag)) return false;
        uint8_t* st = stages + s * C::kStageBytes;
        constexpr int kUnits = D / 8;  // 16-byte units per row
#pragma unroll 4
        for (int u = 0; u < TN / 4; ++u) {
          const int64_t iu = __shfl_sync(0xffffffffu, i, u);
          if (iu < 0) continue;
          const int rr = tw + 4 * u;
          const __nv_bfloat16* src = p.kv_c + ((int64_t)b * p.N_cap + iu) * D;
#pragma unroll
          for (int h = 0; h < (kUnits + 31) / 32; ++h) {
            const int unit = 32 * h + tl;
            if (unit < kUnits) cp_async_16(st + tile_off(rr, 8 * unit), src + 8 * unit);
          }
        }
        cp_async_arrive(&full[s]);
      } else {
        mbar_arrive(&full[s]);
      }
      return true;
    };
    constexpr int kAhead = C::kStages - 1;
    bool fetch_ok = true;
    {
      int64_t ri[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u) ri[u] = u < ntile ? row_index(u) : 0;
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
        if (u < ntile && fetch_ok) fetch_ok = fetch(u, ri[u]);
    }
    int64_t nxt = kAhead < ntile ? row_index(kAhead) : 0;
    for (int it = 0; it < ntile && fetch_ok; ++it) {
      const int s = it % C::kStages;
      if (!wait_all(&full[s], (it / C::kStages) & 1, p, abort_flag)) break;
      Meta& M = meta[s];
      uint8_t* st = stages + s * C::kStageBytes;
      const bool valid = (M.valid[r >> 5] >> (r & 31)) & 1u;
      if (!valid) {  // masked rows enter P.V with P = 0: make them finite zeros
        for (int c = hf; c < D / 8; c += 2)
          *reinterpret_cast<uint4*>(st + tile_off(r, c * 8)) = make_uint4(0u, 0u, 0u, 0u);
      }
      float ss = 0.f;
      if (valid && M.window) {
        float a4[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains, loads in flight
#pragma unroll 8
        for (int c = hf; c < D / 8; c += 2) {  // 16-byte units
          uint4 u = *reinterpret_cast<const uint4*>(st + tile_off(r, c * 8));
          uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = bf16_lo(w4[e]), hi = bf16_hi(w4[e]);
            a4[e] = fmaf(lo, lo, fmaf(hi, hi, a4[e]));
          }
          if (p.gamma_kv) {
            const float* g = gam_s + D + c * 8;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w4[e] = pack_bf16(bf16_lo(w4[e]) * g[2 * e], bf16_hi(w4[e]) * g[2 * e + 1]);
            *reinterpret_cast<uint4*>(st + tile_off(r, c * 8)) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        ss = (a4[0] + a4[1]) + (a4[2] + a4[3]);
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      if (hf == 0) M.rn[r] = (valid && M.window) ? 1.0f / sqrtf(ss / (float)D + p.eps) : 1.0f;
      __syncwarp();  // gain-scaled values are in place before the rotation reads them
      if constexpr (R > 0) {
        if (valid && M.window) {  // compressed entries are stored rotated
          // Pairs (j, j+R/2) of the last R dims; thread half hf rotates pairs
          // [hf*R/4, hf*R/4 + R/4) with 16-byte accesses (8 bf16 each).
          constexpr int half = R / 2;
          constexpr int d0 = D - R;
          const double ppos = (double)M.pos[r];
#pragma unroll
          for (int qq = 0; qq < R / 32; ++qq) {
            const int j0 = hf * (half / 2) + qq * 8;
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
      }
      fence_proxy_async_smem();
      mbar_arrive(&ready[s]);
      if (it + kAhead < ntile) {
        const int64_t cur = nxt;
        if (it + kAhead + 1 < ntile) nxt = row_index(it + kAhead + 1);
        fetch_ok = fetch(it + kAhead, cur);
      }
    }
    cp_async_wait_all();  // no copy may still target shared memory at exit
  } else {
    // ------------------------------------------------- softmax / epilogue --
    // The warp with TMEM lane quarter q serves heads 16q .. 16q+15 of this
    // CTA; thread t: head 16q + (t & 15), columns [32*(t>>4), +32).
    const int q = warp & 3;
    const int hl = 16 * q + (lane & 15);  // head within the CTA
    const int hf = lane >> 4;             // column half
    const int hg = hg0 + hl;              // global head
    const bool head_ok = hg < p.H;
    const uint32_t lq = (uint32_t)(32 * q) << 16;  // lane base of this quarter
    // Query prologue: qhat = RoPE(RMSNorm(q) * gamma_q), bf16 pairs -> TMEM.
    // Thread half hf holds dims [hf*D/2, hf*D/2 + D/2), i.e. Qhat columns
    // [hf*D/4, hf*D/4 + D/4): one 16x32bx2 store (second half at +D/4
    // columns) writes 64 dims of both halves.  The rotated dims (the last R)
    // all sit in the last 64-dim chunk of half 1.
    {
      for (int i = threadIdx.x - 192; i < D; i += 128)
        gam_s[i] = p.gamma_q ? __ldg(p.gamma_q + i) : 1.f;
      named_barrier_sync(1, 128);  // the softmax warps
      // The block is in the last stage (TMA, 128-byte swizzled chunks):
      // row hl, dims [hf*D/2, hf*D/2 + D/2).
      const uint8_t* qs = stages + (C::kStages - 1) * C::kStageBytes;
      const int d_half = hf * (D / 2);
      constexpr int NU = D / 16;  // 16-byte units of a half row
      // The query's rotation angles (one position for every head): lane j
      // of each softmax warp computes pair j into the (still unused) P
      // buffer, so the rotating threads read them instead of each
      // recomputing all of them.
      float2* qang = reinterpret_cast<float2*>(pbuf) + 32 * q;
      if constexpr (R > 0) {
        if (lane < R / 2) {
          float sn, cs;
          sincos_reduced((double)pos * p.inv_freq[lane], &sn, &cs);
          qang[lane] = make_float2(sn, cs);
        }
        __syncwarp();
      }
      const bool qok = wait_all(qfull, 0, p, abort_flag);
      // Sum of squares in packed FMAs: word e of each 16-byte unit in pair
      // accumulator e (its low and high halves in the two lanes).
      float2 a2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll 8
      for (int c = 0; c < NU; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(qs + tile_off(hl, d_half + 8 * c));
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = make_float2(bf16_lo(w4[e]), bf16_hi(w4[e]));
          a2[e] = fma_f32x2(x, x, a2[e]);
        }
      }
      float ss = ((a2[0].x + a2[0].y) + (a2[1].x + a2[1].y)) +
                 ((a2[2].x + a2[2].y) + (a2[3].x + a2[3].y));
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);  // the row's other half
      const float inv = (head_ok && qok) ? 1.0f / sqrtf(ss / (float)D + p.eps) : 0.f;
      const float* gq = gam_s + hf * (D / 2);
      constexpr int kChunks = D / 128;  // 64-dim chunks per half row
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        // x = (q * inv) * gamma, two dims per packed multiply.
        float x[64];
        const float2 inv2 = make_float2(inv, inv);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v =
              *reinterpret_cast<const uint4*>(qs + tile_off(hl, d_half + 64 * c + 8 * u));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          const float4 ga = *reinterpret_cast<const float4*>(gq + 64 * c + 8 * u);
          const float4 gb = *reinterpret_cast<const float4*>(gq + 64 * c + 8 * u + 4);
          const float2 g2[4] = {make_float2(ga.x, ga.y), make_float2(ga.z, ga.w),
                                make_float2(gb.x, gb.y), make_float2(gb.z, gb.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 y =
                mul_f32x2(mul_f32x2(make_float2(bf16_lo(w4[e]), bf16_hi(w4[e])), inv2), g2[e]);
            x[8 * u + 2 * e] = y.x;
            x[8 * u + 2 * e + 1] = y.y;
          }
        }
        if constexpr (R > 0) {
          if (hf == 1 && c == kChunks - 1) {
            constexpr int half = R / 2, b0 = 64 - R;
#pragma unroll
            for (int j = 0; j < half; ++j) {
              const float2 sc = qang[j];
              const float sn = sc.x, cs = sc.y;
              const float a1 = x[b0 + j], a2 = x[b0 + half + j];
              x[b0 + j] = a1 * cs - a2 * sn;
              x[b0 + half + j] = a2 * cs + a1 * sn;
            }
          }
        }
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(x[2 * e], x[2 * e + 1]);
        tmem_st_16x32bx2_x32<D / 4>(t_q + lq + 32 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(qready);
    }
    // (No wait: these warps read only tiles the producer and the transform
    // warps have made ready, which waited where a tile needed it.)

    float m_run = -INFINITY, l_run = 0.f;
    for (int it = 0; it < ntile; ++it) {
      const int s = it % C::kStages, a = it & 1;
      if (!wait_all(&sfull[a], (it >> 1) & 1, p, abort_flag)) break;
      tc_fence_after();
      float sv[32];
      {
        uint32_t v[32];
        tmem_ld_16x32bx2_x32<32>(t_s + lq + a * TN, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[j] = __uint_as_float(v[j]);
      }
      if (!wait_all(&ready[s], (it / C::kStages) & 1, p, abort_flag)) break;
      const Meta& M = meta[s];
      const bool win = M.window != 0;
      const uint32_t vw = M.valid[hf];
      // Logits (log2 domain); window columns times 1/rms(c_t).
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float x = sv[j];
        if (win) x *= M.rn[32 * hf + j];
        x = ((vw >> j) & 1u) ? x * p.scale_log2 : -INFINITY;
        sv[j] = x;
        m4[j & 3] = fmaxf(m4[j & 3], x);
      }
      float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));  // the row's other half
      // Online softmax with lazy rescaling.
      const bool grow = mt > m_run + kRescaleThreshold * 1.4426950408889634f || m_run == -INFINITY;
      const float m_new = grow ? fmaxf(mt, m_run) : m_run;
      const bool need = grow && m_run != -INFINITY;
      // P buffer a was last read by P.V of tile it-2; rescaling O needs
      // every earlier P.V complete (the latest is tile it-1).  pvdone[x]
      // completes once per tile of parity x, and tile it's P.V cannot be
      // issued before pfull(it) below, so neither wait can see its barrier
      // two phases ahead.  Without a rescale, P.V(it-1) overlaps this tile.
      const bool rescale = __any_sync(0xffffffffu, need) && it > 0;
      if (rescale) {
        if (!wait_all(&pvdone[(it - 1) & 1], ((it - 1) >> 1) & 1, p, abort_flag)) break;
        tc_fence_after();
      } else if (it >= 2) {
        if (!wait_all(&pvdone[it & 1], ((it - 2) >> 1) & 1, p, abort_flag)) break;
      }
      if (rescale) {
        const float f = need ? fast_exp2(m_run - m_new) : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 2; c += 32) {
          uint32_t v[32];
          tmem_ld_16x32bx2_x32<D / 2>(t_o + lq + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * f);
          tmem_st_16x32bx2_x32<D / 2>(t_o + lq + c, v);
        }
        tmem_wait_st();
      }
      if (need) l_run *= fast_exp2(m_run - m_new);
      m_run = m_new;
      // P = 2^(logit - m) (times the window norm: V = norm * stored row) in
      // bf16, into P buffer a: row hl, columns [32hf, 32hf+32), K-major with
      // the 128-byte swizzle.
      const bool live = m_run != -INFINITY;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float p0 = live ? fast_exp2(sv[j] - m_run) : 0.f;
        float p1 = live ? fast_exp2(sv[j + 1] - m_run) : 0.f;
        l4[j & 3] += p0;
        l4[(j + 1) & 3] += p1;
        if (win) {
          p0 *= M.rn[32 * hf + j];
          p1 *= M.rn[32 * hf + j + 1];
        }
        pk[j / 2] = pack_bf16(p0, p1);
      }
      float ls = (l4[0] + l4[1]) + (l4[2] + l4[3]);
      ls += __shfl_xor_sync(0xffffffffu, ls, 16);
      l_run += ls;
      uint8_t* prow = pbuf + a * C::kPBytes + hl * 128;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int chunk = 4 * hf + u;
        *reinterpret_cast<uint4*>(prow + ((chunk ^ (hl & 7)) << 4)) =
            make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&pfull[a]);
    }
    // Epilogue: this CTA's O rows and running max / sum (an empty split
    // leaves an empty partial).  With one split (p.fused) the rows are
    // finished here: out = RoPE^-1(O * 2^(m - M) / L) with M = max(m, z) and
    // L = l * 2^(m - M) + 2^(z - M) (log2 domain; z the head's sink).
    const float LOG2E = 1.4426950408889634f;
    const float zs = (p.fused && head_ok) ? p.sink[hg] : 0.f;
    const float z2 = zs * LOG2E;
    if (ntile <= 0) {
      if (p.fused) {
        // Nothing to attend: a zero row; the log-sum-exp is the sink's.
        if (head_ok) {
          uint4* o4 = reinterpret_cast<uint4*>(p.out + ((int64_t)row * p.H + hg) * D + hf * (D / 2));
          for (int i = 0; i < D / 16; ++i) o4[i] = make_uint4(0u, 0u, 0u, 0u);
          if (p.lse && hf == 0) p.lse[(int64_t)row * p.H + hg] = zs;
        }
      } else if (head_ok && hf == 0) {
        pml[hg] = -INFINITY;
        pml[p.H + hg] = 0.f;
      }
    } else if (!*abort_flag &&
               wait_all(&pvdone[(ntile - 1) & 1], ((ntile - 1) >> 1) & 1, p, abort_flag)) {
      tc_fence_after();
      // O / l rows (fp16: |O / l| is at most the largest |v|) go through
      // shared memory (the stages are free now: every MMA has completed)
      // and leave as one bulk copy per half row.
      void* po = p.fused
                     ? static_cast<void*>(p.out + ((int64_t)row * p.H + (head_ok ? hg : 0)) * D +
                                          hf * (D / 2))
                     : static_cast<void*>(p.part_o + (((int64_t)row * p.splits + split) * p.H +
                                                      (head_ok ? hg : 0)) * D + hf * (D / 2));
      constexpr int kORow = D * 2 + 16;  // padded row: spreads the banks
      uint8_t* ob = stages + hl * kORow + hf * D;
      float scale = l_run > 0.f ? 1.0f / l_run : 0.f;
      float M = m_run, L = l_run;
      bool zero = false;
      float ang_s = 0.f, ang_c = 1.f;
      if (p.fused) {
        M = fmaxf(m_run, z2);
        zero = zs == INFINITY || M == -INFINITY;
        if (!zero) {
          const float wm = m_run == -INFINITY ? 0.f : exp2f(m_run - M);
          L = l_run * wm + (z2 == -INFINITY ? 0.f : exp2f(z2 - M));
          scale = wm / L;
        } else {
          scale = 0.f;
        }
        if constexpr (R > 0) {
          if (lane < R / 2) sincos_reduced((double)pos * p.inv_freq[lane], &ang_s, &ang_c);
        }
      }
#pragma unroll 1
      for (int c = 0; c < D / 2; c += 64) {  // two 32-column loads per wait
        uint32_t v[64];
        tmem_ld_16x32bx2_x32<D / 2>(t_o + lq + c, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld_16x32bx2_x32<D / 2>(t_o + lq + c + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (p.fused) {
          if constexpr (R > 0) {
            // The rotated dims (the last R) are the end of this chunk in
            // half 1: pair j is (v[64-R+j], v[64-R/2+j]); rotation by -pos.
            if (c == D / 2 - 64) {
#pragma unroll
              for (int j = 0; j < R / 2; ++j) {
                const float cs = __shfl_sync(0xffffffffu, ang_c, j);
                const float sn = __shfl_sync(0xffffffffu, ang_s, j);
                if (hf == 1) {
                  const float x1 = __uint_as_float(v[64 - R + j]);
                  const float x2 = __uint_as_float(v[64 - R / 2 + j]);
                  v[64 - R + j] = __float_as_uint(x1 * cs + x2 * sn);
                  v[64 - R / 2 + j] = __float_as_uint(x2 * cs - x1 * sn);
                }
              }
            }
          }
#pragma unroll
          for (int j = 0; j < 64; j += 8) {
            uint4 u;
            u.x = pack_bf16(__uint_as_float(v[j]) * scale, __uint_as_float(v[j + 1]) * scale);
            u.y = pack_bf16(__uint_as_float(v[j + 2]) * scale, __uint_as_float(v[j + 3]) * scale);
            u.z = pack_bf16(__uint_as_float(v[j + 4]) * scale, __uint_as_float(v[j + 5]) * scale);
            u.w = pack_bf16(__uint_as_float(v[j + 6]) * scale, __uint_as_float(v[j + 7]) * scale);
            *reinterpret_cast<uint4*>(ob + 2 * (c + j)) = u;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 64; j += 8) {
            uint4 u;
            u.x = h2_bits(__floats2half2_rn(__uint_as_float(v[j]) * scale, __uint_as_float(v[j + 1]) * scale));
            u.y = h2_bits(__floats2half2_rn(__uint_as_float(v[j + 2]) * scale, __uint_as_float(v[j + 3]) * scale));
            u.z = h2_bits(__floats2half2_rn(__uint_as_float(v[j + 4]) * scale, __uint_as_float(v[j + 5]) * scale));
            u.w = h2_bits(__floats2half2_rn(__uint_as_float(v[j + 6]) * scale, __uint_as_float(v[j + 7]) * scale));
            *reinterpret_cast<uint4*>(ob + 2 * (c + j)) = u;
          }
        }
      }
      if (head_ok) {
        if (p.cluster_merge && !p.fused) {
          // Plain stores: the other CTAs of the cluster read the partial
          // back after the cluster barrier below.
          const uint4* s4 = reinterpret_cast<const uint4*>(ob);
          uint4* g4 = reinterpret_cast<uint4*>(po);
#pragma unroll 8
          for (int i = 0; i < D / 16; ++i) g4[i] = s4[i];
        } else {
          fence_proxy_async_smem();
          bulk_store(po, ob, (D / 2) * 2);
          bulk_commit();
          bulk_wait_read();  // shared memory may be released; the kernel end publishes the data
        }
      }
      if (head_ok && hf == 0) {
        if (p.fused) {
          if (p.lse)
            p.lse[(int64_t)row * p.H + hg] =
                zero ? (zs == INFINITY ? INFINITY : -INFINITY) : (M + log2f(L)) / LOG2E;
        } else {
          pml[hg] = m_run;  // log2 domain
          pml[p.H + hg] = l_run;
        }
      }
    }
  }
  // Teardown: every warp reports (converged) that it is done with tensor
  // memory; warp 0 frees it after all of them (bounded wait).
  __syncwarp();
  tc_fence_before();
  if (lane == 0) mbar_arrive(done);
  if (warp == 0) {
    wait_all(done, 0, p, nullptr);
    tc_fence_after();
    tmem_dealloc(tmem, C::kAlloc);
  }
  if (p.cluster_merge) {
    // Every CTA of the cluster (the S splits of this head group) has written
    // its partial and its (max, sum): the release / acquire cluster barrier
    // publishes them, and CTA `split` then merges heads split, split + S, ...
    // of the group, one warp per head.  Every thread of every CTA reaches
    // this point exactly once (no role returns early).
    __threadfence();
    __syncwarp();
    cluster_sync();
    const int nh = pair ? min(HC, p.H - hg0) : p.H;
    float* wsplit = reinterpret_cast<float*>(stages) + warp * 32;  // S <= 16 weights
    for (int j = split + p.splits * warp; j < nh; j += p.splits * (kThreads / 32))
      merge_head<D, R, 4, false>(p, row, hg0 + j, lane, wsplit);
  }
}

// How many clusters of S attention CTAs (one per SM) can be resident at once
// on this device (S <= 8 portable, up to 16 with the non-portable cluster
// size); 0 when none can.  Cached per (device, kernel variant, S).
int clusters_resident(const void* kern, int variant, int S, size_t smem) {
  static int cached[64][8][17] = {};  // 0 unknown, else count + 1
  if (S < 2 || S > 16) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || variant < 0 || variant >= 8)
    return 0;
  int& c = cached[dev][variant][S];
  if (c) return c - 1;
  bool ok = true;
  if (S > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                   cudaSuccess)
    ok = false;
  if (ok) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(S, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    ok = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1;
    c = ok ? n + 1 : 1;
  } else {
    c = 1;
  }
  if (!ok) cudaGetLastError();  // a refused query is not the caller's error
  return c - 1;
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
  p.entry_offset = a.entry_offset;
  p.L_cap = a.L_cap;
  p.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  p.pos_q = a.pos_q;
  p.pos_base = a.pos_base;
  p.sel_idx = a.sel_idx;
  p.sel_cnt = a.sel_cnt;
  p.safe_pos = a.safe_pos;
  p.safe_fixed = a.safe_fixed;
  p.kv_c = reinterpret_cast<const __nv_bfloat16*>(a.kv_c);
  p.kmax = a.kmax;
  p.gamma_q = a.gamma_q;
  p.gamma_kv = a.gamma_kv;
  p.eps = a.eps;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.part_o = reinterpret_cast<__half*>(a.part_o);
  p.part_ml = a.part_ml;
  p.status = a.status;
  p.fused = (a.splits == 1 && !a.emit_partials) ? 1 : 0;
  p.sink = a.sink;
  p.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  for (int j = 0; j < 64; ++j) p.inv_freq[j] = a.inv_freq[j];
  const int rows = a.B * a.Q;
  const int cps = a.H > HC ? 2 : 1;  // CTAs per (row, split)
  if (rows > 65535 || a.splits * cps > 65535) return cudaErrorInvalidConfiguration;

  // Row-gather maps (one-row boxes) and 64-row box maps, 128-byte swizzle.
  CUtensorMap map_q, box_c, box_t;
  cudaError_t e = make_tmap_2d(&map_q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                               (uint64_t)rows * a.H, D, TN, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&box_c, a.kv_c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.B * a.N_cap,
                   D, TN, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&box_t, a.kv_tok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.B * a.L_cap,
                   D, TN, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;

  const size_t smem = 1024 + (size_t)C::kStages * C::kStageBytes + 2 * C::kPBytes +
                      C::kStages * sizeof(Meta) + 32 * 8 + 16 + 16 + 2 * D * sizeof(float);
  auto kern = mqa_heads_kernel<D, R>;
  const int variant = (D == 512 ? 0 : 3) + R / 32;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), 3 + variant, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(cps * a.splits, rows, 1);
  // The splits of each head group form one cluster and merge in-kernel, when
  // every cluster of the launch can be resident at once (otherwise the
  // clusters would run in waves: the separate merge kernel is faster).
  if (!p.fused && !a.emit_partials &&
      (int64_t)cps * rows <=
          clusters_resident(reinterpret_cast<const void*>(kern), variant, a.splits, smem)) {
    p.cluster_merge = 1;
    return launch_pdl(kern, grid, dim3(kThreads), smem, stream, a.splits, a.chained, map_q, box_c,
                      box_t, p);
  }
  e = launch_pdl(kern, grid, dim3(kThreads), smem, stream, 0, a.chained, map_q, box_c, box_t, p);
  if (e != cudaSuccess) return e;
  if (p.fused) return cudaSuccess;  // the attention kernel finished the rows
  if (a.emit_partials) return cudaSuccess;  // the caller merges the partials
  const unsigned nblk = (unsigned)(((int64_t)rows * a.H + 3) / 4);
  const size_t wsm = (size_t)4 * a.splits * sizeof(float);
  // Groups of 8 or 16 splits (the first group's loads go out with the
  // (max, sum) pairs).
  auto merge = a.splits <= 8 ? mqa_combine_kernel<D, R, 8> : mqa_combine_kernel<D, R, 16>;
  return launch_pdl(merge, dim3(nblk), dim3(128), wsm, stream, 0, 1, p, rows);
}

template <int D, int R>
cudaError_t launch_merge_impl(const MqaLaunch& a, cudaStream_t stream) {
  Params p{};
  p.Q = a.Q;
  p.H = a.H;
  p.R = a.rope_dim;
  p.splits = a.splits;
  p.pos_q = a.pos_q;
  p.pos_base = a.pos_base;
  p.part_o = reinterpret_cast<__half*>(a.part_o);
  p.part_ml = a.part_ml;
  p.status = a.status;
  p.sink = a.sink;
  p.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  for (int j = 0; j < 64; ++j) p.inv_freq[j] = a.inv_freq[j];
  const int rows = a.B * a.Q;
  const unsigned nblk = (unsigned)(((int64_t)rows * a.H + 3) / 4);
  const size_t wsm = (size_t)4 * a.splits * sizeof(float);
  auto merge = a.splits <= 8 ? mqa_combine_kernel<D, R, 8> : mqa_combine_kernel<D, R, 16>;
  return launch_pdl(merge, dim3(nblk), dim3(128), wsm, stream, 0, a.chained, p, rows);
}

}  // namespace

cudaError_t launch_mqa_merge(const MqaLaunch& a, cudaStream_t stream) {
  if (a.D == 512) {
    if (a.rope_dim == 64) return launch_merge_impl<512, 64>(a, stream);
    if (a.rope_dim == 32) return launch_merge_impl<512, 32>(a, stream);
    if (a.rope_dim == 0) return launch_merge_impl<512, 0>(a, stream);
  } else if (a.D == 128) {
    if (a.rope_dim == 32) return launch_merge_impl<128, 32>(a, stream);
    if (a.rope_dim == 0) return launch_merge_impl<128, 0>(a, stream);
  }
  return cudaErrorInvalidValue;
}

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
