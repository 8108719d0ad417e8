// Exact top-k of the indexer scores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), CSA step 2 keeps the k
// highest-scoring compressed blocks per query; "DeepSeek V4-Pro" (llm-arch-kb)
// sets k = 1024.  Tie rule (the build's): score descending, then index
// ascending; NaN below every number; -0 == +0.  Output: ascending indices,
// padded with -1, and the count min(k, n_vis).
//
// Design: one thread-block cluster of C CTAs (C = 1..8) per query row.  CTA r
// keeps its slice of the row in shared memory as order-preserving 32-bit
// keys.  A radix select finds the exact k-th largest key over the whole row:
//   - every exchange is a "push": each CTA adds its contribution into the
//     shared memory of every CTA of the cluster (remote atomics), then
//     arrives on each CTA's mbarrier; every CTA waits for the C arrivals of
//     the round (bounded wait) and so holds the cluster-wide sum -- one
//     one-way hop per round, no cluster-wide barrier;
//   - round 0 exchanges min / max; the digits then start right below the
//     bits common to every key of the row, 11 bits per round, histograms
//     built with warp-aggregated shared atomics; the rounds stop as soon as
//     the threshold digit's bin is taken whole;
//   - a last round exchanges the per-CTA counts of keys above / equal to the
//     threshold, which gives every CTA its offset in the index-ordered
//     output (keys above the threshold, then the lowest-index equal keys).
// No global atomics; deterministic.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;  // 11-bit digits
constexpr int kMaxK = 1024;
constexpr int kMaxRounds = 8;  // min/max + at most 3 digit rounds + counts (+ slack)

struct Params {
  int Q, m, k, C;
  int64_t N_cap, slice;
  const float* scores;
  const int64_t* pos_q;
  int64_t pos_base;
  int32_t* idx;
  int32_t* cnt;
  int32_t* status;
};

CSA_DEV uint32_t orderable(float s) {
  if (isnan(s)) return 0u;
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7FFFFFFFu) == 0u) u = 0u;  // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  uint32_t hist[2][kBins];  // cluster-wide histograms (double-buffered by round)
  uint32_t local[kBins];    // this CTA's histogram of the round
  uint32_t gmin, gmax;      // cluster-wide min / max key
  uint32_t gt_before, eq_before;  // counts of lower-rank CTAs
  uint32_t warp_a[32], warp_b[32];
  uint32_t bcast[4];
  uint64_t bar[kMaxRounds];  // one mbarrier per round, C arrivals each
};

CSA_DEV void red_add_remote(uint32_t caddr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(caddr), "r"(v)
               : "memory");
}
CSA_DEV void red_min_remote(uint32_t caddr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.min.u32 [%0], %1;" ::"r"(caddr), "r"(v)
               : "memory");
}
CSA_DEV void red_max_remote(uint32_t caddr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.max.u32 [%0], %1;" ::"r"(caddr), "r"(v)
               : "memory");
}

// End of a round: every thread's remote contributions are issued; one thread
// arrives on round `rd`'s barrier of every CTA, then everyone waits for the C
// arrivals of the round.  Returns false when the (bounded) wait gave up.
CSA_DEV bool round_sync(Shared& sh, int rd, int C, int32_t* status) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t a = smem_u32(&sh.bar[rd]);
    for (int c = 0; c < C; ++c) mbar_arrive_remote(mapa(a, c));
  }
  const bool ok = mbar_wait<true>(&sh.bar[rd], 0, status);
  return __syncthreads_and(ok) != 0;
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Shared& sh = *reinterpret_cast<Shared*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(Shared));

  const int row = blockIdx.y;
  const int C = p.C;
  const uint32_t r = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t pos = p.pos_q ? p.pos_q[row] : p.pos_base + row % p.Q;
  int64_t n = pos < 0 ? 0 : (pos + 1) / p.m;
  if (n > p.N_cap) {
    n = p.N_cap;
    if (r == 0 && tid == 0) report(p.status, CSA_ERR_CAPACITY);
  }
  int32_t* out = p.idx + (int64_t)row * p.k;
  if (n <= p.k) {  // every visible entry is kept (uniform over the cluster)
    if (r == 0) {
      for (int j = tid; j < p.k; j += kThreads) out[j] = j < n ? j : -1;
      if (tid == 0) p.cnt[row] = (int32_t)n;
    }
    return;
  }
  // Initial state, visible cluster-wide before any remote update.
  for (int b = tid; b < kBins; b += kThreads) sh.hist[0][b] = sh.hist[1][b] = 0;
  if (tid == 0) {
    sh.gmin = 0xFFFFFFFFu;
    sh.gmax = 0u;
    sh.gt_before = sh.eq_before = 0u;
    for (int rd = 0; rd < kMaxRounds; ++rd) mbar_init(&sh.bar[rd], C);
    fence_mbar_init();
  }
  cluster_sync();

  const int64_t lo = (int64_t)r * p.slice;
  const int64_t hi = lo + p.slice < n ? lo + p.slice : n;
  const int len = hi > lo ? (int)(hi - lo) : 0;
  const float* src = p.scores + (int64_t)row * p.N_cap + lo;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll 4
  for (int i = tid; i < len; i += kThreads) {
    const uint32_t key = orderable(__ldg(src + i));
    keys[i] = key;
    kmin = min(kmin, key);
    kmax = max(kmax, key);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  // Round 0: min / max into every CTA.
  if (lane == 0 && len > 0) {
    const uint32_t amin = smem_u32(&sh.gmin), amax = smem_u32(&sh.gmax);
    for (int c = 0; c < C; ++c) {
      red_min_remote(mapa(amin, c), kmin);
      red_max_remote(mapa(amax, c), kmax);
    }
  }
  int rd = 0;
  if (!round_sync(sh, rd++, C, p.status)) return;
  const uint32_t gmin = sh.gmin, gmax = sh.gmax;

  // Radix rounds below the common prefix.
  uint32_t prefix, mask;
  uint32_t k_rem = (uint32_t)p.k;
  if (gmin == gmax) {
    prefix = gmin;
    mask = 0xFFFFFFFFu;
  } else {
    const int top = 31 - __clz(gmin ^ gmax);
    mask = top == 31 ? 0u : (0xFFFFFFFFu << (top + 1));
    prefix = gmin & mask;
    int shift = top + 1;
    int buf = 0;
    while (shift > 0) {
      const int width = shift >= 11 ? 11 : shift;
      shift -= width;
      const uint32_t dmask = (1u << width) - 1u;
      for (int b = tid; b < kBins; b += kThreads) sh.local[b] = 0;
      __syncthreads();
      for (int i0 = 0; i0 < len; i0 += kThreads) {
        const int i = i0 + tid;
        bool act = false;
        uint32_t bin = 0;
        if (i < len) {
          const uint32_t key = keys[i];
          act = (key & mask) == prefix;
          bin = (key >> shift) & dmask;
        }
        const uint32_t am = __ballot_sync(0xffffffffu, act);
        if (act) {
          const uint32_t peers = __match_any_sync(am, bin);
          if (lane == __ffs(peers) - 1) atomicAdd(&sh.local[bin], __popc(peers));
        }
      }
      __syncthreads();
      // Clear the other buffer before arriving (the next round's adds only
      // come from CTAs that have seen this round's arrival of this CTA).
      for (int b = tid; b < kBins; b += kThreads) sh.hist[buf ^ 1][b] = 0;
      const uint32_t base = smem_u32(&sh.hist[buf][0]);
      for (int b = tid; b <= (int)dmask; b += kThreads) {
        const uint32_t v = sh.local[b];
        if (v)
          for (int c = 0; c < C; ++c) red_add_remote(mapa(base + 4u * b, c), v);
      }
      if (!round_sync(sh, rd++, C, p.status)) return;
      // Warp 0 finds the digit d with above(d) < k_rem <= above(d) + count(d),
      // scanning from the top digit down (64 digits per lane).
      if (warp == 0) {
        const int nb = (int)dmask + 1;
        const int per = (nb + 31) / 32;
        const int d_hi = nb - 1 - lane * per;  // this lane's digits: d_hi down to d_hi-per+1
        uint32_t sum = 0;
        for (int j = 0; j < per; ++j) {
          const int d = d_hi - j;
          if (d >= 0) sum += sh.hist[buf][d];
        }
        uint32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        uint32_t above = incl - sum;  // keys in digits owned by lower lanes (larger digits)
        if (above < k_rem && incl >= k_rem) {
          for (int j = 0; j < per; ++j) {
            const int d = d_hi - j;
            if (d < 0) break;
            const uint32_t cd = sh.hist[buf][d];
            if (above + cd >= k_rem) {
              sh.bcast[0] = (uint32_t)d;
              sh.bcast[1] = above;
              sh.bcast[2] = cd;
              break;
            }
            above += cd;
          }
        }
      }
      __syncthreads();
      const uint32_t d = sh.bcast[0], abv = sh.bcast[1], cnt_d = sh.bcast[2];
      k_rem -= abv;
      prefix |= d << shift;
      mask |= dmask << shift;
      buf ^= 1;
      __syncthreads();
      if (cnt_d == k_rem) break;  // the whole bin is taken
    }
  }
  const uint32_t T = prefix, M = mask, need_eq = k_rem;

  // Index-ordered output.  Warp w owns the slice elements
  // [w*chunk, (w+1)*chunk) (chunk a multiple of 32); lane l reads element
  // j*32 + l of the chunk, so a ballot gives each element its rank.
  const int chunk = (((len + 31) / 32) + 31) & ~31;
  const int w0 = min(len, warp * chunk), w1 = min(len, w0 + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = w0 + lane; i < w1; i += 32) {
    const uint32_t km = keys[i] & M;
    n_gt += km > T;
    n_eq += km == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
    n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
  }
  if (lane == 0) {
    sh.warp_a[warp] = n_gt;
    sh.warp_b[warp] = n_eq;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t a = sh.warp_a[lane], b = sh.warp_b[lane];
    uint32_t sa = a, sb = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ya = __shfl_up_sync(0xffffffffu, sa, o);
      const uint32_t yb = __shfl_up_sync(0xffffffffu, sb, o);
      if (lane >= o) {
        sa += ya;
        sb += yb;
      }
    }
    sh.warp_a[lane] = sa - a;
    sh.warp_b[lane] = sb - b;
    if (lane == 31) {
      sh.bcast[0] = sa;
      sh.bcast[1] = sb;
    }
  }
  __syncthreads();
  // Last round: this CTA's totals into every higher-rank CTA.
  if (tid == 0) {
    const uint32_t ag = smem_u32(&sh.gt_before), ae = smem_u32(&sh.eq_before);
    for (int c = (int)r + 1; c < C; ++c) {
      red_add_remote(mapa(ag, c), sh.bcast[0]);
      red_add_remote(mapa(ae, c), sh.bcast[1]);
    }
  }
  if (!round_sync(sh, rd++, C, p.status)) return;
  uint32_t gt_run = sh.gt_before + sh.warp_a[warp];
  uint32_t eq_run = sh.eq_before + sh.warp_b[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int i = w0 + lane; i - lane < w1; i += 32) {
    const uint32_t km = i < w1 ? keys[i] & M : 0u;
    const bool gt = i < w1 && km > T;
    const bool eq = i < w1 && km == T;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const uint32_t eq_rank = eq_run + __popc(be & lt);
    if (gt || (eq && eq_rank < need_eq)) {
      const uint32_t o = gt_run + __popc(bg & lt) + min(need_eq, eq_rank);
      if (o < (uint32_t)p.k) out[o] = (int32_t)(lo + i);
    }
    gt_run += __popc(bg);
    eq_run += __popc(be);
  }
  if (r == 0 && tid == 0) p.cnt[row] = p.k;
}

}  // namespace

cudaError_t launch_topk(const TopkLaunch& a, cudaStream_t stream) {
  if (a.rows < 1) return cudaSuccess;
  if (a.rows > 65535 || a.k > kMaxK) return cudaErrorInvalidConfiguration;
  const int sms = device_sm_count();
  const int need = (int)((a.N_cap + 32767) / 32768);
  if (need > 8) return cudaErrorInvalidValue;
  int C = 1;
  while (C < need) C <<= 1;
  if (a.rows < sms) {  // spread small batches: slices of at least 4096 scores
    const int fill = std::max(1, sms / a.rows);
    while (C * 2 <= 8 && C * 2 <= fill && a.N_cap / (C * 2) >= 4096) C *= 2;
  }
  Params p{};
  p.Q = a.Q;
  p.m = a.m;
  p.k = a.k;
  p.C = C;
  p.N_cap = a.N_cap;
  p.slice = (a.N_cap + C - 1) / C;
  p.scores = a.scores;
  p.pos_q = a.pos_q;
  p.pos_base = a.pos_base;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.status = a.status;
  const size_t smem = sizeof(Shared) + (size_t)p.slice * 4;
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(topk_kernel), 2, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(C, a.rows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, topk_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa
