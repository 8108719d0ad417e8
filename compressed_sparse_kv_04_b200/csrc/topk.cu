// Exact top-k of the indexer scores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), CSA step 2 keeps the k
// highest-scoring compressed blocks per query; "DeepSeek V4-Pro" (llm-arch-kb)
// sets k = 1024.  Tie rule (the build's): score descending, then index
// ascending; NaN below every number; -0 == +0.  Output: ascending indices,
// padded with -1, and the count min(k, n_vis).
//
// Design: a cluster of C CTAs (1024 threads each) per query row, C = 1..8.
//   Stage 1: CTA r holds its slice of the row in shared memory as
//     order-preserving 32-bit keys and selects the exact top-k of the slice
//     with a radix select: the digits start just below the bits common to
//     every key of the slice (min/max reduction), 11 bits per pass,
//     histograms with warp-aggregated shared atomics, and the passes stop as
//     soon as the threshold digit's bin is taken whole.  The selected
//     (key, index) pairs are compacted in index order.
//   Stage 2 (C > 1): every CTA pushes its list into the leader CTA's shared
//     memory (distributed shared memory stores) and arrives on the leader's
//     mbarrier; the leader selects the final top-k among the C*k candidates
//     with the same routine.  The global top-k of a row is contained in the
//     union of the slices' top-k under the same total order, so the result is
//     exact.  The leader's wait is bounded.
// No global atomics, no inter-CTA spin on memory; deterministic.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;  // 11-bit digits
constexpr int kMaxK = 1024;

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

struct Scratch {
  uint32_t hist[kBins];
  uint32_t warp_a[32];
  uint32_t warp_b[32];
  uint32_t bcast[4];
};

// Inclusive block-wide scan helpers (1024 threads).
CSA_DEV uint32_t block_excl_scan(uint32_t v, Scratch& sc, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sc.warp_a[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = sc.warp_a[lane], s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sc.warp_a[lane] = s - t;
    if (lane == 31) sc.bcast[3] = s;
  }
  __syncthreads();
  const uint32_t r = sc.warp_a[warp] + x - v;
  if (total) *total = sc.bcast[3];
  __syncthreads();
  return r;
}

CSA_DEV uint32_t block_min_max(uint32_t lo, uint32_t hi, Scratch& sc, uint32_t* out_hi) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sc.warp_a[warp] = lo;
    sc.warp_b[warp] = hi;
  }
  __syncthreads();
  if (warp == 0) {
    lo = sc.warp_a[lane];
    hi = sc.warp_b[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (lane == 0) {
      sc.bcast[0] = lo;
      sc.bcast[1] = hi;
    }
  }
  __syncthreads();
  lo = sc.bcast[0];
  *out_hi = sc.bcast[1];
  __syncthreads();
  return lo;
}

// Radix select over keys[0..n) (shared memory; `valid` filters slots).
// Result: prefix T and mask M such that the selection is every key with
// (key & M) > T, plus the first `need_eq` keys (in position order) with
// (key & M) == T.  |selection| = min(k, count of valid keys).
template <typename Valid>
CSA_DEV void radix_select(const uint32_t* keys, int n, int k, Valid valid, Scratch& sc,
                          uint32_t& T, uint32_t& M, uint32_t& need_eq) {
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int i = tid; i < n; i += kThreads)
    if (valid(i)) {
      lo = min(lo, keys[i]);
      hi = max(hi, keys[i]);
    }
  uint32_t gmax;
  const uint32_t gmin = block_min_max(lo, hi, sc, &gmax);
  uint32_t prefix = gmin & gmax, mask = 0u;
  uint32_t k_rem = (uint32_t)k;
  if (gmin == gmax) {  // every key equal (or a single key)
    T = gmin;
    M = 0xFFFFFFFFu;
    need_eq = k_rem;
    return;
  }
  int top = 31 - __clz(gmin ^ gmax);  // highest bit that differs
  mask = top == 31 ? 0u : (0xFFFFFFFFu << (top + 1));
  prefix &= mask;
  int shift = top + 1;
  while (shift > 0) {
    const int width = shift >= 11 ? 11 : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < kBins; b += kThreads) sc.hist[b] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += kThreads) {
      const int i = i0 + tid;
      bool act = false;
      uint32_t bin = 0;
      if (i < n && valid(i)) {
        const uint32_t key = keys[i];
        act = (key & mask) == prefix;
        bin = (key >> shift) & dmask;
      }
      const uint32_t am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t peers = __match_any_sync(am, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&sc.hist[bin], __popc(peers));
      }
    }
    __syncthreads();
    // Suffix sums over the digits: thread t owns digits 2t, 2t+1 (descending
    // digit = ascending thread from the top).
    const int nb = (int)dmask + 1;
    uint32_t c1 = 0, c0 = 0;  // counts of digits (nb-1-2t) and (nb-2-2t)
    const int d1 = nb - 1 - 2 * tid, d0 = nb - 2 - 2 * tid;
    if (d1 >= 0) c1 = sc.hist[d1];
    if (d0 >= 0) c0 = sc.hist[d0];
    uint32_t tot;
    const uint32_t above = block_excl_scan(c1 + c0, sc, &tot);  // keys in larger digits
    // Exactly one digit d satisfies above(d) < k_rem <= above(d) + count(d).
    if (d1 >= 0 && above < k_rem && above + c1 >= k_rem) {
      sc.bcast[0] = (uint32_t)d1;
      sc.bcast[1] = above;
      sc.bcast[2] = c1;
    }
    if (d0 >= 0 && above + c1 < k_rem && above + c1 + c0 >= k_rem) {
      sc.bcast[0] = (uint32_t)d0;
      sc.bcast[1] = above + c1;
      sc.bcast[2] = c0;
    }
    __syncthreads();
    const uint32_t d = sc.bcast[0], abv = sc.bcast[1], cnt_d = sc.bcast[2];
    __syncthreads();
    k_rem -= abv;
    prefix |= d << shift;
    mask |= dmask << shift;
    if (cnt_d == k_rem) break;  // the whole bin is taken: no need to resolve lower bits
  }
  T = prefix;
  M = mask;
  need_eq = k_rem;
}

// Index-ordered compaction of the selection; calls emit(position, out_slot).
template <typename Valid, typename Emit>
CSA_DEV uint32_t compact(const uint32_t* keys, int n, uint32_t T, uint32_t M, uint32_t need_eq,
                         Valid valid, Scratch& sc, Emit emit) {
  const int tid = threadIdx.x;
  const int E = (n + kThreads - 1) / kThreads;
  const int i0 = min(n, tid * E), i1 = min(n, i0 + E);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = i0; i < i1; ++i)
    if (valid(i)) {
      const uint32_t km = keys[i] & M;
      n_gt += km > T;
      n_eq += km == T;
    }
  const uint32_t eq_base = block_excl_scan(n_eq, sc, nullptr);
  const uint32_t take_eq = need_eq > eq_base ? min(need_eq - eq_base, n_eq) : 0u;
  uint32_t total;
  uint32_t o = block_excl_scan(n_gt + take_eq, sc, &total);
  uint32_t eq_seen = 0;
  for (int i = i0; i < i1; ++i) {
    if (!valid(i)) continue;
    const uint32_t km = keys[i] & M;
    bool take = km > T;
    if (km == T) take = eq_seen++ < take_eq;
    if (take) emit(i, o++);
  }
  return total;
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Scratch& sc = *reinterpret_cast<Scratch*>(smem_raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + sizeof(Scratch));
  uint32_t* cand_cnt = reinterpret_cast<uint32_t*>(bar + 1);         // [8]
  uint32_t* keys = cand_cnt + 8;                                      // slice
  uint32_t* cand_key = keys + p.slice;                                // [C][k] (leader)
  int32_t* cand_idx = reinterpret_cast<int32_t*>(cand_key + (p.C > 1 ? p.C * p.k : 0));

  const int row = blockIdx.y;
  const uint32_t r = cluster_ctarank();
  const int tid = threadIdx.x;
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
  if (p.C > 1) {
    if (tid == 0) {
      mbar_init(bar, p.C);
      fence_mbar_init();
    }
    cluster_sync();  // the leader's barrier exists before anyone arrives on it
  }
  const int64_t lo = (int64_t)r * p.slice;
  const int64_t hi = std::min<int64_t>(lo + p.slice, n);
  const int len = hi > lo ? (int)(hi - lo) : 0;
  const float* src = p.scores + (int64_t)row * p.N_cap + lo;
  for (int i = tid; i < len; i += kThreads) keys[i] = orderable(__ldg(src + i));
  __syncthreads();
  auto all_valid = [](int) { return true; };

  // Stage 1: the exact top-k of this slice.
  const int kl = std::min(p.k, len);
  uint32_t T = 0, M = 0xFFFFFFFFu, need_eq = (uint32_t)len;
  if (len > kl) radix_select(keys, len, kl, all_valid, sc, T, M, need_eq);
  if (p.C == 1) {
    compact(keys, len, T, M, need_eq, all_valid, sc,
            [&](int i, uint32_t o) { out[o] = (int32_t)(lo + i); });
    if (tid == 0) p.cnt[row] = p.k;
    return;
  }
  // Push the slice's list (index order) to the leader: slots r*k ...
  const uint32_t ck = mapa(smem_u32(cand_key), 0) + r * p.k * 4u;
  const uint32_t ci = mapa(smem_u32(cand_idx), 0) + r * p.k * 4u;
  const uint32_t total = compact(keys, len, T, M, need_eq, all_valid, sc, [&](int i, uint32_t o) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ck + o * 4u), "r"(keys[i]) : "memory");
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(ci + o * 4u), "r"((uint32_t)(lo + i))
                 : "memory");
  });
  if (tid == 0) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa(smem_u32(&cand_cnt[r]), 0)),
                 "r"(total)
                 : "memory");
  }
  __syncthreads();  // every store of this CTA precedes the release below
  if (tid == 0) mbar_arrive_remote(mapa(smem_u32(bar), 0));
  if (r != 0) return;

  // Stage 2 (leader): the top-k of the C lists.
  const bool ok = mbar_wait<true>(bar, 0, p.status);
  if (!__syncthreads_and(ok)) return;
  const int nc = p.C * p.k;
  auto cand_valid = [&](int j) { return (uint32_t)(j % p.k) < cand_cnt[j / p.k]; };
  radix_select(cand_key, nc, p.k, cand_valid, sc, T, M, need_eq);
  compact(cand_key, nc, T, M, need_eq, cand_valid, sc,
          [&](int j, uint32_t o) { out[o] = cand_idx[j]; });
  if (tid == 0) p.cnt[row] = p.k;
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
  const size_t smem = sizeof(Scratch) + 8 + 8 * 4 + (size_t)p.slice * 4 +
                      (C > 1 ? (size_t)C * a.k * 8 : 0);
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
