// Exact top-k of the indexer scores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), CSA step 2 keeps the k
// highest-scoring compressed blocks per query; "DeepSeek V4-Pro" (llm-arch-kb)
// sets k = 1024.  Tie rule (the build's): score descending, then index
// ascending; NaN below every number; -0 == +0.  Output: ascending indices,
// padded with -1, and the count min(k, n_vis).
//
// Design: one thread-block cluster of C CTAs (1024 threads each) per query
// row; CTA r keeps its slice of the row in shared memory as order-preserving
// 32-bit keys.  Four 8-bit radix passes find the exact k-th largest key T:
// each CTA histograms its slice (shared atomics), the C histograms are summed
// through distributed shared memory, and every CTA derives the same digit.
// The output is then compacted in index order: keys > T, plus the
// lowest-index keys == T up to k, with block and cluster exclusive scans
// giving each thread its output offset.  The row is read from global memory
// once; there are no global atomics and no inter-CTA spin waits (cluster
// barriers only), so the result is deterministic.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 1024;

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

CSA_DEV uint32_t ld_cluster_u32(uint32_t caddr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(caddr) : "memory");
  return v;
}

// Exclusive scan of one value per thread over the CTA; returns the exclusive
// prefix and writes the CTA total to *total.
CSA_DEV uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = warp_tot[lane];
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s - t;  // exclusive prefix of warp totals
    if (lane == 31) *total = s;
  }
  __syncthreads();
  uint32_t r = warp_tot[warp] + x - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const Params p) {
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* hist = sm;             // 256
  uint32_t* red = hist + 256;      // 256
  uint32_t* warp_tot = red + 256;  // 32
  uint32_t* misc = warp_tot + 32;  // 8: [0]=digit [1]=above [2]=eq_total [3]=sel_total [4]=scan tot
  uint32_t* keys = misc + 8;       // slice

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
  const int64_t lo = (int64_t)r * p.slice;
  const int64_t hi = std::min<int64_t>(lo + p.slice, n);
  const int len = hi > lo ? (int)(hi - lo) : 0;
  const float* src = p.scores + (int64_t)row * p.N_cap + lo;
  for (int i = tid; i < len; i += kThreads) keys[i] = orderable(__ldg(src + i));

  uint32_t prefix = 0, mask = 0;
  uint32_t k_rem = (uint32_t)p.k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0;
    __syncthreads();
    for (int i = tid; i < len; i += kThreads) {
      uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    cluster_sync();
    if (tid < 256) {
      uint32_t tot = 0;
      const uint32_t a = smem_u32(&hist[tid]);
      for (int c = 0; c < p.C; ++c) tot += ld_cluster_u32(mapa(a, c));
      red[tid] = tot;
    }
    cluster_sync();  // remote reads done before the next pass clears hist
    if (tid < 32) {
      // Suffix sums over digits 255..0: lane l owns digits 8l .. 8l+7.
      uint32_t v[8], s = 0;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        v[j] = red[tid * 8 + j];
        s += v[j];
      }
      // Exclusive suffix over lanes (lanes above hold larger digits).
      uint32_t above = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, above, o);
        if (tid + o < 32) above += y;
      }
      above -= s;  // count of keys in digits owned by higher lanes
      // The digit d with suffix(d+1) < k_rem <= suffix(d).
      uint32_t acc = above;
      int found = -1;
      uint32_t found_above = 0;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        if (found < 0 && acc < k_rem && acc + v[j] >= k_rem) {
          found = tid * 8 + j;
          found_above = acc;
        }
        acc += v[j];
      }
      if (found >= 0) {
        misc[0] = (uint32_t)found;
        misc[1] = found_above;
      }
    }
    __syncthreads();
    const uint32_t d = misc[0];
    k_rem -= misc[1];
    prefix |= d << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;     // the k-th largest key
  const uint32_t need_eq = k_rem;  // keys == T to keep, lowest index first

  // Index-ordered compaction: thread t owns slice elements [t*E, t*E+E).
  const int E = (len + kThreads - 1) / kThreads;
  const int i0 = std::min(len, tid * E), i1 = std::min(len, i0 + E);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = keys[i];
    n_gt += key > T;
    n_eq += key == T;
  }
  uint32_t eq_scan = block_exclusive_scan(n_eq, warp_tot, &misc[2]);
  cluster_sync();
  uint32_t eq_before = 0;
  {
    const uint32_t a = smem_u32(&misc[2]);
    for (uint32_t c = 0; c < r; ++c) eq_before += ld_cluster_u32(mapa(a, c));
  }
  const uint32_t eq_base = eq_before + eq_scan;
  const uint32_t take_eq =
      need_eq > eq_base ? std::min<uint32_t>(need_eq - eq_base, n_eq) : 0u;
  uint32_t sel_scan = block_exclusive_scan(n_gt + take_eq, warp_tot, &misc[3]);
  cluster_sync();
  uint32_t out_before = 0;
  {
    const uint32_t a = smem_u32(&misc[3]);
    for (uint32_t c = 0; c < r; ++c) out_before += ld_cluster_u32(mapa(a, c));
  }
  uint32_t o = out_before + sel_scan;
  uint32_t eq_seen = 0;
  for (int i = i0; i < i1; ++i) {
    uint32_t key = keys[i];
    bool take = key > T;
    if (key == T) {
      take = eq_seen < take_eq;
      ++eq_seen;
    }
    if (take) {
      if (o < (uint32_t)p.k) out[o] = (int32_t)(lo + i);
      ++o;
    }
  }
  if (r == 0 && tid == 0) p.cnt[row] = p.k;
  cluster_sync();  // keep shared memory alive until every remote read is done
}

}  // namespace

cudaError_t launch_topk(const TopkLaunch& a, cudaStream_t stream) {
  if (a.rows < 1) return cudaSuccess;
  if (a.rows > 65535) return cudaErrorInvalidConfiguration;
  const int sms = device_sm_count();
  int need = (int)((a.N_cap + 32767) / 32768);
  if (need > 8) return cudaErrorInvalidValue;
  int C = 1;
  while (C < need) C <<= 1;
  if (a.rows < sms) {
    int fill = std::max(1, sms / a.rows);
    while (C * 2 <= 8 && C * 2 <= fill && (a.N_cap + C * 2 - 1) / (C * 2) >= 1024) C *= 2;
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
  size_t smem = (256 + 256 + 32 + 8) * 4 + (size_t)p.slice * 4;
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
