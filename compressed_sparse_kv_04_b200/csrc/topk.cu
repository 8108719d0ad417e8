// Exact top-k of the indexer scores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), CSA step 2 keeps the k
// highest-scoring compressed blocks per query; "DeepSeek V4-Pro" (llm-arch-kb)
// sets k = 1024.  Tie rule (chosen here): score descending, then index
// ascending; NaN below every number; -0 == +0.  Output: ascending indices,
// padded with -1, and the count min(k, n_vis).
//
// Many rows, or short ones, that fit in one CTA's shared memory (up to ~47K
// scores) are ranked by topk_row_kernel, one CTA per row; the other rows by
// topk_kernel: one thread-block cluster of C CTAs (C = 1..16) per query row.  CTA r
// keeps its slice of the row in shared memory as order-preserving 32-bit
// keys.  A radix select finds the exact k-th largest key over the whole row:
//   - every exchange is a push of plain 16-byte stores: each CTA writes its
//     contribution into its own slot of every CTA's receive buffer, then one
//     hardware cluster barrier (arrive.release / wait.acquire) makes all
//     slots visible; each CTA sums the C slots itself.  (Remote atomics and
//     mbarrier hops cost several times more per round on this part.)
//   - round 0 exchanges min / max; the digits then start right below the
//     bits common to every key of the row, kDigitBits per round; the rounds
//     stop as soon as the threshold digit's bin is taken whole;
//   - a last round exchanges the per-CTA counts of keys above / equal to the
//     threshold, which gives every CTA its offset in the index-ordered
//     output (keys above the threshold, then the lowest-index equal keys).
// Every decision that steers the control flow (early exit, number of
// rounds) is computed from cluster-wide sums that all CTAs of the cluster
// hold identically, so all of them reach every cluster barrier.
// No global atomics; deterministic.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 1024;
constexpr int kDigitBits = 8;  // radix digit width (256 bins)
constexpr int kMaxK = 2048;
constexpr int kMaxC = 16;      // CTAs per cluster (16 needs the non-portable size)

struct Params {
  int Q, m, k, C;
  int64_t N_cap, slice;
  int64_t entry_offset;  // the scores are of entries entry_offset .. of the sequence
  const float* scores;
  const int64_t* pos_q;
  int64_t pos_base;
  int32_t* idx;
  int32_t* cnt;
  int32_t* status;
  uint32_t* hist;     // topk_hist_kernel: [rows, kScoreHistBins]
  int32_t* path;      // [rows] or null
  uint32_t hist_off;  // topk_hist_kernel: byte offset of HistShared
};

CSA_DEV uint32_t orderable(float s) { return score_key(s); }

template <int kBins>
struct Shared {
  uint32_t recv[2][kMaxC][kBins];  // per-source histograms, by round parity
  uint32_t local[2][kBins];        // this CTA's histogram, by round parity
  uint32_t mm[kMaxC][2];           // per-source (min, max) key
  uint32_t cn[kMaxC][2];           // per-source (above, equal) counts
  uint32_t warp_a[32], warp_b[32];
  uint32_t bcast[4];
};

// The aligned barriers below need converged warps: each helper reconverges
// its warp first.
CSA_DEV void cluster_arrive() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
CSA_DEV void cluster_wait() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
CSA_DEV void cta_sync() {
  __syncwarp();
  __syncthreads();
}
CSA_DEV void st_remote_v2(uint32_t caddr, uint32_t a, uint32_t b) {
  asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(caddr), "r"(a), "r"(b)
               : "memory");
}
CSA_DEV void st_remote_v4(uint32_t caddr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// The radix select over the cluster and the index-ordered emission.  The
// slice is keys[0..len) at row positions lo.. (keys follow the Shared block
// in dynamic shared memory); the selection goes to out[0..k).
// (Out of line: the exchange rounds measured faster that way.)
template <int kBits, bool kAggregate>
__device__ __noinline__ void cluster_select(uint8_t* smem_raw, int C, uint32_t r, int k, int len,
                                            int64_t lo, int32_t* out) {
  constexpr int kBins = 1 << kBits;
  using S = Shared<kBins>;
  S& sh = *reinterpret_cast<S*>(smem_raw);
  const uint32_t* keys = reinterpret_cast<const uint32_t*>(smem_raw + sizeof(S));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  cluster_arrive();  // paired with the wait before the first remote store

  for (int b = tid; b < kBins; b += kThreads) sh.local[0][b] = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int i = tid; i < len; i += kThreads) {  // the keys this thread wrote
    kmin = min(kmin, keys[i]);
    kmax = max(kmax, keys[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    sh.warp_a[warp] = kmin;
    sh.warp_b[warp] = kmax;
  }
  cta_sync();
  cluster_wait();  // every CTA of the cluster is running
  // Round 0: (min, max) of this CTA into slot r of every CTA.
  if (warp == 0) {
    kmin = sh.warp_a[lane];
    kmax = sh.warp_b[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane < C) st_remote_v2(mapa(smem_u32(&sh.mm[r][0]), lane), kmin, kmax);
  }
  cluster_arrive();
  cluster_wait();
  uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
  for (int c = 0; c < C; ++c) {
    gmin = min(gmin, sh.mm[c][0]);
    gmax = max(gmax, sh.mm[c][1]);
  }

  // Radix rounds below the common prefix.
  uint32_t prefix, mask;
  uint32_t k_rem = (uint32_t)k;
  if (gmin == gmax) {
    prefix = gmin;
    mask = 0xFFFFFFFFu;
  } else {
    const int top = 31 - __clz(gmin ^ gmax);
    mask = top == 31 ? 0u : (0xFFFFFFFFu << (top + 1));
    prefix = gmin & mask;
    int shift = top + 1;
    int par = 0;
    while (shift > 0) {
      const int width = shift >= kBits ? kBits : shift;
      shift -= width;
      const uint32_t dmask = (1u << width) - 1u;
      uint32_t* loc = sh.local[par];
      for (int i = tid; i < len; i += kThreads) {
        const uint32_t key = keys[i];
        const bool act = (key & mask) == prefix;
        const uint32_t bin = (key >> shift) & dmask;
        if (kAggregate) {
          const uint32_t am = __ballot_sync(__activemask(), act);
          if (act) {
            const uint32_t peers = __match_any_sync(am, bin);
            if (lane == __ffs(peers) - 1) atomicAdd(&loc[bin], __popc(peers));
          }
        } else if (act) {
          atomicAdd(&loc[bin], 1u);
        }
      }
      cta_sync();
      // Push: this CTA's histogram into slot r of every CTA (16-byte stores);
      // the other threads clear next round's local histogram.
      constexpr int kVec = kBins / 4;
      for (int t = tid; t < C * kVec; t += kThreads) {
        const int c = t / kVec, j = t % kVec;
        const uint4 v = reinterpret_cast<const uint4*>(loc)[j];
        st_remote_v4(mapa(smem_u32(&sh.recv[par][r][4 * j]), c), v);
      }
      for (int b = tid; b < kBins; b += kThreads) sh.local[par ^ 1][b] = 0;
      cluster_arrive();
      cluster_wait();
      // Thread t < nb owns digit d = nb-1-t: its cluster-wide count, then a
      // scan over t gives the keys in digits >= d; the one thread with
      // above(d) < k_rem <= above(d) + count(d) publishes d.
      const int nb = (int)dmask + 1;
      uint32_t cnt_t = 0;
      if (tid < nb)
        for (int c = 0; c < C; ++c) cnt_t += sh.recv[par][c][nb - 1 - tid];
      uint32_t incl = cnt_t;
      if (warp < kBins / 32) {
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) sh.warp_a[warp] = incl;
      }
      cta_sync();
      if (tid < nb) {
        for (int w2 = 0; w2 < warp; ++w2) incl += sh.warp_a[w2];
        const uint32_t above = incl - cnt_t;
        if (above < k_rem && incl >= k_rem) {
          sh.bcast[0] = (uint32_t)(nb - 1 - tid);
          sh.bcast[1] = above;
          sh.bcast[2] = cnt_t;
        }
      }
      cta_sync();
      const uint32_t d = sh.bcast[0], abv = sh.bcast[1], cnt_d = sh.bcast[2];
      k_rem -= abv;
      prefix |= d << shift;
      mask |= dmask << shift;
      par ^= 1;
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
  cta_sync();  // bcast / warp slots of the last round are read
  if (lane == 0) {
    sh.warp_a[warp] = n_gt;
    sh.warp_b[warp] = n_eq;
  }
  cta_sync();
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
    // Last round: this CTA's totals into slot r of every higher-rank CTA.
    const uint32_t ga = __shfl_sync(0xffffffffu, sa, 31), gb = __shfl_sync(0xffffffffu, sb, 31);
    if (lane > (int)r && lane < C) st_remote_v2(mapa(smem_u32(&sh.cn[r][0]), lane), ga, gb);
  }
  cluster_arrive();
  cluster_wait();
  uint32_t gt_run = sh.warp_a[warp], eq_run = sh.warp_b[warp];
  for (int c = 0; c < (int)r; ++c) {
    gt_run += sh.cn[c][0];
    eq_run += sh.cn[c][1];
  }
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
      if (o < (uint32_t)k) out[o] = (int32_t)(lo + i);
    }
    gt_run += __popc(bg);
    eq_run += __popc(be);
  }
}

template <int kBits, bool kAggregate>
__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const Params p) {
  constexpr int kBins = 1 << kBits;
  using S = Shared<kBins>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(S));

  const int row = blockIdx.y;
  const int C = p.C;
  const uint32_t r = cluster_ctarank();
  const int tid = threadIdx.x;
  pdl_trigger();
  const int64_t pos = p.pos_q ? p.pos_q[row] : p.pos_base + row % p.Q;
  const int64_t lo = (int64_t)r * p.slice;
  pdl_wait();  // the scores come from the indexer kernel
  // The slice's scores are loaded before the visible count is known (the
  // row holds N_cap scores, so every address is in bounds).
  const int cap = (int)(p.N_cap - lo < p.slice ? (p.N_cap - lo > 0 ? p.N_cap - lo : 0) : p.slice);
  const float* src = p.scores + (int64_t)row * p.N_cap + lo;
#pragma unroll 8
  for (int i = tid; i < cap; i += kThreads) keys[i] = orderable(__ldg(src + i));
  int64_t n = pos < 0 ? 0 : (pos + 1) / p.m - p.entry_offset;
  if (n < 0) n = 0;
  if (n > p.N_cap) {
    n = p.N_cap;
    if (r == 0 && tid == 0) report(p.status, CSA_ERR_CAPACITY);
  }
  int32_t* out = p.idx + (int64_t)row * p.k;
  if (n <= p.k) {  // every visible entry is kept (the whole cluster returns)
    if (r == 0) {
      for (int j = tid; j < p.k; j += kThreads) out[j] = j < n ? j : -1;
      if (tid == 0) p.cnt[row] = (int32_t)n;
    }
    return;
  }
  const int len = (int)(n - lo < cap ? (n - lo > 0 ? n - lo : 0) : cap);
  cluster_select<kBits, kAggregate>(smem_raw, C, r, p.k, len, lo, out);
  if (r == 0 && tid == 0) p.cnt[row] = p.k;
}


// One CTA per query row, for rows whose visible scores fit in shared memory
// (decode at 128K context, every prefill row).  The same radix select as
// above with no cluster exchange: 1024 threads hold the row as keys in shared
// memory, a block-wide (min, max) gives the common prefix, and each round
// histograms the next kRowBits bits of the keys that still match the prefix
// (shared-memory atomics) and finds the threshold digit with a block scan.
// Rounds stop once the threshold bin is taken whole; the index-ordered
// output is the same ballot-ranked pass.  Only __syncthreads barriers.
constexpr int kRowBits = 12;

struct RowShared {
  uint32_t hist[1 << kRowBits];
  uint32_t warp_a[32], warp_b[32];
  uint32_t scan[33];
  uint32_t bcast[4];
};
// The keys follow RowShared in dynamic shared memory, on a 16-byte boundary
// (they are written with 16-byte stores).
constexpr size_t kRowKeysOff = (sizeof(RowShared) + 15) / 16 * 16;

// Exclusive prefix over the block of per-thread values (1024 threads, one
// value each); warp_tot is 33 words of shared scratch.
CSA_DEV uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  cta_sync();
  if (warp == 0) {
    const uint32_t t = warp_tot[lane];
    uint32_t x = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    warp_tot[lane] = x - t;  // exclusive over warps
  }
  cta_sync();
  return warp_tot[warp] + incl - v;
}

// Radix rounds over keys[0..n): the keys whose bits under `mask` equal
// `prefix` take part, and the digits start at bit `shift`, kRowBits per
// round, until the threshold digit's bin is taken whole.  sh.hist must be
// zero on entry (it is zero again on return).  On return prefix / mask are
// the threshold key T and the mask M of its decided bits; the selection is
// every key above T (under M) and the first need_eq keys equal to it, where
// need_eq is the return value and k_rem the number of keys still to choose
// among those taking part.  All 1024 threads call it.
template <int kBits = kRowBits>
CSA_DEV uint32_t row_rounds(const uint32_t* keys, int n, uint32_t k_rem, RowShared& sh,
                            uint32_t& prefix, uint32_t& mask, int shift) {
  static_assert(kBits >= 10 && kBits <= kRowBits, "1 to 4 bins per thread");
  constexpr int kBins = 1 << kBits;
  constexpr int kPer = kBins / kThreads;  // bins per thread in the digit scan
  const int tid = threadIdx.x;
  while (shift > 0) {
    const int width = shift >= kBits ? kBits : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
#pragma unroll 4
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & dmask], 1u);
    }
    cta_sync();
    // Thread t owns digits nb-1-t*kPer down to nb-(t+1)*kPer (descending),
    // so an exclusive scan over t counts the keys in higher digits.
    const int nb = (int)dmask + 1;
    uint32_t c[kPer];
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int d = nb - 1 - (tid * kPer + j);
      c[j] = d >= 0 ? sh.hist[d] : 0u;
      local += c[j];
    }
    uint32_t above = block_excl_scan(local, sh.scan);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int d = nb - 1 - (tid * kPer + j);
      if (d >= 0 && above < k_rem && above + c[j] >= k_rem) {
        sh.bcast[0] = (uint32_t)d;
        sh.bcast[1] = above;
        sh.bcast[2] = c[j];
      }
      above += c[j];
    }
    for (int b = tid; b < kBins; b += kThreads) sh.hist[b] = 0;
    cta_sync();
    const uint32_t d = sh.bcast[0], abv = sh.bcast[1], cnt_d = sh.bcast[2];
    cta_sync();  // bcast is read before the next round can rewrite it
    k_rem -= abv;
    prefix |= d << shift;
    mask |= dmask << shift;
    if (cnt_d == k_rem) break;  // the whole bin is taken
  }
  return k_rem;
}

// Index-ordered output of a selection (threshold T under mask M, need_eq
// equal keys): calls emit(o, i) for each selected position i of keys[0..n)
// with its output slot o < k, given gt_base / eq_base keys above / equal to
// T that precede keys[0] in index order.  Warp w owns positions
// [w*chunk, (w+1)*chunk) (chunk a multiple of 32); lane l takes element
// j*32 + l of the chunk, so a ballot ranks it.  All 1024 threads call it.
// Sums each warp's (a, b) over its lanes and returns, to every thread of
// the warp, the sums of the warps before it (block exclusive prefix in warp
// order).  All 1024 threads call it.
CSA_DEV void warp_excl_prefix(uint32_t a, uint32_t b, RowShared& sh, uint32_t& pa, uint32_t& pb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (lane == 0) {
    sh.warp_a[warp] = a;
    sh.warp_b[warp] = b;
  }
  cta_sync();
  if (warp == 0) {
    const uint32_t x = sh.warp_a[lane], y = sh.warp_b[lane];
    uint32_t sa = x, sb = y;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ya = __shfl_up_sync(0xffffffffu, sa, o);
      const uint32_t yb = __shfl_up_sync(0xffffffffu, sb, o);
      if (lane >= o) {
        sa += ya;
        sb += yb;
      }
    }
    sh.warp_a[lane] = sa - x;
    sh.warp_b[lane] = sb - y;
  }
  cta_sync();
  pa = sh.warp_a[warp];
  pb = sh.warp_b[warp];
}

template <typename Emit>
CSA_DEV void ordered_emit(const uint32_t* keys, int n, int k, uint32_t T, uint32_t M,
                          uint32_t need_eq, uint32_t gt_base, uint32_t eq_base, RowShared& sh,
                          Emit emit) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = (((n + 31) / 32) + 31) & ~31;
  const int w0 = min(n, warp * chunk), w1 = min(n, w0 + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int i = w0 + lane; i < w1; i += 32) {
    const uint32_t km = keys[i] & M;
    n_gt += km > T;
    n_eq += km == T;
  }
  uint32_t gt_run, eq_run;
  warp_excl_prefix(n_gt, n_eq, sh, gt_run, eq_run);
  gt_run += gt_base;
  eq_run += eq_base;
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
      if (o < (uint32_t)k) emit(o, i);
    }
    gt_run += __popc(bg);
    eq_run += __popc(be);
  }
}

// Keys above T and equal to T (under mask M) among a warp's listed
// positions, summed over the warp (every lane gets the sums).
CSA_DEV void list_counts(const uint32_t* keys, const uint16_t* list, int n_list, uint32_t T,
                         uint32_t M, uint32_t& gt, uint32_t& eq) {
  const int lane = threadIdx.x & 31;
  gt = 0;
  eq = 0;
  for (int e = lane; e < n_list; e += 32) {
    const uint32_t km = keys[list[e]] & M;
    gt += km > T;
    eq += km == T;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
}

// The same output as ordered_emit when every key the selection can take
// is listed: warp w passes its list of n_list positions (ascending, and all
// of them below those of warp w + 1), so only the listed keys are read.
// gt_run / eq_run: keys above / equal to T before the warp's first position
// in index order (the slice's base plus the warps before it).
template <typename Emit>
CSA_DEV void list_emit(const uint32_t* keys, const uint16_t* list, int n_list, int k, uint32_t T,
                       uint32_t M, uint32_t need_eq, uint32_t gt_run, uint32_t eq_run,
                       Emit emit) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  for (int e = lane; e - lane < n_list; e += 32) {
    const int i = e < n_list ? (int)list[e] : 0;
    const uint32_t km = e < n_list ? keys[i] & M : 0u;
    const bool gt = e < n_list && km > T;
    const bool eq = e < n_list && km == T;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const uint32_t eq_rank = eq_run + __popc(be & lt);
    if (gt || (eq && eq_rank < need_eq)) {
      const uint32_t o = gt_run + __popc(bg & lt) + min(need_eq, eq_rank);
      if (o < (uint32_t)k) emit(o, i);
    }
    gt_run += __popc(bg);
    eq_run += __popc(be);
  }
}

// Selects the k largest of keys[0..n) (n > k; order-preserving keys in
// shared memory, written by this CTA) under (key descending, position
// ascending) and calls emit(o, i) once for each output slot o < k with the
// selected position i, slots in ascending order of i.  kmin / kmax: this
// thread's min and max over the keys it wrote.  All 1024 threads call it.
template <typename Emit>
CSA_DEV void row_select(const uint32_t* keys, int n, int k, RowShared& sh, uint32_t kmin,
                        uint32_t kmax, Emit emit) {
  constexpr int kBins = 1 << kRowBits;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    sh.warp_a[warp] = kmin;
    sh.warp_b[warp] = kmax;
  }
  for (int b = tid; b < kBins; b += kThreads) sh.hist[b] = 0;
  cta_sync();
  uint32_t gmin = sh.warp_a[lane], gmax = sh.warp_b[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
    gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
  }
  cta_sync();  // every warp has read the min / max slots

  uint32_t prefix, mask;
  uint32_t k_rem = (uint32_t)k;
  if (gmin == gmax) {
    prefix = gmin;
    mask = 0xFFFFFFFFu;
  } else {
    const int top = 31 - __clz(gmin ^ gmax);
    mask = top == 31 ? 0u : (0xFFFFFFFFu << (top + 1));
    prefix = gmin & mask;
    k_rem = row_rounds(keys, n, k_rem, sh, prefix, mask, top + 1);
  }
  ordered_emit(keys, n, k, prefix, mask, k_rem, 0u, 0u, sh, emit);
}

__global__ void __launch_bounds__(kThreads, 1) topk_row_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kRowKeysOff);
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t pos = p.pos_q ? p.pos_q[row] : p.pos_base + row % p.Q;
  pdl_trigger();
  pdl_wait();  // the scores come from the indexer kernel
  int64_t n64 = pos < 0 ? 0 : (pos + 1) / p.m - p.entry_offset;
  if (n64 < 0) n64 = 0;
  if (n64 > p.N_cap) {
    n64 = p.N_cap;
    if (tid == 0) report(p.status, CSA_ERR_CAPACITY);
  }
  const int n = (int)n64;
  int32_t* out = p.idx + (int64_t)row * p.k;
  if (n <= p.k) {  // every visible entry is kept
    for (int j = tid; j < p.k; j += kThreads) out[j] = j < n ? j : -1;
    if (tid == 0) p.cnt[row] = n;
    return;
  }
  // The visible scores as order-preserving keys, with this thread's min/max.
  const float* src = p.scores + (int64_t)row * p.N_cap;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  const bool vec = ((reinterpret_cast<uintptr_t>(src) & 15u) == 0);
  const int n4 = vec ? (n & ~3) : 0;
#pragma unroll 4
  for (int i = 4 * tid; i < n4; i += 4 * kThreads) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(src + i));
    const uint4 u = make_uint4(orderable(v.x), orderable(v.y), orderable(v.z), orderable(v.w));
    *reinterpret_cast<uint4*>(keys + i) = u;
    kmin = min(kmin, min(min(u.x, u.y), min(u.z, u.w)));
    kmax = max(kmax, max(max(u.x, u.y), max(u.z, u.w)));
  }
  for (int i = n4 + tid; i < n; i += kThreads) {
    const uint32_t u = orderable(__ldg(src + i));
    keys[i] = u;
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  }
  row_select(keys, n, p.k, sh, kmin, kmax, [&](uint32_t o, int i) { out[o] = i; });
  if (tid == 0) p.cnt[row] = p.k;
}

// --------------------------------------------- histogram-seeded selection --
// Decode chain (a few long rows): the indexer kernel has counted each row's
// visible scores by the top kScoreHistBits bits of their keys, so the bin
// b* holding the k-th largest key is known from the histogram alone, and
// one exchange replaces the (min, max) round and the first digit rounds.
// One cluster of C CTAs per row, each with its slice of the row in shared
// memory as keys (the layout of topk_kernel, whose select is the fallback):
//   - every CTA reads the whole histogram and finds b* (a block scan);
//   - each CTA counts its keys above b* and copies its keys in b* (the
//     candidates, at most kScoreHistBins / C) into its slot of a candidate
//     buffer; one push sends both to every CTA, then one cluster barrier;
//   - the counts are the keys' own, so whether b* holds the threshold is
//     checked, not assumed (A above b* < k <= A + candidates); if not, or
//     if a slot overflowed, the cluster runs the full radix select;
//   - otherwise each CTA ranks the candidates of all slots locally (radix
//     rounds below b*), which gives the threshold key, and from the
//     per-slot counts above / equal to it its offset in the index-ordered
//     output, then emits its slice.  Each warp owns a contiguous chunk of
//     the slice and lists, in order, the positions of its keys in b* or
//     above (every key the selection can take), so the emission reads only
//     those; a warp whose list overflows sends the CTA through the emission
//     over its whole slice.
// The histogram is cleared (each CTA its share) once every CTA has read it.
constexpr int kListCap = 64;  // listed positions per warp
struct HistShared {
  alignas(16) uint32_t cbuf[kScoreHistBins];  // candidates, slot c at [c*cap, (c+1)*cap)
  alignas(16) uint32_t cn[kMaxC][2];           // per-slot (above b*, candidates)
  uint32_t gq[kMaxC][2];                       // per-slot (above T, equal to T)
  uint32_t cand_n, above_n, bstar, list_ovf;
  uint32_t list_n[32];                         // per-warp list lengths
  uint16_t list[32][kListCap];                 // per-warp positions at or above b*
  RowShared row;                               // rounds over the candidates
};

__global__ void __launch_bounds__(kThreads, 1) topk_hist_kernel(const Params p) {
  using S = Shared<(1 << kDigitBits)>;
  constexpr int kShift = 32 - kScoreHistBits;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(S));
  HistShared& hs = *reinterpret_cast<HistShared*>(smem_raw + p.hist_off);

  const int row = blockIdx.y;
  const int C = p.C;
  const int cap = kScoreHistBins / C;  // candidate slots per CTA
  const uint32_t r = cluster_ctarank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_trigger();
  const int64_t pos = p.pos_q ? p.pos_q[row] : p.pos_base + row % p.Q;
  const int64_t lo = (int64_t)r * p.slice;
  int64_t n = pos < 0 ? 0 : (pos + 1) / p.m - p.entry_offset;
  if (n < 0) n = 0;
  if (tid == 0) {
    hs.cand_n = 0;
    hs.above_n = 0;
    hs.bstar = 0xFFFFFFFFu;  // no bin found
    hs.list_ovf = 0;
  }
  cluster_arrive();  // paired with the wait before the first remote store
  pdl_wait();  // the scores and the histogram come from the indexer kernel
  uint32_t* gh = p.hist + (int64_t)row * kScoreHistBins;
  const int zb = kScoreHistBins / C;  // bins this CTA clears, from r * zb
  int32_t* out = p.idx + (int64_t)row * p.k;
  if (n > p.N_cap) {
    n = p.N_cap;
    if (r == 0 && tid == 0) report(p.status, CSA_ERR_CAPACITY);
  }
  if (n <= p.k) {  // every visible entry is kept; nobody reads the histogram
    if (r == 0) {
      for (int j = tid; j < p.k; j += kThreads) out[j] = j < n ? j : -1;
      if (tid == 0) {
        p.cnt[row] = (int32_t)n;
        if (p.path) p.path[row] = 0;
      }
    }
    for (int j = tid; j < zb; j += kThreads) gh[r * zb + j] = 0u;
    cluster_wait();
    return;
  }
  // Thread t's four bins, highest first (kScoreHistBins == 4 * kThreads),
  // and the first kPer of its slice's scores, both in flight during the scan.
  const uint4 h4 = __ldcg(reinterpret_cast<const uint4*>(gh) + (kThreads - 1 - tid));
  const int cap_n = (int)(p.N_cap - lo < p.slice ? (p.N_cap - lo > 0 ? p.N_cap - lo : 0) : p.slice);
  const float* src = p.scores + (int64_t)row * p.N_cap + lo;
  const int len = (int)(n - lo < cap_n ? (n - lo > 0 ? n - lo : 0) : cap_n);
  // Warp w owns positions [w*ch, (w+1)*ch) of the slice (ch a multiple of
  // 32); lane l reads position w*ch + 32*j + l at step j, kPer steps per pass.
  const int ch = (((len + 31) / 32) + 31) & ~31;
  const int wbase = warp * ch;
  constexpr int kPer = 8;  // scores per thread per pass (slices up to 8192 in one)
  float sv[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = wbase + 32 * j + lane;
    sv[j] = (32 * j < ch && i < len) ? __ldg(src + i) : 0.f;
  }

  // b*: an exclusive scan over threads counts the scores in higher bins.
  {
    const uint32_t c4[4] = {h4.w, h4.z, h4.y, h4.x};
    uint32_t above = block_excl_scan(c4[0] + c4[1] + c4[2] + c4[3], hs.row.scan);
    const uint32_t k = (uint32_t)p.k;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // (The lowest such bin: with a histogram that does not add up, the
      // CTAs of the cluster still agree on b*.)
      if (above < k && above + c4[j] >= k)
        atomicMin(&hs.bstar, (uint32_t)(kScoreHistBins - 1 - 4 * tid - j));
      above += c4[j];
    }
  }
  cta_sync();
  const uint32_t bstar = hs.bstar;

  // This CTA's keys (to shared memory) above b* (counted), pass by pass
  // over the visible part of the slice; each warp lists the positions of its
  // keys in b* or above, in order.
  uint32_t n_above = 0, n_list = 0;
  uint32_t* mine = hs.cbuf + r * cap;
  uint16_t* my_list = hs.list[warp];
  const uint32_t lt = (1u << lane) - 1u;
  for (int j0 = 0; 32 * j0 < ch; j0 += kPer) {
    if (j0 > 0) {
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = wbase + 32 * (j0 + j) + lane;
        sv[j] = (32 * (j0 + j) < ch && i < len) ? __ldg(src + i) : 0.f;
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = wbase + 32 * (j0 + j) + lane;
      const bool in = 32 * (j0 + j) < ch && i < len;
      const uint32_t key = orderable(sv[j]);
      if (in) keys[i] = key;
      const uint32_t bin = key >> kShift;
      n_above += (in && bin > bstar) ? 1u : 0u;
      const bool ge = in && bin >= bstar;
      const uint32_t bge = __ballot_sync(0xffffffffu, ge);
      const uint32_t o = n_list + __popc(bge & lt);
      if (ge && o < (uint32_t)kListCap) my_list[o] = (uint16_t)i;
      n_list += __popc(bge);
    }
  }
  // The keys in b* (the candidates) to this CTA's slot, from the warp's list
  // or, where it overflowed, from its chunk of keys.
  __syncwarp();  // the warp's keys are in shared memory
  auto append = [&](bool cand, uint32_t key) {
    const uint32_t bal = __ballot_sync(0xffffffffu, cand);
    if (bal) {
      uint32_t at = 0;
      if (lane == 0) at = atomicAdd(&hs.cand_n, (uint32_t)__popc(bal));
      at = __shfl_sync(0xffffffffu, at, 0);
      const uint32_t o = at + __popc(bal & lt);
      if (cand && o < (uint32_t)cap) mine[o] = key;
    }
  };
  if (n_list <= (uint32_t)kListCap) {
    for (int e0 = 0; e0 < (int)n_list; e0 += 32) {
      const int e = e0 + lane;
      const uint32_t key = e < (int)n_list ? keys[my_list[e]] : 0u;
      append(e < (int)n_list && (key >> kShift) == bstar, key);
    }
  } else {
    const int wend = min(len, wbase + ch);
    for (int i0 = wbase; i0 < wend; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t key = i < wend ? keys[i] : 0u;
      append(i < wend && (key >> kShift) == bstar, key);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n_above += __shfl_xor_sync(0xffffffffu, n_above, o);
  if (lane == 0) {
    if (n_above) atomicAdd(&hs.above_n, n_above);
    hs.list_n[warp] = n_list;
    if (n_list > (uint32_t)kListCap) hs.list_ovf = 1;
  }
  cta_sync();
  cluster_wait();  // every CTA of the cluster is running

  // One exchange: counts and candidates into slot r of every CTA.
  const uint32_t my_a = hs.above_n, my_c = hs.cand_n;
  if (tid < C) st_remote_v2(mapa(smem_u32(&hs.cn[r][0]), tid), my_a, my_c);
  const int nv4 = ((int)min(my_c, (uint32_t)cap) + 3) / 4;
  for (int t = tid; t < C * nv4; t += kThreads) {
    const int c = t / nv4, j = t % nv4;
    if (c == (int)r) continue;
    const uint4 v = reinterpret_cast<const uint4*>(mine)[j];
    st_remote_v4(mapa(smem_u32(mine + 4 * j), c), v);
  }
  cluster_arrive();
  cluster_wait();
  // Every CTA has read the histogram: clear this CTA's share.
  for (int j = tid; j < zb / 4; j += kThreads)
    reinterpret_cast<uint4*>(gh + r * zb)[j] = make_uint4(0u, 0u, 0u, 0u);

  uint32_t A = 0, Mc = 0;
  bool ovf = false;
  for (int c = 0; c < C; ++c) {
    A += hs.cn[c][0];
    Mc += hs.cn[c][1];
    ovf = ovf || hs.cn[c][1] > (uint32_t)cap;
  }
  const uint32_t k = (uint32_t)p.k;
  if (bstar == 0xFFFFFFFFu || ovf || A >= k || A + Mc < k) {
    // The histogram did not hold this row's scores: the full select.
    cluster_select<kDigitBits, false>(smem_raw, C, r, p.k, len, lo, out);
    if (r == 0 && tid == 0) {
      p.cnt[row] = p.k;
      if (p.path) p.path[row] = 2;
    }
    return;
  }

  // The threshold among the candidates (unused slots hold a key outside b*).
  const uint32_t pad = (bstar ^ 1u) << kShift;
  for (int i = tid; i < kScoreHistBins; i += kThreads)
    if ((uint32_t)(i % cap) >= hs.cn[i / cap][1]) hs.cbuf[i] = pad;
  for (int b = tid; b < (1 << 10); b += kThreads) hs.row.hist[b] = 0u;
  cta_sync();
  uint32_t T = bstar << kShift, M = 0xFFFFFFFFu << kShift;
  const uint32_t need_eq = row_rounds<10>(hs.cbuf, kScoreHistBins, k - A, hs.row, T, M, kShift);
  // Per slot: keys above T (those above b* included) and equal to it; for
  // the emission over the lists, each warp's own counts (read by every warp
  // after the barrier below, which serves both).
  const bool lists = hs.list_ovf == 0;
  const int n_mine = (int)hs.list_n[warp];
  if (lists) {
    uint32_t gt, eq;
    list_counts(keys, hs.list[warp], n_mine, T, M, gt, eq);
    if (lane == 0) {
      hs.row.warp_a[warp] = gt;
      hs.row.warp_b[warp] = eq;
    }
  }
  if (warp < C) {
    const uint32_t nc = hs.cn[warp][1];
    uint32_t gt = 0, eq = 0;
    for (uint32_t j = lane; j < nc; j += 32) {
      const uint32_t km = hs.cbuf[warp * cap + j] & M;
      gt += km > T;
      eq += km == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
      hs.gq[warp][0] = hs.cn[warp][0] + gt;
      hs.gq[warp][1] = eq;
    }
  }
  cta_sync();
  uint32_t gt_base = 0, eq_base = 0;
  for (int c = 0; c < (int)r; ++c) {
    gt_base += hs.gq[c][0];
    eq_base += hs.gq[c][1];
  }
  auto put = [&](uint32_t o, int i) { out[o] = (int32_t)(lo + i); };
  if (!lists) {
    ordered_emit(keys, len, p.k, T, M, need_eq, gt_base, eq_base, hs.row, put);
  } else {
    // This warp's offset: the counts of the warps before it (a scan over
    // the 32 warps' counts, in every warp).
    const uint32_t a = hs.row.warp_a[lane], b = hs.row.warp_b[lane];
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
    const uint32_t pa = __shfl_sync(0xffffffffu, sa - a, warp);
    const uint32_t pb = __shfl_sync(0xffffffffu, sb - b, warp);
    list_emit(keys, hs.list[warp], n_mine, p.k, T, M, need_eq, gt_base + pa, eq_base + pb, put);
  }
  if (r == 0 && tid == 0) {
    p.cnt[row] = p.k;
    if (p.path) p.path[row] = 1;
  }
}

// ------------------------------------------------- context split over ranks --
// Candidates of one shard: the (score, sequence index) of each entry its
// local top-k kept; slots past the count get (NaN, -1).
__global__ void __launch_bounds__(256) shard_candidates_kernel(
    const float* __restrict__ scores, int64_t N_cap, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ cnt, int rows, int k, int64_t offset, float* __restrict__ cand_s,
    int32_t* __restrict__ cand_i) {
  pdl_trigger();
  pdl_wait();  // the selection comes from the top-k kernel
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)rows * k) return;
  const int row = (int)(t / k), j = (int)(t % k);
  const int c = cnt[row];
  const int32_t i = idx[t];
  if (j < c && i >= 0 && i < N_cap) {
    cand_s[t] = scores[(int64_t)row * N_cap + i];
    cand_i[t] = (int32_t)(i + offset);
  } else {
    cand_s[t] = __int_as_float(0x7fffffff);
    cand_i[t] = -1;
  }
}

struct MergeParams {
  int G, rows, k;
  const float* cand_s;     // [G, rows, k]
  const int32_t* cand_i;   // [G, rows, k] sequence indices, ascending per (rank, row)
  const int32_t* cand_c;   // [G, rows] candidates per rank
  int32_t* idx;            // [rows, k] sequence indices (written)
  int32_t* cnt;            // [rows]
  int64_t lo, hi;          // this rank's entries [lo, hi)
  int32_t* local_idx;      // [rows, k] local indices of this rank's selected entries
  int32_t* local_cnt;      // [rows]
  int32_t* status;
};

// Global top-k over the candidates of all ranks (one CTA per row).  The
// ranks' candidate lists are concatenated in rank order; each list holds
// ascending sequence indices and rank r's indices lie below rank r+1's, so a
// position in the concatenation orders candidates exactly as their sequence
// index does, and the tie rule (lower position first) is the method's (lower
// index first).  The exact top-k of the sequence lies within the union of
// the ranks' top-k lists.  Also writes this rank's share of the selection,
// as local indices: a contiguous run of the ascending output.
__global__ void __launch_bounds__(kThreads, 1) merge_candidates_kernel(const MergeParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RowShared& sh = *reinterpret_cast<RowShared*>(smem_raw);
  __shared__ int32_t s_off[65];
  __shared__ int32_t s_first, s_nloc;
  const int nmax = p.G * p.k;
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kRowKeysOff);
  int32_t* gidx = reinterpret_cast<int32_t*>(keys + nmax);
  const int row = blockIdx.x, tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
  if (tid == 0) {
    int o = 0;
    for (int r = 0; r < p.G; ++r) {
      s_off[r] = o;
      int c = p.cand_c[(int64_t)r * p.rows + row];
      c = c < 0 ? 0 : (c > p.k ? p.k : c);
      o += c;
    }
    s_off[p.G] = o;
    s_first = 0x7fffffff;
    s_nloc = 0;
  }
  cta_sync();
  const int n = s_off[p.G];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int r = 0; r < p.G; ++r) {
    const int base = s_off[r], c = s_off[r + 1] - base;
    const int64_t src = ((int64_t)r * p.rows + row) * p.k;
    for (int j = tid; j < c; j += kThreads) {
      const uint32_t u = orderable(p.cand_s[src + j]);
      keys[base + j] = u;
      gidx[base + j] = p.cand_i[src + j];
      kmin = min(kmin, u);
      kmax = max(kmax, u);
    }
  }
  cta_sync();
  int32_t* out = p.idx + (int64_t)row * p.k;
  const int total = n < p.k ? n : p.k;
  if (n <= p.k) {
    for (int j = tid; j < p.k; j += kThreads) out[j] = j < n ? gidx[j] : -1;
  } else {
    row_select(keys, n, p.k, sh, kmin, kmax, [&](uint32_t o, int i) { out[o] = gidx[i]; });
  }
  if (tid == 0) p.cnt[row] = total;
  __threadfence_block();
  cta_sync();  // the output row is complete (read back below)
  int32_t* loc = p.local_idx + (int64_t)row * p.k;
  for (int j = tid; j < total; j += kThreads) {
    const int64_t g = out[j];
    if (g >= p.lo && g < p.hi) {
      atomicMin(&s_first, j);
      atomicAdd(&s_nloc, 1);
    }
  }
  cta_sync();
  const int first = s_first, nloc = s_nloc;
  for (int j = tid; j < p.k; j += kThreads)
    loc[j] = j < nloc ? (int32_t)(out[first + j] - p.lo) : -1;
  if (tid == 0) p.local_cnt[row] = nloc;
}

}  // namespace

cudaError_t launch_shard_candidates(const float* scores, int64_t N_cap, const int32_t* idx,
                                    const int32_t* cnt, int rows, int k, int64_t offset,
                                    float* cand_s, int32_t* cand_i, cudaStream_t stream) {
  const int64_t n = (int64_t)rows * k;
  if (n <= 0) return cudaSuccess;
  return launch_pdl(shard_candidates_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                    stream, 0, 0, scores, N_cap, idx, cnt, rows, k, offset, cand_s, cand_i);
}

cudaError_t launch_merge_candidates(const MergeLaunch& a, cudaStream_t stream) {
  if (a.rows < 1) return cudaSuccess;
  if (a.G < 1 || a.G > 64 || a.k < 1 || a.k > kMaxK || a.rows > 65535)
    return cudaErrorInvalidConfiguration;
  MergeParams p{};
  p.G = a.G;
  p.rows = a.rows;
  p.k = a.k;
  p.cand_s = a.cand_s;
  p.cand_i = a.cand_i;
  p.cand_c = a.cand_c;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.lo = a.lo;
  p.hi = a.hi;
  p.local_idx = a.local_idx;
  p.local_cnt = a.local_cnt;
  p.status = a.status;
  const size_t smem = kRowKeysOff + (size_t)a.G * a.k * 8;
  if (smem > 220 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(merge_candidates_kernel), 9, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(merge_candidates_kernel, dim3(a.rows), dim3(kThreads), smem, stream, 0,
                    a.chained, p);
}

// Largest cluster size (8 or 16) that can be resident for this kernel and
// shared-memory size on the current device; cached per device and kernel
// (`which`: 0 topk_kernel, 1 topk_hist_kernel).  Also allows the 16-CTA
// size on the kernel.
int max_cluster(const void* kern, size_t smem, int which) {
  static int cached[64][2][2] = {};
  static size_t cached_smem[64][2] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (cached[dev][which][0] && cached_smem[dev][which] == smem) return cached[dev][which][1];
  int best = 8;
  bool failed = true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(16, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess) {
      failed = false;
      if (n >= 1) best = 16;
    }
  }
  if (failed) cudaGetLastError();  // a refused query is not the caller's error
  cached[dev][which][0] = 1;
  cached[dev][which][1] = best;
  cached_smem[dev][which] = smem;
  return best;
}

// Rows of at most this many scores take the one-CTA-per-row kernel.
constexpr int64_t kRowMaxScores = (200 * 1024 - (int64_t)kRowKeysOff) / 4;

// One CTA per row when rows fill the GPU (prefill) or are short; a few
// long rows (decode) spread each row over a cluster instead.
static bool row_path(int rows, int64_t N_cap) {
  return N_cap <= kRowMaxScores && (rows >= device_sm_count() / 4 || N_cap <= 8192);
}

bool topk_uses_hist(int rows, int64_t N_cap) {
  return rows >= 1 && rows <= 65535 && !row_path(rows, N_cap) && N_cap <= 8 * 32768;
}

// Cluster size of the radix (hist false) or histogram kernel for these rows,
// with the kernel's shared-memory limit set on the way; 0 if the rows do not
// fit.  Slices of at most 32768 scores; small batches spread each row over
// more CTAs (slices of at least 4096 scores), up to 16 where 16-CTA clusters
// fit.  The histogram kernel's HistShared follows the largest slice.
static int cluster_size(int rows, int64_t N_cap, bool hist) {
  const int need = (int)((N_cap + 32767) / 32768);
  if (need > 8 || rows < 1) return 0;
  auto kern = hist ? topk_hist_kernel : topk_kernel<kDigitBits, false>;
  using S = Shared<(1 << kDigitBits)>;
  const int64_t slice_max = (N_cap + need - 1) / need;
  const size_t hist_off = (sizeof(S) + (size_t)slice_max * 4 + 15) / 16 * 16;
  const size_t smem_max = hist ? hist_off + sizeof(HistShared) : sizeof(S) + (size_t)slice_max * 4;
  if (ensure_smem_attr(reinterpret_cast<const void*>(kern), hist ? 17 : 2, smem_max) !=
      cudaSuccess)
    return 0;
  const int limit = max_cluster(reinterpret_cast<const void*>(kern), smem_max, hist ? 1 : 0);
  int C = 1;
  while (C < need) C <<= 1;
  const int sms = device_sm_count();
  if (rows < sms) {
    const int fill = std::max(1, sms / rows);
    while (C * 2 <= limit && C * 2 <= fill && N_cap / (C * 2) >= 4096) C *= 2;
  }
  return C;
}

int topk_hist_ctas(int rows, int64_t N_cap) {
  if (!topk_uses_hist(rows, N_cap)) return 0;
  return rows * cluster_size(rows, N_cap, true);
}

static cudaError_t launch_topk_impl(const TopkLaunch& a, cudaStream_t stream) {
  if (a.rows < 1) return cudaSuccess;
  if (a.rows > 65535 || a.k > kMaxK) return cudaErrorInvalidConfiguration;
  if (row_path(a.rows, a.N_cap)) {
    Params p{};
    p.Q = a.Q;
    p.m = a.m;
    p.k = a.k;
    p.C = 1;
    p.N_cap = a.N_cap;
    p.entry_offset = a.entry_offset;
    p.slice = a.N_cap;
    p.scores = a.scores;
    p.pos_q = a.pos_q;
    p.pos_base = a.pos_base;
    p.idx = a.idx;
    p.cnt = a.cnt;
    p.status = a.status;
    const size_t smem = kRowKeysOff + (size_t)((a.N_cap + 3) / 4 * 4) * 4;
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(topk_row_kernel), 8, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_row_kernel, dim3(a.rows), dim3(kThreads), smem, stream, 0, a.chained,
                      p);
  }
  const bool hist = a.hist != nullptr;
  auto kern = hist ? topk_hist_kernel : topk_kernel<kDigitBits, false>;
  using S = Shared<(1 << kDigitBits)>;
  const int C = cluster_size(a.rows, a.N_cap, hist);
  if (C == 0) return cudaErrorInvalidValue;
  Params p{};
  p.Q = a.Q;
  p.m = a.m;
  p.k = a.k;
  p.C = C;
  p.N_cap = a.N_cap;
  p.entry_offset = a.entry_offset;
  p.slice = (a.N_cap + C - 1) / C;
  p.scores = a.scores;
  p.pos_q = a.pos_q;
  p.pos_base = a.pos_base;
  p.idx = a.idx;
  p.cnt = a.cnt;
  p.status = a.status;
  p.hist = a.hist;
  p.path = a.path;
  size_t smem = sizeof(S) + (size_t)p.slice * 4;
  if (hist) {
    p.hist_off = (uint32_t)((smem + 15) / 16 * 16);
    smem = p.hist_off + sizeof(HistShared);
  }
  return launch_pdl(kern, dim3(C, a.rows, 1), dim3(kThreads), smem, stream, C, a.chained, p);
}

cudaError_t launch_topk(const TopkLaunch& a, cudaStream_t stream) {
  if (a.hist && !topk_uses_hist(a.rows, a.N_cap)) return cudaErrorInvalidValue;
  return launch_topk_impl(a, stream);
}

}  // namespace csa
