// Lightning Indexer scores on the 5th-generation tensor cores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), hybrid attention, CSA step
// 2: a light indexer scores each query against every compressed block;
// "DeepSeek V4-Pro" (llm-arch-kb), "Hybrid attention" CSA bullet: 64 indexer
// heads of dim 128; "KV Cache Compression ... Visualised" (webconsulting.at),
// "Dual Compression and Indexing": a low-precision pass.  Score form (the
// DSA reading): score_i = sum_h w_h ReLU(q_h . k_i) on dequantised E4M3
// values, computed as
//     score_i = s_k[i] * sum_h (w_h s_q[h]) * ReLU(sum_d q8[h,d] k8[i,d])
// which is the same number because every scale is >= 0.
//
// Design (swap-AB): A = a 128-entry tile of E4M3 keys (K-major, TMA with
// 128B/64B swizzle), B = the G queries' H_I heads (N = G * roundup16(H_I) <=
// 256 rows, K-major, loaded once per CTA), D = 128 entries x N in TMEM (fp32).
// With one TMEM lane per entry, the epilogue's reduction over heads is a
// per-thread loop over columns: no shuffles.  Warp roles: 0 = TMA producer,
// 1 = MMA issuer, 2..5 = epilogue (TMEM -> score).  The key ring is 6-8 stages
// deep and the accumulator is double-buffered, so loads, MMAs and the
// epilogue of consecutive tiles overlap.  Each CTA owns one query group and
// a contiguous range of tiles; the grid is sized to fill every SM.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma.h"

namespace csa {
namespace {

constexpr int kTileRows = 128;

// kHist: the histogram's 16 KB of shared memory come out of the key ring
// (five stages instead of six at D_I = 128), which keeps two CTAs per SM.
template <int DI, bool kHist = false>
struct Cfg {
  static constexpr int kStageBytes = kTileRows * DI;
  static constexpr int kStages = DI == 128 ? (kHist ? 5 : 6) : 8;
  static constexpr uint32_t kSBO = 8 * DI;               // 8 rows per swizzle atom
  static constexpr uint32_t kSwzMask = DI == 128 ? 7 : 3;  // 128B / 64B swizzle
  static constexpr uint64_t kLayout = DI == 128 ? 2 : 4;   // descriptor layout type
};

struct Params {
  int B, Q, H_I, HP, G, N, m;
  int64_t N_cap;
  int64_t entry_offset;  // the cache holds entries entry_offset .. of the sequence
  // Entries below this bound were written before this call and may be read
  // before pdl_wait(); the rest (written by the previous kernel of the
  // call) only after it.  safe_pos: per sequence, entries below
  // safe_pos[b] / m - entry_offset (the block holding position safe_pos[b]
  // is the one being written); else safe_fixed for every sequence.
  const int64_t* safe_pos;
  int64_t safe_fixed;
  int nchunks, ntiles, qgroups;  // chunk c: tiles [c*ntiles/nchunks, (c+1)*ntiles/nchunks)
  const uint8_t* q_idx;
  const float* q_scale;
  const float* w;
  const float* key_scale;
  const int64_t* pos_q;
  int64_t pos_base;
  float* scores;
  uint32_t* hist;  // [B, kScoreHistBins] (kHist launches)
  int32_t* status;
  uint32_t tmem_cols;
};

template <int DI>
CSA_DEV uint64_t desc_kmajor(uint32_t saddr) {
  uint64_t d = sdesc_sw128(saddr, 16, Cfg<DI>::kSBO);
  d &= ~(7ull << 61);
  d |= Cfg<DI>::kLayout << 61;
  return d;
}

// Entries of sequence b below this bound may be read before pdl_wait().
CSA_DEV int64_t safe_bound(const Params& p, int b) {
  if (!p.safe_pos) return p.safe_fixed;
  const int64_t t = p.safe_pos[b];
  const int64_t i = (t < 0 ? 0 : t / p.m) - p.entry_offset;
  return i < 0 ? 0 : i;
}

// Tiles the set-up issues into the key ring: the CTA's first tiles, up to
// one per stage, while their entries lie below the safe bound.
CSA_DEV int early_tiles(const Params& p, int b, int t_begin, int t_end, int stages) {
  const int64_t safe = safe_bound(p, b);
  int n = 0;
  while (n < stages && t_begin + n < t_end && (int64_t)(t_begin + n + 1) * kTileRows <= safe) ++n;
  return n;
}

// EW epilogue warps: 4 (one per TMEM lane quarter; two CTAs per SM), or 8
// when the group holds several queries (two warps per quarter, queries
// alternating), which halves the epilogue's work per thread where it bounds
// the kernel (prefill: four queries x 64 heads per entry and tile).
// kHist (one query per sequence): the epilogue also counts each visible
// score by the top kScoreHistBits bits of its key in a shared-memory
// histogram, added to the sequence's global histogram when the CTA is done
// (only the non-zero bins), so that the top-k that follows knows which bin
// holds its threshold before it reads a score.
template <int DI, int EW, bool kHist>
__global__ void __launch_bounds__(64 + 32 * EW, EW == 4 ? 2 : 1)
    index_score_kernel(const __grid_constant__ CUtensorMap kmap, const Params p) {
  using C = Cfg<DI, kHist>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;                                      // kStages x kStageBytes
  uint8_t* qtile = ring + C::kStages * C::kStageBytes;       // N x DI
  float* wq = reinterpret_cast<float*>(qtile + p.N * DI);    // N
  uint64_t* bars = reinterpret_cast<uint64_t*>(wq + 256);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* done = drain + 1;  // one arrival per warp when its role is over
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  // kHist: the lowest and highest bin any score of the CTA fell in, then
  // the histogram on the next 16-byte boundary.
  uint32_t* hrange = reinterpret_cast<uint32_t*>(const_cast<int*>(abort_flag + 1));
  uint32_t* shist = reinterpret_cast<uint32_t*>(
      (reinterpret_cast<uintptr_t>(hrange + 2) + 15) & ~uintptr_t(15));

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  pdl_trigger();
  const int group = blockIdx.y;
  const int b = group / p.qgroups;
  const int q0 = (group % p.qgroups) * p.G;
  const int nq = min(p.G, p.Q - q0);
  constexpr int kThr = 64 + 32 * EW;

  // The query tile's codes (B operand; row g*HP + h holds head h of query
  // q0+g, zero for padding heads and absent queries) and the head weights
  // are caller inputs, loaded first: the key stream, started below before
  // the rest of the set-up, would otherwise queue ahead of them.
  constexpr int kQPre = 3;  // chunks per thread held in registers (decode: all)
  const int nchunk = p.N * (DI / 16);
  auto q_chunk = [&](int c) -> uint4 {
    const int row = c / (DI / 16), chunk = c % (DI / 16);
    const int g = row / p.HP, h = row % p.HP;
    if (g >= nq || h >= p.H_I) return make_uint4(0, 0, 0, 0);
    return __ldg(reinterpret_cast<const uint4*>(
        p.q_idx + (((int64_t)b * p.Q + q0 + g) * p.H_I + h) * DI + chunk * 16));
  };
  uint4 qpre[kQPre];
#pragma unroll
  for (int j = 0; j < kQPre; ++j) {
    const int c = threadIdx.x + j * kThr;
    qpre[j] = c < nchunk ? q_chunk(c) : make_uint4(0, 0, 0, 0);
  }
  float wpre[2], spre[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int r = threadIdx.x + j * kThr;
    const int g = r / p.HP, h = r % p.HP;
    wpre[j] = spre[j] = 0.f;
    if (r < p.N && g < nq && h < p.H_I) {
      const int64_t o = ((int64_t)b * p.Q + q0 + g) * p.H_I + h;
      wpre[j] = __ldg(p.w + o);
      spre[j] = __ldg(p.q_scale + o);
    }
  }

  // Visible entries per query of the group (causal), clamped to capacity.
  int64_t nv_max = 0;
  for (int g = 0; g < nq; ++g) {
    int64_t pos = p.pos_q ? p.pos_q[(int64_t)b * p.Q + q0 + g] : p.pos_base + q0 + g;
    int64_t nv = pos < 0 ? 0 : (pos + 1) / p.m - p.entry_offset;
    if (nv < 0) nv = 0;
    if (nv > p.N_cap) nv = p.N_cap;
    nv_max = max(nv_max, nv);
  }
  const int t_begin = (int)((int64_t)blockIdx.x * p.ntiles / p.nchunks);
  const int t_vis = (int)((nv_max + kTileRows - 1) / kTileRows);
  const int t_end = min((int)((int64_t)(blockIdx.x + 1) * p.ntiles / p.nchunks), t_vis);
  if (t_begin >= t_end) {  // uniform over the CTA
    pdl_wait();  // this grid completes only after its predecessor
    return;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * EW);
    }
    mbar_init(drain, 1);
    mbar_init(done, 2 + EW);
    *abort_flag = 0;
    hrange[0] = kScoreHistBins;
    hrange[1] = 0u;
    fence_mbar_init();
    fence_proxy_async_smem();
    // The key stream starts here: the ring's stages take the CTA's first
    // tiles of entries written before this call (the producer continues
    // after them), so their latency overlaps the rest of the set-up.
    tma_prefetch_desc(&kmap);
    const int n_early = early_tiles(p, b, t_begin, t_end, C::kStages);
    for (int j = 0; j < n_early; ++j) {
      mbar_expect_tx(&full[j], C::kStageBytes);
      tma_load_2d(ring + j * C::kStageBytes, &kmap, &full[j], 0,
                  (int32_t)((int64_t)b * p.N_cap + (int64_t)(t_begin + j) * kTileRows));
    }
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(tmem_base_slot, p.tmem_cols);
    tmem_relinquish();
  }
  // The query tile in shared memory, with the swizzle the MMA descriptor
  // expects (chunks past the registers' share are loaded here).
  auto put_chunk = [&](int c, uint4 v) {
    const uint32_t lin = (c / (DI / 16)) * DI + (c % (DI / 16)) * 16;
    const uint32_t phys = lin ^ (((lin >> 7) & C::kSwzMask) << 4);
    *reinterpret_cast<uint4*>(qtile + phys) = v;
  };
#pragma unroll
  for (int j = 0; j < kQPre; ++j) {
    const int c = threadIdx.x + j * kThr;
    if (c < nchunk) put_chunk(c, qpre[j]);
  }
  for (int c = threadIdx.x + kQPre * kThr; c < nchunk; c += kThr) put_chunk(c, q_chunk(c));
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int r = threadIdx.x + j * kThr;
    if (r < p.N) wq[r] = wpre[j] * spre[j];
  }
  if (kHist)
    for (int i = threadIdx.x; i < kScoreHistBins; i += 64 + 32 * EW) shist[i] = 0u;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer --
    if (elect_one()) {
      // Tiles of entries written before this call stream at once (the first
      // ones were issued during the set-up); the first tile with an entry
      // that the previous kernel writes waits for it.
      const int64_t safe = safe_bound(p, b);
      bool waited = false;
      int it = early_tiles(p, b, t_begin, t_end, C::kStages);
      for (int t = t_begin + it; t < t_end; ++t, ++it) {
        int s = it % C::kStages;
        uint32_t ph = (it / C::kStages) & 1;
        if (!waited && (int64_t)(t + 1) * kTileRows > safe) {
          pdl_wait();
          waited = true;
        }
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abort_flag)) break;
        mbar_expect_tx(&full[s], C::kStageBytes);
        tma_load_2d(ring + s * C::kStageBytes, &kmap, &full[s], 0,
                    (int32_t)((int64_t)b * p.N_cap + (int64_t)t * kTileRows));
      }
      if (!waited) pdl_wait();  // this grid completes only after its predecessor
      // On abort, wait for the copies still in flight before the CTA exits.
      if (*abort_flag) {
        int issued = it;
        for (int j = max(0, issued - C::kStages); j < issued; ++j)
          mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.status);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (elect_one()) {
      const uint32_t idesc = idesc_e4m3(128, p.N);
      const uint32_t q_addr = smem_u32(qtile);
      int it = 0;
      bool issued_any = false;
      for (int t = t_begin; t < t_end; ++t, ++it) {
        int s = it % C::kStages;
        uint32_t ph = (it / C::kStages) & 1;
        if (!mbar_wait(&full[s], ph, p.status, abort_flag)) break;
        int a = it & 1;
        uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[a], aph ^ 1, p.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
        for (int k = 0; k < DI / 32; ++k)
          mma_e4m3_ss(tmem + a * p.N, desc_kmajor<DI>(a_addr + k * 32),
                      desc_kmajor<DI>(q_addr + k * 32), idesc, k > 0 ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&tfull[a]);
        issued_any = true;
      }
      if (*abort_flag && issued_any) {
        mma_commit(drain);
        mbar_wait(drain, 0, p.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int wg = (warp - 2) / 4;  // queries wg, wg + EW/4, ... of the group
    // Key scales follow the producer's rule (read through L2: a line may
    // hold scales from both sides of the bound); the scores are a buffer no
    // earlier kernel of the call touches.
    const int64_t safe = safe_bound(p, b);
    bool waited = false;
    auto ensure = [&](int t) {
      if (!waited && (int64_t)(t + 1) * kTileRows > safe) {
        pdl_wait();
        waited = true;
      }
    };
    int64_t nv[8];
#pragma unroll
    for (int g = 0; g < 8; ++g) nv[g] = 0;
    for (int g = 0; g < nq && g < 8; ++g) {
      int64_t pos = p.pos_q ? p.pos_q[(int64_t)b * p.Q + q0 + g] : p.pos_base + q0 + g;
      int64_t v = pos < 0 ? 0 : (pos + 1) / p.m - p.entry_offset;
      if (v < 0) v = 0;
      if (v > p.N_cap) {
        v = p.N_cap;
        if (row == 0 && t_begin == 0) report(p.status, CSA_ERR_CAPACITY);
      }
      nv[g] = v;
    }
    // Key scales of the next kKsAhead tiles are in flight (a register queue):
    // a tile's own work is far shorter than a load's latency, so one tile
    // ahead would leave the loop waiting on every load.  Tiles past the safe
    // bound load theirs on use, after the wait.
    constexpr int kKsAhead = 8;
    auto tile_safe = [&](int t) { return (int64_t)(t + 1) * kTileRows <= safe; };
    auto load_ks = [&](int t) -> float {
      const int64_t e = (int64_t)t * kTileRows + row;
      return e < p.N_cap ? __ldcg(p.key_scale + (int64_t)b * p.N_cap + e) : 0.f;
    };
    uint32_t hlo = kScoreHistBins, hhi = 0;  // kHist: this thread's bins
    float ksq[kKsAhead];
#pragma unroll
    for (int j = 0; j < kKsAhead; ++j)
      ksq[j] = (t_begin + j < t_end && tile_safe(t_begin + j)) ? load_ks(t_begin + j) : 0.f;
    int it = 0;
    for (int t = t_begin; t < t_end; ++t, ++it) {
      const int a = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const int64_t entry = (int64_t)t * kTileRows + row;
      float ks = ksq[0];
#pragma unroll
      for (int j = 0; j + 1 < kKsAhead; ++j) ksq[j] = ksq[j + 1];
      {
        const int tn = t + kKsAhead;
        ksq[kKsAhead - 1] = (tn < t_end && tile_safe(tn)) ? load_ks(tn) : 0.f;
      }
      if (!tile_safe(t)) {
        ensure(t);
        ks = load_ks(t);
      }
      bool ok = mbar_wait(&tfull[a], aph, p.status, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // keep the warp converged for tcgen05.ld
      tc_fence_after();
      for (int g = wg; g < nq; g += EW / 4) {
        if (p.HP == 64) {
          // 64 head columns in two loads; the weighted sum in packed fp32
          // FMAs (lane pairs = chains j & 3 of the generic path below, in
          // the same order: the same number).
          const uint32_t col = tmem_addr(tmem, quarter * 32, a * p.N + g * 64);
          const float4* wg4 = reinterpret_cast<const float4*>(wq + g * 64);
          float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int h0 = 0; h0 < 64; h0 += 32) {
            uint32_t v[32];
            tmem_ld32(col + h0, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 w4 = wg4[(h0 + j) >> 2];
              acc2[0] = fma_f32x2(make_float2(w4.x, w4.y),
                                  make_float2(fmaxf(__uint_as_float(v[j]), 0.f),
                                              fmaxf(__uint_as_float(v[j + 1]), 0.f)),
                                  acc2[0]);
              acc2[1] = fma_f32x2(make_float2(w4.z, w4.w),
                                  make_float2(fmaxf(__uint_as_float(v[j + 2]), 0.f),
                                              fmaxf(__uint_as_float(v[j + 3]), 0.f)),
                                  acc2[1]);
            }
          }
          const float acc = (acc2[0].x + acc2[0].y) + (acc2[1].x + acc2[1].y);
          if (entry < nv[g < 8 ? g : 7]) {
            const float sc = acc * ks;
            p.scores[((int64_t)b * p.Q + q0 + g) * p.N_cap + entry] = sc;
            if (kHist) {
              const uint32_t bin = score_key(sc) >> (32 - kScoreHistBits);
              atomicAdd(&shist[bin], 1u);
              hlo = min(hlo, bin);
              hhi = max(hhi, bin);
            }
          }
          continue;
        }
        // All of this query's head columns (<= 64) in flight, one wait.
        uint32_t v[4][16];
        const uint32_t col = tmem_addr(tmem, quarter * 32, a * p.N + g * p.HP);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c * 16 < p.HP) tmem_ld16(col + c * 16, v[c]);
        tmem_wait_ld();
        float a4[4] = {0.f, 0.f, 0.f, 0.f};  // independent FMA chains
        const float* wg = wq + g * p.HP;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c * 16 < p.HP) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              a4[j & 3] = fmaf(wg[c * 16 + j], fmaxf(__uint_as_float(v[c][j]), 0.f), a4[j & 3]);
          }
        const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
        if (entry < nv[g < 8 ? g : 7]) {
          const float sc = acc * ks;
          p.scores[((int64_t)b * p.Q + q0 + g) * p.N_cap + entry] = sc;
          if (kHist) {
            const uint32_t bin = score_key(sc) >> (32 - kScoreHistBits);
            atomicAdd(&shist[bin], 1u);
            hlo = min(hlo, bin);
            hhi = max(hhi, bin);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[a]);
    }
    if (!waited) pdl_wait();  // this grid completes only after its predecessor
    if (kHist) {
      // Every epilogue warp has counted its last score: add the non-zero
      // bins (within the range the CTA's scores fell in) to the sequence's
      // histogram.
      hlo = __reduce_min_sync(0xffffffffu, hlo);
      hhi = __reduce_max_sync(0xffffffffu, hhi);
      if (lane == 0) {
        atomicMin(&hrange[0], hlo);
        atomicMax(&hrange[1], hhi);
      }
      named_barrier_sync(1, 32 * EW);
      uint32_t* gh = p.hist + (int64_t)b * kScoreHistBins;
      const int lo = (int)hrange[0], hi = (int)hrange[1];
      for (int i = lo + threadIdx.x - 64; i <= hi; i += 32 * EW) {
        const uint32_t v = shist[i];
        if (v) atomicAdd(gh + i, v);
      }
    }
  }
  // Teardown: every warp reports (converged) that it is done with tensor
  // memory; warp 0 frees it after all of them (bounded wait).
  __syncwarp();
  tc_fence_before();
  if (lane == 0) mbar_arrive(done);
  if (warp == 0) {
    mbar_wait(done, 0, p.status);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

template <int DI, int EW, bool kHist>
cudaError_t launch_impl(const IndexLaunch& a, cudaStream_t stream) {
  using C = Cfg<DI, kHist>;
  Params p{};
  p.B = a.B;
  p.Q = a.Q;
  p.H_I = a.H_I;
  p.HP = (a.H_I + 15) / 16 * 16;
  p.G = std::max(1, std::min(std::min(a.Q, 256 / p.HP), 8));
  p.N = p.G * p.HP;
  p.m = a.m;
  p.N_cap = a.N_cap;
  p.entry_offset = a.entry_offset;
  p.safe_pos = a.safe_pos;
  p.safe_fixed = a.safe_fixed;
  p.ntiles = (int)((a.N_cap + kTileRows - 1) / kTileRows);
  p.qgroups = (a.Q + p.G - 1) / p.G;
  p.q_idx = a.q_idx;
  p.q_scale = a.q_scale;
  p.w = a.w;
  p.key_scale = a.key_scale;
  p.pos_q = a.pos_q;
  p.pos_base = a.pos_base;
  p.scores = a.scores;
  p.hist = a.hist;
  p.status = a.status;
  uint32_t cols = 32;
  while (cols < (uint32_t)(2 * p.N)) cols <<= 1;
  p.tmem_cols = cols;

  size_t smem = 1024 + (size_t)C::kStages * C::kStageBytes + (size_t)p.N * DI + 256 * 4 +
                (2 * C::kStages + 6) * 8 + 16;
  if (kHist) smem += 16 + kScoreHistBins * 4;  // range words + histogram
  auto kern = index_score_kernel<DI, EW, kHist>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern),
                                   (DI == 128 ? 0 : 1) + (EW == 8 ? 19 : 0) + (kHist ? 15 : 0),
                                   smem);
  if (e != cudaSuccess) return e;
  // Two CTAs per SM when shared memory allows it (228 KB per SM).
  int occ = (2 * (smem + 1024) <= 228 * 1024) ? 2 : 1;
  if (2 * cols > 512) occ = 1;  // two CTAs would contend for tensor memory
  if (EW == 8) occ = 1;  // 320 threads x ~130 registers: one CTA per SM
  int64_t groups = (int64_t)a.B * p.qgroups;
  if (groups > 65535) return cudaErrorInvalidConfiguration;
  // Every CTA resident at once: the slots the call's earlier kernel holds
  // (reserve_slots) are left out, so that no CTA starts only when it ends.
  // The tiles are split evenly (chunk sizes differ by at most one).
  const int64_t slots = std::max<int64_t>(1, (int64_t)a.num_sms * occ - a.reserve_slots);
  int chunks = 1;
  if (groups < slots) chunks = (int)std::max<int64_t>(1, std::min<int64_t>(p.ntiles, slots / groups));
  p.nchunks = chunks;

  CUtensorMap kmap;
  e = make_tmap_2d(&kmap, a.key, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.B * a.N_cap, DI,
                   kTileRows, DI, DI == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
  if (e != cudaSuccess) return e;
  dim3 grid(chunks, (unsigned)groups);
  return launch_pdl(kern, grid, dim3(64 + 32 * EW), smem, stream, 0, a.chained, kmap, p);
}

}  // namespace

cudaError_t launch_index_scores(const IndexLaunch& a, cudaStream_t stream) {
  if (a.B * (int64_t)a.N_cap > 0x7FFFFFFF) return cudaErrorInvalidValue;
  // Groups of several queries (prefill) take eight epilogue warps.
  const int HP = (a.H_I + 15) / 16 * 16;
  const bool wide = std::min(std::min(a.Q, 256 / HP), 8) >= 2;
  if (a.hist) {  // one query per sequence
    if (a.Q != 1) return cudaErrorInvalidValue;
    if (a.D_I == 128) return launch_impl<128, 4, true>(a, stream);
    if (a.D_I == 64) return launch_impl<64, 4, true>(a, stream);
    return cudaErrorInvalidValue;
  }
  if (a.D_I == 128)
    return wide ? launch_impl<128, 8, false>(a, stream) : launch_impl<128, 4, false>(a, stream);
  if (a.D_I == 64)
    return wide ? launch_impl<64, 8, false>(a, stream) : launch_impl<64, 4, false>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace csa
