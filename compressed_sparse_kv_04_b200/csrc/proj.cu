// Grouped output projection on the 5th-generation tensor cores.
//
// "DeepSeek V4 technical report" (agentupdate.ai), 混合注意力机制, item
// 分组输出投影 (grouped output projection): with head dim 512, projecting all
// head outputs straight back to the model dim d is costly, so the n_h heads
// are split into g groups, each group is first projected to an intermediate
// dim d_g, and the results are projected together back to d.  "DeepSeek
// V4-Pro" (llm-arch-kb), "1. Hybrid attention": g = 16, d_g = 1024.
//
//   y[t, j*d_g + r] = sum_c W_g[j, r, c] * o[t, j*H/g*D + c]      (per group j)
//   z[t, n]         = sum_i W_o[n, i]    * y[t, i]
//
// Both projections are one kernel, a bf16 GEMM with fp32 accumulation in
// tensor memory: C[t, c_off + n] = sum_k A[t, a_off + k] * W[w_off + n, k]
// per group (a_off, w_off, c_off step with the group index).
//
// Design (swap-AB): the MMA's M = 128 weight rows (output features), its
// N = a tile of BN tokens (16 .. 256), K in 64-element chunks.  Both
// operands are K-major with the 128-byte swizzle, loaded by TMA into a
// multi-stage ring (weights 16 KB + tokens BN*128 B per stage); tokens past
// T are zero-filled by the tensor map.  Warp 0 issues TMA, warp 1 issues
// tcgen05.mma (one elected thread), warps 2..5 read the 128 x BN fp32
// accumulator (one TMEM lane per output feature) and store bf16, or fp32
// split-K partials that proj_reduce_kernel sums.  At decode (a few tokens)
// the weights dominate the bytes: the grid splits K so that every SM
// streams weights.  Every wait is bounded.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tma.h"

namespace csa {
namespace {

constexpr int kThreads = 192;
constexpr int BM = 128;      // weight rows per tile (MMA M)
constexpr int KC = 64;       // K elements per chunk (one 128-byte swizzle row)

struct ProjParams {
  int T;                     // tokens
  int K;                     // inner dim per group
  int ksplit;                // K chunks per split
  int splits;                // split-K factor
  int n_tiles;               // BM-row tiles per group
  int a_group_cols;          // A column offset step per group
  int w_group_rows;          // W row offset step per group
  int c_group_cols;          // C column offset step per group
  int ldc;                   // C row stride (elements)
  __nv_bfloat16* c;          // splits == 1: bf16 [T, ldc]
  float* part;               // splits > 1: fp32 [splits, T, ldc]
  int32_t* status;
};

template <int BN>
struct PCfg {
  static constexpr int kWBytes = BM * KC * 2;   // 16 KB
  static constexpr int kABytes = BN * KC * 2;
  static constexpr int kStageBytes = kWBytes + kABytes;
  static constexpr int kStages = (200 * 1024) / kStageBytes < 8 ? (200 * 1024) / kStageBytes : 8;
  static constexpr uint32_t kCols = BN < 32 ? 32 : BN;  // TMEM columns (power of 2)
};

CSA_DEV uint64_t desc_kmaj(uint32_t saddr) { return sdesc_sw128(saddr, 16, 1024); }

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                     const __grid_constant__ CUtensorMap map_w, const ProjParams p) {
  using C = PCfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + C::kStages;
  uint64_t* accf = empty + C::kStages;  // the accumulator is complete
  uint64_t* drain = accf + 1;           // issued MMAs finished (abort path)
  uint64_t* done = drain + 1;           // one arrival per warp when its role is over
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_tile = blockIdx.x;
  const int t0 = blockIdx.y * BN;
  const int group = blockIdx.z / p.splits, split = blockIdx.z % p.splits;
  const int k_chunks = p.ksplit;
  const int k0 = split * p.ksplit * KC;
  const int w_row = group * p.w_group_rows + n_tile * BM;
  const int a_col = group * p.a_group_cols + k0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(drain, 1);
    mbar_init(done, kThreads / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();  // the next kernel may set itself up while this one runs

  if (warp == 0) {
    // ---------------------------------------------------------- producer --
    // Weights are caller inputs: the first ring's worth is requested before
    // the wait on the previous kernel; the token tile (which the previous
    // kernel may have written) only after it.
    if (elect_one()) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_w);
      constexpr int kS = C::kStages;
      const int pre = k_chunks < kS ? k_chunks : kS;
      for (int it = 0; it < pre; ++it) {
        uint8_t* st = smem + it * C::kStageBytes;
        mbar_expect_tx(&full[it], C::kStageBytes);
        tma_load_2d(st, &map_w, &full[it], k0 + it * KC, w_row);
      }
      pdl_wait();
      for (int it = 0; it < pre; ++it)
        tma_load_2d(smem + it * C::kStageBytes + C::kWBytes, &map_a, &full[it], a_col + it * KC,
                    t0);
      int it = pre;
      for (; it < k_chunks; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abort_flag)) break;
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_expect_tx(&full[s], C::kStageBytes);
        tma_load_2d(st, &map_w, &full[s], k0 + it * KC, w_row);
        tma_load_2d(st + C::kWBytes, &map_a, &full[s], a_col + it * KC, t0);
      }
      if (*abort_flag) {  // copies still in flight land before the CTA exits
        for (int j = it - kS > 0 ? it - kS : 0; j < it; ++j)
          mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    const uint32_t idesc = idesc_bf16(BM, BN, 0, 0);
    bool issued = false;
    for (int it = 0; it < k_chunks; ++it) {
      const int s = it % C::kStages;
      const bool ok = mbar_wait(&full[s], (it / C::kStages) & 1, p.status, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t wb = smem_u32(smem + s * C::kStageBytes);
        const uint32_t ab = wb + C::kWBytes;
#pragma unroll
        for (int kk = 0; kk < KC / 16; ++kk)
          mma_bf16_ss(tmem, desc_kmaj(wb + kk * 32), desc_kmaj(ab + kk * 32), idesc,
                      (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
        if (it == k_chunks - 1) mma_commit(accf);
      }
      __syncwarp();
      issued = true;
    }
    if (*abort_flag && issued) {  // let issued MMAs finish before TMEM is freed
      if (elect_one()) mma_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, p.status);
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    // Warp w reads TMEM lanes 32*(w%4) .. +31: output features; columns are
    // tokens.  One coalesced store per token per warp.
    const int q = warp & 3;
    const int n = n_tile * BM + 32 * q + lane;  // feature within the group
    const bool ok = mbar_wait(accf, 0, p.status, abort_flag);
    if (__all_sync(0xffffffffu, ok) && !*abort_flag) {
      tc_fence_after();
      const int col = group * p.c_group_cols + n;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        if (BN >= 32) {
          tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + c, v);
        } else {
          uint32_t h[16];
          tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + c, h);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = h[j];
        }
        tmem_wait_ld();
        const int nt = BN >= 32 ? 32 : BN;
        if (p.splits == 1) {
#pragma unroll
          for (int j = 0; j < nt; ++j) {
            const int t = t0 + c + j;
            if (t < p.T)
              p.c[(int64_t)t * p.ldc + col] = __float2bfloat16_rn(__uint_as_float(v[j]));
          }
        } else {
          float* dst = p.part + (int64_t)split * p.T * p.ldc;
#pragma unroll
          for (int j = 0; j < nt; ++j) {
            const int t = t0 + c + j;
            if (t < p.T) dst[(int64_t)t * p.ldc + col] = __uint_as_float(v[j]);
          }
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
    mbar_wait(done, 0, p.status);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kCols);
  }
}

// Sum of the split-K partials [splits, T, ldc] fp32 -> bf16 [T, ldc]; four
// columns per thread.
__global__ void __launch_bounds__(256) proj_reduce_kernel(const float* __restrict__ part,
                                                          int splits, int64_t n4,
                                                          int64_t stride,
                                                          __nv_bfloat16* __restrict__ out) {
  pdl_wait();  // the partials come from the GEMM kernel
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  pdl_trigger();
  if (i < n4) {
    float4 a = __ldcg(reinterpret_cast<const float4*>(part) + i);
    for (int s = 1; s < splits; ++s) {
      const float4 b = __ldcg(reinterpret_cast<const float4*>(part + s * stride) + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    uint2 w;
    w.x = pack_bf16(a.x, a.y);
    w.y = pack_bf16(a.z, a.w);
    reinterpret_cast<uint2*>(out)[i] = w;
  }
}

template <int BN>
cudaError_t launch_gemm(const ProjGemm& g, cudaStream_t stream) {
  using C = PCfg<BN>;
  CUtensorMap map_a, map_w;
  cudaError_t e = make_tmap_2d(&map_a, g.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.T,
                               (uint64_t)g.lda, BN, KC, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&map_w, g.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)g.w_rows,
                   (uint64_t)g.K, BM, KC, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  ProjParams p{};
  p.T = g.T;
  p.K = g.K;
  p.splits = g.splits;
  p.ksplit = g.K / KC / g.splits;
  p.n_tiles = g.N / BM;
  p.a_group_cols = g.K;
  p.w_group_rows = g.N;
  p.c_group_cols = g.N;
  p.ldc = g.ldc;
  p.c = reinterpret_cast<__nv_bfloat16*>(g.c);
  p.part = g.part;
  p.status = g.status;
  const size_t smem = 1024 + (size_t)C::kStages * C::kStageBytes + (2 * C::kStages + 3) * 8 + 16;
  auto kern = proj_gemm_kernel<BN>;
  int slot = 10;
  for (int b = 16; b < BN; b <<= 1) ++slot;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), slot, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(g.N / BM, (g.T + BN - 1) / BN, g.groups * g.splits);
  e = launch_pdl(kern, grid, dim3(kThreads), smem, stream, 0, g.chained, map_a, map_w, p);
  if (e != cudaSuccess || g.splits == 1) return e;
  const int64_t n4 = (int64_t)g.T * g.ldc / 4;
  return launch_pdl(proj_reduce_kernel, dim3((unsigned)((n4 + 255) / 256)), dim3(256), 0, stream, 0,
                    1, (const float*)g.part, g.splits, n4, (int64_t)g.T * g.ldc,
                    reinterpret_cast<__nv_bfloat16*>(g.c));
}

}  // namespace

int proj_token_tile(int T) {
  if (T <= 16) return 16;
  if (T <= 32) return 32;
  if (T <= 64) return 64;
  if (T <= 128) return 128;
  return 256;
}

int proj_choose_splits(int T, int N, int groups, int K, int num_sms) {
  const int bn = proj_token_tile(T);
  const int64_t tiles = (int64_t)(N / BM) * ((T + bn - 1) / bn) * groups;
  const int chunks = K / KC;
  int s = 1;
  // Split K while the grid stays within one wave and each split keeps at
  // least 8 chunks (and divides the chunk count).
  while (tiles * s * 2 <= num_sms && chunks % (s * 2) == 0 && chunks / (s * 2) >= 8) s *= 2;
  return s;
}

cudaError_t launch_proj_gemm(const ProjGemm& g, cudaStream_t stream) {
  if (g.T < 1 || g.N % BM || g.K % KC || g.splits < 1 || (g.K / KC) % g.splits) return cudaErrorInvalidValue;
  if ((g.T + 255) / 256 > 65535 || g.groups * g.splits > 65535) return cudaErrorInvalidConfiguration;
  switch (proj_token_tile(g.T)) {
    case 16: return launch_gemm<16>(g, stream);
    case 32: return launch_gemm<32>(g, stream);
    case 64: return launch_gemm<64>(g, stream);
    case 128: return launch_gemm<128>(g, stream);
    default: return launch_gemm<256>(g, stream);
  }
}

}  // namespace csa
