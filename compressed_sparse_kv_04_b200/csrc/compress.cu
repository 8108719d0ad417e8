// KV compression (CSA m=4, HCA m'=128): learned softmax pooling of each
// block of m token vectors, RMSNorm, bf16 storage; for the indexer-key
// stream, E4M3 row quantisation with one fp32 scale per row.
//
// "DeepSeek V4 technical report" (agentupdate.ai), hybrid attention: CSA step
// 1 (m tokens merged with learned attention-like weights) and the HCA
// paragraph (m' = 128, no overlap); "DeepSeek V4-Pro" (llm-arch-kb), "Hybrid
// attention" CSA / HCA bullets.  Weight form (the reading taken here):
// softmax_j(c_t . w_s + b_pos[j]) over the present tokens of the block.
// Overlapping variant (CSA; the pages fix "no overlap" for HCA only): entry i
// pools the window of m + overlap tokens i*m - overlap .. (i+1)*m - 1, with
// b_pos indexed by the window position, clipped at the sequence start and at
// the context end.
//
// Storage (the reading taken here): a KV entry is stored already rotated (RoPE
// on the last rope_dim dims, "DeepSeek V4-Pro" (llm-arch-kb), "Hybrid
// attention") to its own position (i+1)*m - 1, so attention uses it as
// stored; indexer keys are not rotated.
//
// Design: pure HBM streaming on CUDA cores.  A warp owns up to 16 tokens of
// a block and keeps an online-softmax accumulator of the block row in
// registers (16 fp32 per lane at d = 512); token rows are read with 16-byte
// coalesced loads, up to eight rows in flight per warp.  m <= 16: one warp
// per block, 8 blocks per 256-thread CTA.  m > 16: 8 warps per block, merged
// through shared memory.  Both streams of csa_compress run in one launch
// (blockIdx.y selects the stream).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct StreamArgs {
  const __nv_bfloat16* tok;  // [B, L_cap, dim]
  const float* w_s;          // [dim]
  const float* b_pos;        // [m + overlap]
  const float* gamma;        // [dim] or null
  __nv_bfloat16* out_bf16;   // [B, N_cap, dim] or null
  uint8_t* out_e4m3;         // [B, N_cap, dim] or null
  float* out_scale;          // [B, N_cap] (with out_e4m3)
  int dim;
  int rope_dim;              // > 0: the entry is stored rotated to (i+1)*m - 1
};

struct PoolArgs {
  StreamArgs s[2];
  int nstreams;
  int B, m;
  int overlap;             // tokens of block i-1 that entry i also pools
  int64_t L_cap, N_cap;
  const int64_t* ctx_len;  // [B] device, or null -> ctx_len_value
  int64_t ctx_len_value;
  int64_t first_block, n_blocks;
  // The cache holds entries entry_offset .. of the sequence: local entry i is
  // block entry_offset + i (its tokens and its rotation position).
  int64_t entry_offset;
  // 1: launched as the first kernel of a call with programmatic serialization
  // (it may start while the caller's previous kernel runs): every global
  // read waits for that kernel, and dependents are let in only afterwards.
  int pdl_head;
  // [B] device, or null.  Set: one block per sequence, the one holding
  // position pos_newest[b], pooled over tokens up to pos_newest[b].
  const int64_t* pos_newest;
  float eps;
  double inv_freq[64];  // rotation frequencies (rope_dim/2 entries)
  int32_t* status;
};

// Lane l holds elements  part * (32 * VEC) + l * VEC + v,  v < VEC.
template <int DIM>
struct Lane {
  static constexpr int E = DIM / 32;
  static constexpr int VEC = E < 8 ? E : 8;
  static constexpr int NPART = E / VEC;
  CSA_DEV static int elem(int lane, int part, int v) { return part * (32 * VEC) + lane * VEC + v; }
};

template <int DIM>
CSA_DEV void load_row(const __nv_bfloat16* row, int lane, float (&x)[DIM / 32]) {
  using LN = Lane<DIM>;
#pragma unroll
  for (int p = 0; p < LN::NPART; ++p) {
    const __nv_bfloat16* src = row + LN::elem(lane, p, 0);
    if constexpr (LN::VEC == 8) {
      uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
      uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        x[p * 8 + 2 * q] = bf16_lo(w[q]);
        x[p * 8 + 2 * q + 1] = bf16_hi(w[q]);
      }
    } else if constexpr (LN::VEC == 4) {
      uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
      x[p * 4 + 0] = bf16_lo(u.x);
      x[p * 4 + 1] = bf16_hi(u.x);
      x[p * 4 + 2] = bf16_lo(u.y);
      x[p * 4 + 3] = bf16_hi(u.y);
    } else {
      uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(src));
      x[p * 2 + 0] = bf16_lo(u);
      x[p * 2 + 1] = bf16_hi(u);
    }
  }
}

// A row's elements of this lane, still packed as bf16 pairs.
template <int DIM>
CSA_DEV void load_row_packed(const __nv_bfloat16* row, int lane, uint32_t (&w)[DIM / 64]) {
  using LN = Lane<DIM>;
#pragma unroll
  for (int p = 0; p < LN::NPART; ++p) {
    const __nv_bfloat16* src = row + LN::elem(lane, p, 0);
    if constexpr (LN::VEC == 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(src));
      w[p * 4] = u.x;
      w[p * 4 + 1] = u.y;
      w[p * 4 + 2] = u.z;
      w[p * 4 + 3] = u.w;
    } else if constexpr (LN::VEC == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
      w[p * 2] = u.x;
      w[p * 2 + 1] = u.y;
    } else {
      w[p] = __ldg(reinterpret_cast<const uint32_t*>(src));
    }
  }
}

// Online-softmax pooling of tokens [j0, j_use) of one block by one warp.
// Rows are fetched up to 8 at a time (packed, so 8 rows of d = 512 take 64
// registers); rows [j_use, j_load) may be fetched too (they are in bounds)
// so that the loads need not wait for the context length.
template <int DIM>
CSA_DEV void pool_tokens(const __nv_bfloat16* blk, int j0, int j_load, int j_use, int lane,
                         const float (&ws)[DIM / 32], const float* b_pos, float& mx, float& l,
                         float (&acc)[DIM / 32]) {
  constexpr int E = DIM / 32;
  constexpr int RB = 8;
  mx = -INFINITY;
  l = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  // The position biases of this warp's tokens (at most 32), one load per
  // lane up front instead of one dependent load per token.
  const float bp = j0 + lane < j_use ? __ldg(b_pos + j0 + lane) : 0.f;
  for (int j = j0; j < j_load; j += RB) {
    uint32_t w[RB][E / 2];
#pragma unroll
    for (int u = 0; u < RB; ++u)
      if (j + u < j_load) load_row_packed<DIM>(blk + (int64_t)(j + u) * DIM, lane, w[u]);
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      if (j + u >= j_use) break;
      float x[E];
#pragma unroll
      for (int e = 0; e < E / 2; ++e) {
        x[2 * e] = bf16_lo(w[u][e]);
        x[2 * e + 1] = bf16_hi(w[u][e]);
      }
      float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < E; ++e) d4[e & 3] = fmaf(x[e], ws[e], d4[e & 3]);
      float s = warp_sum((d4[0] + d4[1]) + (d4[2] + d4[3])) +
                __shfl_sync(0xffffffffu, bp, (j + u - j0) & 31);
      float mn = fmaxf(mx, s);
      float corr = __expf(mx - mn);
      float p = __expf(s - mn);
      l = l * corr + p;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(acc[e], corr, p * x[e]);
      mx = mn;
    }
  }
}

template <int DIM>
CSA_DEV void finish_row(const StreamArgs& sa, const PoolArgs& a, int64_t row, int64_t pos,
                        int lane, float (&p)[DIM / 32], float eps, const float (&gam)[DIM / 32]) {
  using LN = Lane<DIM>;
  constexpr int E = DIM / 32;
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss = fmaf(p[e], p[e], ss);
  ss = warp_sum(ss);
  float inv = 1.0f / sqrtf(ss / (float)DIM + eps);
#pragma unroll
  for (int part = 0; part < LN::NPART; ++part)
#pragma unroll
    for (int v = 0; v < LN::VEC; ++v) {
      int e = part * LN::VEC + v;
      p[e] = p[e] * inv * gam[e];
    }
  if (sa.rope_dim > 0) {
    // Rotate-half over the last R dims, to the entry's position.  Those dims
    // sit in the last part of lanes 32 - R/VEC .. 31; the partner of dim d
    // (d +- R/2) is held by lane ^ (R/2 / VEC).
    const int R = sa.rope_dim, half = R / 2;
    constexpr int lp = LN::NPART - 1;
    float other[LN::VEC];
#pragma unroll
    for (int v = 0; v < LN::VEC; ++v)
      other[v] = __shfl_xor_sync(0xffffffffu, p[lp * LN::VEC + v], half / LN::VEC);
    const int d0 = LN::elem(lane, lp, 0);
    if (d0 >= DIM - R) {
      const bool first = d0 < DIM - half;
#pragma unroll
      for (int v = 0; v < LN::VEC; ++v) {
        const int j = (d0 + v - (DIM - R)) % half;
        float sn, cs;
        sincos_reduced((double)pos * a.inv_freq[j], &sn, &cs);
        const float x = p[lp * LN::VEC + v], y = other[v];
        p[lp * LN::VEC + v] = first ? x * cs - y * sn : x * cs + y * sn;
      }
    }
  }
  pdl_wait();  // stores come after every earlier kernel of the stream
  if (sa.out_bf16) {
    __nv_bfloat16* dst = sa.out_bf16 + row * DIM;
#pragma unroll
    for (int part = 0; part < LN::NPART; ++part) {
      uint32_t w[LN::VEC / 2];
#pragma unroll
      for (int q = 0; q < LN::VEC / 2; ++q)
        w[q] = pack_bf16(p[part * LN::VEC + 2 * q], p[part * LN::VEC + 2 * q + 1]);
      __nv_bfloat16* d = dst + LN::elem(lane, part, 0);
      if constexpr (LN::VEC == 8)
        *reinterpret_cast<uint4*>(d) = make_uint4(w[0], w[1], w[2], w[3]);
      else if constexpr (LN::VEC == 4)
        *reinterpret_cast<uint2*>(d) = make_uint2(w[0], w[1]);
      else
        *reinterpret_cast<uint32_t*>(d) = w[0];
    }
  }
  if (sa.out_e4m3) {
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(p[e]));
    amax = warp_max(amax);
    float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    uint8_t* dst = sa.out_e4m3 + row * DIM;
#pragma unroll
    for (int part = 0; part < LN::NPART; ++part) {
      uint8_t codes[LN::VEC];
#pragma unroll
      for (int v = 0; v < LN::VEC; v += 2) {
        float2 f = make_float2(__fdiv_rn(p[part * LN::VEC + v], scale),
                               __fdiv_rn(p[part * LN::VEC + v + 1], scale));
        __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
        codes[v] = (uint8_t)(c2 & 0xFF);
        codes[v + 1] = (uint8_t)(c2 >> 8);
      }
      uint8_t* d = dst + LN::elem(lane, part, 0);
      if constexpr (LN::VEC == 8) {
        uint2 w;
        w.x = codes[0] | (codes[1] << 8) | (codes[2] << 16) | ((uint32_t)codes[3] << 24);
        w.y = codes[4] | (codes[5] << 8) | (codes[6] << 16) | ((uint32_t)codes[7] << 24);
        *reinterpret_cast<uint2*>(d) = w;
      } else if constexpr (LN::VEC == 4) {
        *reinterpret_cast<uint32_t*>(d) =
            codes[0] | (codes[1] << 8) | (codes[2] << 16) | ((uint32_t)codes[3] << 24);
      } else {
        *reinterpret_cast<uint16_t*>(d) = (uint16_t)(codes[0] | (codes[1] << 8));
      }
    }
    if (lane == 0) sa.out_scale[row] = scale;
  }
}

template <int DIM>
CSA_DEV void pool_stream(const PoolArgs& a, const StreamArgs& sa, float* smem) {
  constexpr int E = DIM / 32;
  using LN = Lane<DIM>;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Entry i pools the window of span = m + overlap tokens that ends with its
  // own block: window position j holds token i*m - overlap + j.
  const int span = a.m + a.overlap;
  const int G = span <= 16 ? 1 : kWarps;           // warps per block
  const int per_cta = kWarps / G;                  // blocks per CTA
  const int64_t unit = (int64_t)blockIdx.x * per_cta + warp / G;  // (b, block) pair
  const int64_t total = (int64_t)a.B * a.n_blocks;
  bool active = unit < total;
  int64_t b = 0, i = 0;
  int present = 0;
  if (active) {
    b = unit / a.n_blocks;
    int64_t L;
    if (a.pos_newest) {
      const int64_t t = a.pos_newest[b];
      L = t + 1;
      i = t < 0 ? 0 : t / a.m - a.entry_offset;
      if (t < 0 || i < 0 || i >= a.N_cap) {  // no block, or one outside the cache
        active = false;
        L = 0;
        i = 0;
        if (t >= 0 && threadIdx.x % 32 == 0) {
          pdl_wait();
          report(a.status, CSA_ERR_DEVICE_INDEX);
        }
      }
    } else {
      i = a.first_block + unit % a.n_blocks;
      L = a.ctx_len ? a.ctx_len[b] : a.ctx_len_value;
    }
    if (L > a.L_cap) L = a.L_cap;
    // Window positions [jlo, present) are present: none before token 0, none
    // at or past the context end, and nothing at all while the block's own
    // range is empty.
    const int64_t gi = a.entry_offset + i;  // block index in the sequence
    const int64_t rem = L - (gi * a.m - a.overlap);
    present = L - gi * a.m <= 0 ? 0 : (rem < span ? (int)rem : span);
  }
  const int64_t gblk = a.entry_offset + i;
  const int jlo = active && gblk * a.m < a.overlap ? (int)(a.overlap - gblk * a.m) : 0;
  float ws[E];
#pragma unroll
  for (int part = 0; part < LN::NPART; ++part)
#pragma unroll
    for (int v = 0; v < LN::VEC; ++v) ws[part * LN::VEC + v] = __ldg(sa.w_s + LN::elem(lane, part, v));
  // The gains, loaded with the other inputs (used after the pooling).
  float gam[E];
#pragma unroll
  for (int part = 0; part < LN::NPART; ++part)
#pragma unroll
    for (int v = 0; v < LN::VEC; ++v)
      gam[part * LN::VEC + v] = sa.gamma ? __ldg(sa.gamma + LN::elem(lane, part, v)) : 1.f;

  // Row j of the window is blk + j*DIM (only rows j >= jlo are touched).
  const __nv_bfloat16* blk = sa.tok + ((int64_t)b * a.L_cap + gblk * a.m - a.overlap) * DIM;
  float mx, l, acc[E];
  const int g = warp % G;
  const int per_warp = (span + G - 1) / G;
  // Rows in the buffer (fetched at once) and rows present (pooled).
  const int64_t in_buf = active ? a.L_cap - (gblk * a.m - a.overlap) : 0;
  const int avail = in_buf <= 0 ? 0 : (in_buf < span ? (int)in_buf : span);
  const int j0 = max(g * per_warp, jlo);
  const int j_load = max(j0, min(avail, g * per_warp + per_warp));
  const int j_use = max(j0, min(present, g * per_warp + per_warp));
  pool_tokens<DIM>(blk, j0, j_load, j_use, lane, ws, sa.b_pos, mx, l, acc);

  if (G == 1) {
    if (!active || present == 0) return;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] / l;
    finish_row<DIM>(sa, a, b * a.N_cap + i, (gblk + 1) * a.m - 1, lane, acc, a.eps, gam);
    return;
  }
  // Merge the G warp partials of the one block of this CTA.
  float* s_acc = smem;                 // [kWarps][DIM]
  float* s_ml = smem + kWarps * DIM;   // [kWarps][2]
#pragma unroll
  for (int part = 0; part < LN::NPART; ++part)
#pragma unroll
    for (int v = 0; v < LN::VEC; ++v)
      s_acc[warp * DIM + LN::elem(lane, part, v)] = acc[part * LN::VEC + v];
  if (lane == 0) {
    s_ml[2 * warp] = mx;
    s_ml[2 * warp + 1] = l;
  }
  __syncthreads();
  if (warp != 0 || !active || present == 0) return;
  float M = -INFINITY;
  for (int w = 0; w < G; ++w) M = fmaxf(M, s_ml[2 * w]);
  float L = 0.f, p[E];
#pragma unroll
  for (int e = 0; e < E; ++e) p[e] = 0.f;
  for (int w = 0; w < G; ++w) {
    float mw = s_ml[2 * w];
    if (mw == -INFINITY) continue;
    float c = __expf(mw - M);
    L = fmaf(s_ml[2 * w + 1], c, L);
#pragma unroll
    for (int part = 0; part < LN::NPART; ++part)
#pragma unroll
      for (int v = 0; v < LN::VEC; ++v)
        p[part * LN::VEC + v] = fmaf(s_acc[w * DIM + LN::elem(lane, part, v)], c,
                                     p[part * LN::VEC + v]);
  }
#pragma unroll
  for (int e = 0; e < E; ++e) p[e] = p[e] / L;
  finish_row<DIM>(sa, a, b * a.N_cap + i, (gblk + 1) * a.m - 1, lane, p, a.eps, gam);
}

__global__ void __launch_bounds__(kThreads) compress_kernel(const PoolArgs a) {
  extern __shared__ float smem[];
  if (a.pdl_head) pdl_wait();  // nothing of the caller's is read before its kernels end
  pdl_trigger();
  const StreamArgs& sa = a.s[blockIdx.y];
  switch (sa.dim) {
    case 512: pool_stream<512>(a, sa, smem); break;
    case 128: pool_stream<128>(a, sa, smem); break;
    case 64: pool_stream<64>(a, sa, smem); break;
    default:
      pdl_wait();
      report(a.status, CSA_ERR_UNSUPPORTED_SHAPE);
      break;
  }
}

}  // namespace

int compress_ctas(const CompressLaunch& c) {
  const int G = c.m + c.overlap <= 16 ? 1 : kWarps;
  const int per_cta = kWarps / G;
  const int64_t units = (int64_t)c.B * (c.pos_newest ? 1 : c.n_blocks);
  return (int)std::min<int64_t>((units + per_cta - 1) / per_cta * (c.idx_tok ? 2 : 1), 1 << 30);
}

cudaError_t launch_compress(const CompressLaunch& c, cudaStream_t stream) {
  PoolArgs a{};
  a.nstreams = c.idx_tok ? 2 : 1;
  a.s[0] = StreamArgs{reinterpret_cast<const __nv_bfloat16*>(c.kv_tok), c.w_s, c.b_pos, c.gamma,
                      reinterpret_cast<__nv_bfloat16*>(c.kv_c), nullptr, nullptr, c.d, c.rope_dim};
  if (c.idx_tok)
    a.s[1] = StreamArgs{reinterpret_cast<const __nv_bfloat16*>(c.idx_tok), c.w_s_idx, c.b_pos_idx,
                        nullptr, nullptr, c.idx_key, c.idx_scale, c.D_I, 0};
  for (int j = 0; j < 64; ++j) a.inv_freq[j] = c.inv_freq[j];
  a.B = c.B;
  a.m = c.m;
  a.overlap = c.overlap;
  a.L_cap = c.L_cap;
  a.N_cap = c.N_cap;
  a.ctx_len = c.ctx_len;
  a.ctx_len_value = c.ctx_len_value;
  a.first_block = c.first_block;
  a.entry_offset = c.entry_offset;
  a.pdl_head = c.pdl_head;
  a.n_blocks = c.pos_newest ? 1 : c.n_blocks;
  a.pos_newest = c.pos_newest;
  a.eps = c.eps;
  a.status = c.status;
  int G = c.m + c.overlap <= 16 ? 1 : kWarps;
  int per_cta = kWarps / G;
  int64_t units = (int64_t)c.B * a.n_blocks;
  if (units == 0) return cudaSuccess;
  int64_t grid_x = (units + per_cta - 1) / per_cta;
  if (grid_x > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  int maxdim = c.idx_tok && c.D_I > c.d ? c.D_I : c.d;
  size_t smem = G == 1 ? 0 : (size_t)kWarps * (maxdim + 2) * sizeof(float);
  dim3 grid((unsigned)grid_x, a.nstreams);
  return launch_pdl(compress_kernel, grid, dim3(kThreads), smem, stream, 0,
                    c.chained || c.pdl_head, a);
}

}  // namespace csa
