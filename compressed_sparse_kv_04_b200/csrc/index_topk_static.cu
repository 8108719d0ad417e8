// lightning_index_topk_static: lightning_index_topk with its fp32 score
// matrix held in a fixed device array of this library, so that the call
// needs no memory from the caller beyond its inputs and outputs and
// allocates none itself.
//
// Who needs it: a caller running under another memory manager that has
// already reserved the device's memory (a serving engine that pre-reserves
// nearly all HBM for its KV cache, or a framework allocator whose pool must
// not be bypassed), and a caller that may not stall the device -- cudaFree
// synchronises it -- or whose fixed interface has no workspace argument to
// pass.  Such a caller cannot get the score workspace lightning_index_topk
// asks for.
//
// Cost: every GPU that loads the library holds kStaticScores fp32 scores
// (8 MiB) until the process exits, whether or not this call is used.
#include <atomic>
#include <mutex>

#include "kernels.h"

namespace {

// Capacity of the array in fp32 scores: B * Q * N_cap may not exceed it.
// 2^21 scores cover a batch of 8 at 128K tokens (8 x 32768 entries) and a
// batch of 4 at 1M tokens (4 x 262144 entries) with m = 4.
constexpr int64_t kStaticScores = int64_t(1) << 21;

// The scratch itself: one copy per device.  In host code this name is only a
// host-side stand-in; kernels are given the device address obtained below.
static __device__ __align__(256) float g_static_scores[kStaticScores];

constexpr int kMaxDevices = 64;
std::atomic<float*> g_scores_addr[kMaxDevices];
std::mutex g_setup_mu;

// Device address of g_static_scores on the current device, looked up once
// per device (with that device current) and cached.
csa_status static_scores_addr(const char* fn, float** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return csa::set_error(CSA_ERR_CUDA, "%s: cudaGetDevice: %s", fn, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return csa::set_error(CSA_ERR_UNSUPPORTED_SHAPE, "%s: device ordinal %d (supported: < %d)",
                          fn, dev, kMaxDevices);
  float* ptr = g_scores_addr[dev].load(std::memory_order_acquire);
  if (ptr) {
    *out = ptr;
    return CSA_OK;
  }
  std::lock_guard<std::mutex> lock(g_setup_mu);
  ptr = g_scores_addr[dev].load(std::memory_order_relaxed);
  if (!ptr) {
    void* sym = nullptr;
    e = cudaGetSymbolAddress(&sym, g_static_scores);
    if (e != cudaSuccess || sym == nullptr)
      return csa::set_error(CSA_ERR_CUDA, "%s: cudaGetSymbolAddress of the static score buffer: %s",
                            fn, cudaGetErrorString(e));
    ptr = static_cast<float*>(sym);
    g_scores_addr[dev].store(ptr, std::memory_order_release);
  }
  *out = ptr;
  return CSA_OK;
}

}  // namespace

extern "C" csa_status lightning_index_topk_static(
    const csa_params* p, int Q, const uint8_t* q_idx, const float* q_scale, const float* w,
    const uint8_t* idx_key, const float* idx_scale, int64_t N_cap, const int64_t* pos_q,
    int32_t* topk_idx, int32_t* topk_cnt, int32_t* dev_status, void* stream) {
  const char* fn = "lightning_index_topk_static";
  if (!p) return csa::set_error(CSA_ERR_INVALID_ARG, "%s: params is null", fn);
  if (p->B < 1 || Q < 1 || N_cap < 1)
    return csa::set_error(CSA_ERR_INVALID_ARG, "%s: B=%d Q=%d N_cap=%lld must be >= 1", fn, p->B,
                          Q, (long long)N_cap);
  const int64_t rows = (int64_t)p->B * Q;
  if (N_cap > kStaticScores / rows)
    return csa::set_error(CSA_ERR_WORKSPACE,
                          "%s: B*Q*N_cap = %lld*%lld scores exceed the static buffer of %lld "
                          "scores; use lightning_index_topk with a workspace",
                          fn, (long long)rows, (long long)N_cap, (long long)kStaticScores);
  float* scores = nullptr;
  const csa_status st = static_scores_addr(fn, &scores);
  if (st != CSA_OK) return st;
  // The indexer writes every score that the top-k then reads (the first
  // n_vis of each row), so nothing in the array has to start at zero.
  return lightning_index_topk(p, Q, q_idx, q_scale, w, idx_key, idx_scale, N_cap, pos_q,
                              topk_idx, topk_cnt, scores, nullptr, 0, dev_status, stream);
}
