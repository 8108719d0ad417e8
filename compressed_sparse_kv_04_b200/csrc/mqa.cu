// Shared-KV MQA decode (placeholder until the tcgen05 kernel lands).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace csa {

size_t mqa_workspace_bytes(int rows, int splits, int H, int D) {
  size_t o = (size_t)rows * splits * H * D * 4;
  o = (o + 255) / 256 * 256;
  return o + (size_t)rows * splits * 2 * H * 4;
}

int mqa_choose_splits(int rows, int64_t max_kv, int num_sms) {
  int64_t tiles = (max_kv + 63) / 64;
  int pairs = std::max(1, num_sms / 2);
  int64_t s = (pairs + rows - 1) / rows;
  s = std::min<int64_t>(s, std::max<int64_t>(1, tiles));
  return (int)std::max<int64_t>(1, s);
}

cudaError_t launch_mqa(const MqaLaunch&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace csa
