// W8A8 low-rank prefill path (int8 x int8 -> int32 on tcgen05 tensor cores), sm_100a.
#include "common.cuh"
#include "internal.h"

namespace lr {

size_t w8a8_workspace_bytes(int T, int rank) {
  const size_t rp = (size_t(rank) + 127) / 128 * 128;
  const size_t tp = (size_t(T) + 127) / 128 * 128;
  auto ru = [](size_t v) { return (v + 255) / 256 * 256; };
  return ru(size_t(T) * rank * 4) + ru(tp * rp) + ru(tp * 4);
}

cudaError_t launch_w8a8(const W8A8Params&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace lr
