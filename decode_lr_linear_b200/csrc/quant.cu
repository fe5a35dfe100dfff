// Per-token symmetric int8 quantisation of activations (W8A8), sm_100a.
//
// LASER results (W8A8 setting) and WSVD QAT section (weights and
// activations quantised): one scale per token, s = max|x| / 127, and
// q = clamp(rint(x / s), -127, 127).  Division and rounding are IEEE fp32
// (__fdiv_rn, rintf: ties to even) so that the codes are reproducible bit for
// bit; an all-zero row gets s = 1 and q = 0.
#include "common.cuh"
#include "internal.h"

namespace lr {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int cols,
                                                                 int8_t* __restrict__ xq, float* __restrict__ s) {
  extern __shared__ __align__(16) uint4 row[];
  __shared__ float red[kThreads / 32];
  const int t = blockIdx.x;
  const int nchunk = cols / 8;
  pdl_launch_dependents();
  pdl_wait();
  const uint4* src = reinterpret_cast<const uint4*>(x + size_t(t) * cols);
  float amax = 0.f;
  for (int c = threadIdx.x; c < nchunk; c += kThreads) {
    const uint4 v = src[c];
    row[c] = v;
    float f[8];
    bf16x8_to_f32(v, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  float sc = __fdiv_rn(amax, 127.0f);
  const bool zero = (sc == 0.0f);
  if (zero) sc = 1.0f;
  if (threadIdx.x == 0) s[t] = sc;
  uint2* dst = reinterpret_cast<uint2*>(xq + size_t(t) * cols);
  for (int c = threadIdx.x; c < nchunk; c += kThreads) {
    float f[8];
    bf16x8_to_f32(row[c], f);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float q = zero ? 0.f : rintf(__fdiv_rn(f[e], sc));
      q = fminf(fmaxf(q, -127.f), 127.f);
      const uint32_t byte = uint32_t(int(q)) & 0xffu;
      w[e >> 2] |= byte << (8 * (e & 3));
    }
    dst[c] = make_uint2(w[0], w[1]);
  }
}

}  // namespace

cudaError_t launch_quantize_per_token(const void* x, int rows, int cols, int8_t* xq, float* s, cudaStream_t st) {
  const size_t smem = size_t(cols) * 2;
  cudaError_t e = ensure_smem(quantize_rows_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(rows);
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = smem;
  c.stream = st;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, quantize_rows_kernel, reinterpret_cast<const __nv_bfloat16*>(x), cols, xq, s);
}

}  // namespace lr
