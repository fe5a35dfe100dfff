// Per-token symmetric int8 quantisation of activations (W8A8), sm_100a.
//
// LASER results (W8A8 setting) and WSVD QAT section (weights and
// activations quantised): one scale per token, s = max|x| / 127, and
// q = clamp(rint(x / s), -127, 127).  Division and rounding are IEEE fp32
// (the quotient correctly rounded, rint ties to even) so that the codes are
// reproducible bit for bit; the quotient is only evaluated where a product
// with the reciprocal cannot decide the integer (quant_code).  An all-zero
// row gets s = 1 and q = 0.
#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace lr {
namespace {

// Each thread holds up to kPer 16-byte pieces (8 values each) of its row in
// registers, all loads issued before the row maximum is formed; the block
// is sized to the row (cols / (8 kPer) threads, rounded up to whole warps),
// so a row needs one pass over global memory and nothing is staged in
// shared memory.  Longer rows than kPer * kMaxThreads pieces would re-read the rest.
constexpr int kPer = 4;
constexpr int kMaxThreads = 512;

LR_DEV uint2 quantize8(const uint4 v, float sc, float inv, bool zero) {
  float f[8];
  bf16x8_to_f32(v, f);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float q = zero ? 0.f : quant_code(f[e], sc, inv);
    w[e >> 2] |= (uint32_t(int(q)) & 0xffu) << (8 * (e & 3));
  }
  return make_uint2(w[0], w[1]);
}

LR_DEV float amax8(const uint4 v, float m) {
  float f[8];
  bf16x8_to_f32(v, f);
#pragma unroll
  for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
  return m;
}

__global__ void __launch_bounds__(kMaxThreads) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int cols,
                                                             int8_t* __restrict__ xq, float* __restrict__ s) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const int nchunk = cols / 8;
  const int nt = blockDim.x;
  pdl_launch_dependents();
  pdl_wait();
  const uint4* src = reinterpret_cast<const uint4*>(x + size_t(t) * cols);
  uint4 v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = threadIdx.x + i * nt;
    v[i] = c < nchunk ? ld_stream16(src + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) amax = amax8(v[i], amax);
  for (int c = threadIdx.x + kPer * nt; c < nchunk; c += nt) amax = amax8(ld_stream16(src + c), amax);
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int w = 1; w < nt / 32; ++w) amax = fmaxf(amax, red[w]);
  float sc = __fdiv_rn(amax, 127.0f);
  const bool zero = (sc == 0.0f);
  if (zero) sc = 1.0f;
  if (threadIdx.x == 0) s[t] = sc;
  const float inv = __frcp_rn(sc);
  uint2* dst = reinterpret_cast<uint2*>(xq + size_t(t) * cols);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = threadIdx.x + i * nt;
    if (c < nchunk) dst[c] = quantize8(v[i], sc, inv, zero);
  }
  for (int c = threadIdx.x + kPer * nt; c < nchunk; c += nt) dst[c] = quantize8(ld_stream16(src + c), sc, inv, zero);
}

}  // namespace

cudaError_t launch_quantize_per_token(const void* x, int rows, int cols, int8_t* xq, float* s, cudaStream_t st) {
  const int nchunk = cols / 8;
  int threads = (nchunk + kPer - 1) / kPer;
  threads = (threads + 31) / 32 * 32;
  if (threads < 64) threads = 64;
  if (threads > kMaxThreads) threads = kMaxThreads;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(rows);
  c.blockDim = dim3(threads);
  c.dynamicSmemBytes = 0;
  c.stream = st;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, quantize_rows_kernel, reinterpret_cast<const __nv_bfloat16*>(x), cols, xq, s);
}

}  // namespace lr
