// Single-query flash-decoding attention over full K/V caches, sm_100a: the
// uncompressed baseline that the latent-KV path is measured against (WSVD
// "Resultaten" and LASER results report speed-ups over FlashDecoding).
//
// Work is split over the context (split-K): one CTA per (split, head, batch)
// copies its K and V chunk into shared memory with two bulk asynchronous
// copies completing on one mbarrier (rows of head_dim bf16 are contiguous per
// (batch, head), so a chunk is one block), computes the chunk's scores, max,
// exponentials and the weighted value sum, and writes (max, sum, acc[128]);
// the combine kernel merges the splits with log-sum-exp rescaling.
#include "common.cuh"
#include "internal.h"

namespace lr {
namespace {

constexpr int kD = 128;          // head dim
constexpr int kThreads = 128;
constexpr int kPart = kD + 2;    // m, l, acc[head_dim]
constexpr float kLog2e = 1.4426950408889634f;

LR_DEV float block_max(float v, float* scratch) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float m = scratch[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, scratch[w]);
  __syncthreads();
  return m;
}

LR_DEV float block_sum(float v, float* scratch) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s += scratch[w];
  __syncthreads();
  return s;
}

__global__ void __launch_bounds__(kThreads) flash_split_kernel(const __grid_constant__ FlashParams P) {
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int T = P.split_tokens;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* vs = ks + size_t(T) * kD;
  float* sc = reinterpret_cast<float*>(vs + size_t(T) * kD);
  __shared__ float scratch[kThreads / 32];
  __shared__ __align__(8) uint64_t bar;

  pdl_launch_dependents();
  pdl_wait();
  int n_ctx = P.seq_lens[b];
  n_ctx = n_ctx < 0 ? 0 : (n_ctx > P.max_ctx ? P.max_ctx : n_ctx);
  const int t0 = split * T;
  const int n = min(T, n_ctx - t0);
  float* outp = P.partial + ((size_t(b) * P.heads + h) * P.n_splits + split) * kPart;
  if (n <= 0) {
    for (int i = threadIdx.x; i < kPart; i += kThreads) outp[i] = i == 0 ? -INFINITY : 0.f;
    return;
  }
  const size_t base = ((size_t(b) * P.heads + h) * P.max_ctx + t0) * kD;
  const uint32_t bytes = uint32_t(n) * kD * 2;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_g2s(ks, reinterpret_cast<const __nv_bfloat16*>(P.K) + base, bytes, &bar);
    bulk_g2s(vs, reinterpret_cast<const __nv_bfloat16*>(P.V) + base, bytes, &bar);
  }

  // the query slice of this lane (8 lanes per token, 16 dims each), pre-scaled
  // by scale * log2(e) so that exp2 gives e^s
  const int part = threadIdx.x & 7;
  float q16[16];
  {
    const __nv_bfloat16* qv = reinterpret_cast<const __nv_bfloat16*>(P.q) + (size_t(b) * P.heads + h) * kD + part * 16;
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(qv), q16);
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(qv + 8), q16 + 8);
#pragma unroll
    for (int e = 0; e < 16; ++e) q16[e] *= P.scale * kLog2e;
  }
  if (!mbar_wait_bounded(&bar, 0, P.err)) {
    // the copies did not land in time (recorded): wait once more before leaving
    mbar_wait_bounded(&bar, 0, P.err);
    for (int i = threadIdx.x; i < kPart; i += kThreads) outp[i] = i == 0 ? -INFINITY : 0.f;
    return;
  }

  // scores: 16 tokens per pass
  for (int tk0 = 0; tk0 < n; tk0 += kThreads / 8) {
    const int tk = tk0 + (threadIdx.x >> 3);
    float s = 0.f;
    if (tk < n) {
      float k16[16];
      const __nv_bfloat16* kr = ks + size_t(tk) * kD + part * 16;
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(kr), k16);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(kr + 8), k16 + 8);
#pragma unroll
      for (int e = 0; e < 16; ++e) s = fmaf(q16[e], k16[e], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (part == 0 && tk < n) sc[tk] = s;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int t = threadIdx.x; t < n; t += kThreads) m = fmaxf(m, sc[t]);
  m = block_max(m, scratch);
  float lsum = 0.f;
  for (int t = threadIdx.x; t < n; t += kThreads) {
    const float p = exp2f(sc[t] - m);
    sc[t] = p;
    lsum += p;
  }
  lsum = block_sum(lsum, scratch);  // its barriers also publish sc
  // acc[d] = sum_t p_t V_t[d]: thread d
  const int d = threadIdx.x;
  float a0 = 0.f, a1 = 0.f;
  int t = 0;
  for (; t + 1 < n; t += 2) {
    a0 = fmaf(sc[t], __bfloat162float(vs[size_t(t) * kD + d]), a0);
    a1 = fmaf(sc[t + 1], __bfloat162float(vs[size_t(t + 1) * kD + d]), a1);
  }
  if (t < n) a0 = fmaf(sc[t], __bfloat162float(vs[size_t(t) * kD + d]), a0);
  outp[2 + d] = a0 + a1;
  if (threadIdx.x == 0) {
    outp[0] = m;
    outp[1] = lsum;
  }
}

// Merge the splits of one (batch, head): o = sum_s w_s acc_s / sum_s w_s l_s, w_s = 2^(m_s - M).
__global__ void __launch_bounds__(kThreads) flash_combine_kernel(const __grid_constant__ FlashParams P) {
  const int h = blockIdx.x, b = blockIdx.y;
  __shared__ float sM, sL;
  pdl_launch_dependents();
  pdl_wait();
  int n_ctx = P.seq_lens[b];
  n_ctx = n_ctx < 0 ? 0 : (n_ctx > P.max_ctx ? P.max_ctx : n_ctx);
  const int ns = (n_ctx + P.split_tokens - 1) / P.split_tokens;
  const float* pp = P.partial + (size_t(b) * P.heads + h) * P.n_splits * kPart;
  if (threadIdx.x < 32) {
    float M = -INFINITY;
    for (int s = threadIdx.x; s < ns; s += 32) M = fmaxf(M, pp[s * kPart]);
    M = warp_max(M);
    float L = 0.f;
    for (int s = threadIdx.x; s < ns; s += 32) L += exp2f(pp[s * kPart] - M) * pp[s * kPart + 1];
    L = warp_sum(L);
    if (threadIdx.x == 0) { sM = M; sL = L; }
  }
  __syncthreads();
  const int d = threadIdx.x;
  float A = 0.f;
  for (int s = 0; s < ns; ++s) A += exp2f(pp[s * kPart] - sM) * pp[s * kPart + 2 + d];
  reinterpret_cast<__nv_bfloat16*>(P.out)[(size_t(b) * P.heads + h) * kD + d] =
      __float2bfloat16_rn(sL > 0.f ? A / sL : 0.f);
}

}  // namespace

size_t flash_partial_floats() { return kPart; }

cudaError_t launch_flash(const FlashParams& p, cudaStream_t s) {
  const size_t smem = size_t(p.split_tokens) * kD * 2 * 2 + size_t(p.split_tokens) * 4;
  cudaError_t e = ensure_smem(flash_split_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c1 = {};
  c1.gridDim = dim3(p.n_splits, p.heads, p.batch);
  c1.blockDim = dim3(kThreads);
  c1.dynamicSmemBytes = smem;
  c1.stream = s;
  c1.attrs = attr;
  c1.numAttrs = 1;
  e = cudaLaunchKernelEx(&c1, flash_split_kernel, p);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = c1;
  c2.gridDim = dim3(p.heads, p.batch);
  c2.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&c2, flash_combine_kernel, p);
}

}  // namespace lr
