// Single-query flash-decoding attention over per-head latent K/V caches, sm_100a.
//
// WSVD "Fine-Grained Per-Head SVD": head h keeps latents C_K,h and C_V,h of
// rank r instead of full keys and values; K_t = C_K,t B_K,h and
// V_t = C_V,t B_V,h.  WSVD "Quantization-Aware Training (QAT) en Fused Kernel":
// the reconstruction lives inside the flash-decoding pipeline, never in
// global memory.
//
// Absorbed form (this file's split kernel): for one (batch, head) the query
// is moved into the latent space once, q~ = B_K,h q (an r-vector), so a
// token's score is the r-term dot C_K,t . q~; the latent values are averaged
// with the softmax weights and B_V,h is applied once per (batch, head) by the
// combine kernel.  Work is split over the context (split-K): one CTA per
// (split, head, batch) copies its C_K and C_V chunk into shared memory with
// two bulk asynchronous copies completing on one mbarrier, computes the
// chunk's max, sum and r-dim weighted latent, and writes them; the combine
// kernel merges the splits with the usual log-sum-exp rescaling.
#include "common.cuh"
#include "internal.h"

namespace lr {
namespace {

constexpr int kR = 32;        // latent rank per head
constexpr int kD = 128;       // head dim
constexpr int kThreads = 128;
constexpr int kPart = kR + 2; // m, l, acc[r]
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

__global__ void __launch_bounds__(kThreads) latent_kv_split_kernel(const __grid_constant__ LatentKvParams P) {
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int T = P.split_tokens;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* ck = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* cv = ck + size_t(T) * kR;
  float* sc = reinterpret_cast<float*>(cv + size_t(T) * kR);
  __shared__ float qt[kR];
  __shared__ float scratch[kThreads / 32];
  __shared__ float accs[kThreads / 4][kR + 1];
  __shared__ __align__(8) uint64_t bar;

  pdl_launch_dependents();
  pdl_wait();
  int n_ctx = P.seq_lens[b];
  n_ctx = n_ctx < 0 ? 0 : (n_ctx > P.max_ctx ? P.max_ctx : n_ctx);
  const int t0 = split * T;
  const int n = min(T, n_ctx - t0);
  float* outp = P.partial + ((size_t(b) * P.heads + h) * P.n_splits + split) * kPart;
  if (n <= 0) {
    if (threadIdx.x < kPart) outp[threadIdx.x] = threadIdx.x == 0 ? -INFINITY : 0.f;
    return;
  }
  const size_t base = ((size_t(b) * P.heads + h) * P.max_ctx + t0) * kR;
  const uint32_t bytes = uint32_t(n) * kR * 2;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_g2s(ck, reinterpret_cast<const __nv_bfloat16*>(P.CK) + base, bytes, &bar);
    bulk_g2s(cv, reinterpret_cast<const __nv_bfloat16*>(P.CV) + base, bytes, &bar);
  }

  // q~ = B_K,h q, pre-multiplied by scale * log2(e) so that exp2 gives e^{s}
  {
    const int r = threadIdx.x >> 2, quarter = threadIdx.x & 3;
    const __nv_bfloat16* bk = reinterpret_cast<const __nv_bfloat16*>(P.BK) + (size_t(h) * kR + r) * kD + quarter * 32;
    const __nv_bfloat16* qv = reinterpret_cast<const __nv_bfloat16*>(P.q) + (size_t(b) * P.heads + h) * kD + quarter * 32;
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float w[8], x[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(bk + c * 8), w);
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(qv + c * 8), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(w[e], x[e], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (quarter == 0) qt[r] = s * (P.scale * kLog2e);
  }
  __syncthreads();
  if (!mbar_wait_bounded(&bar, 0, P.err)) {
    // the copies did not land in time (the error word says so); they must not
    // land in a later CTA's shared memory, so wait once more before leaving
    mbar_wait_bounded(&bar, 0, P.err);
    if (threadIdx.x < kPart) outp[threadIdx.x] = threadIdx.x == 0 ? -INFINITY : 0.f;
    return;
  }

  // scores: four lanes per token, eight latent dims each
  const int part = threadIdx.x & 3;
  float q8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) q8[e] = qt[part * 8 + e];
  const int n4 = ((n * 4 + kThreads - 1) / kThreads) * kThreads;
  for (int i = threadIdx.x; i < n4; i += kThreads) {
    const int tk = i >> 2;
    float s = 0.f;
    if (tk < n) {
      float c[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(ck + size_t(tk) * kR + part * 8), c);
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(q8[e], c[e], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (part == 0 && tk < n) sc[tk] = s;
  }
  __syncthreads();
  float m = -INFINITY;
  for (int t = threadIdx.x; t < n; t += kThreads) m = fmaxf(m, sc[t]);
  m = block_max(m, scratch);

  // weights and the weighted latent value
  const int tg = threadIdx.x >> 2;  // token group 0..31
  float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float lsum = 0.f;
  for (int tk = tg; tk < n; tk += kThreads / 4) {
    const float p = exp2f(sc[tk] - m);
    lsum += p;
    float c[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(cv + size_t(tk) * kR + part * 8), c);
#pragma unroll
    for (int e = 0; e < 8; ++e) a8[e] = fmaf(p, c[e], a8[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) accs[tg][part * 8 + e] = a8[e];
  if (part == 0) accs[tg][kR] = lsum;
  __syncthreads();
  if (threadIdx.x < kR + 1) {
    float s = 0.f;
    for (int g = 0; g < kThreads / 4; ++g) s += accs[g][threadIdx.x];
    if (threadIdx.x < kR) outp[2 + threadIdx.x] = s;
    else outp[1] = s;
  }
  if (threadIdx.x == 0) outp[0] = m;
}

// Merge the splits of one (batch, head) and apply B_V,h: o = (sum_s w_s acc_s / sum_s w_s l_s) B_V.
__global__ void __launch_bounds__(kThreads) latent_kv_combine_kernel(const __grid_constant__ LatentKvParams P) {
  const int h = blockIdx.x, b = blockIdx.y;
  __shared__ float at[kR];
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
  if (threadIdx.x < kR) {
    float A = 0.f;
    for (int s = 0; s < ns; ++s) A += exp2f(pp[s * kPart] - sM) * pp[s * kPart + 2 + threadIdx.x];
    at[threadIdx.x] = sL > 0.f ? A / sL : 0.f;
  }
  __syncthreads();
  const int d = threadIdx.x;  // kThreads == kD
  const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(P.BV) + size_t(h) * kR * kD + d;
  float o = 0.f;
#pragma unroll 8
  for (int r = 0; r < kR; ++r) o = fmaf(at[r], __bfloat162float(bv[size_t(r) * kD]), o);
  reinterpret_cast<__nv_bfloat16*>(P.out)[(size_t(b) * P.heads + h) * kD + d] = __float2bfloat16_rn(o);
}

}  // namespace

cudaError_t launch_latent_kv(const LatentKvParams& p, cudaStream_t s) {
  const size_t smem = size_t(p.split_tokens) * kR * 2 * 2 + size_t(p.split_tokens) * 4;
  cudaError_t e = ensure_smem(latent_kv_split_kernel, smem);
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
  e = cudaLaunchKernelEx(&c1, latent_kv_split_kernel, p);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = c1;
  c2.gridDim = dim3(p.heads, p.batch);
  c2.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&c2, latent_kv_combine_kernel, p);
}

}  // namespace lr
