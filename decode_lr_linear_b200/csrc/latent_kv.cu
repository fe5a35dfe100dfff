// Single-query flash-decoding attention over per-head latent K/V caches, sm_100a.
//
// WSVD "Fine-Grained Per-Head SVD": head h keeps latents C_K,h and C_V,h of
// rank r instead of full keys and values; K_t = C_K,t B_K,h and
// V_t = C_V,t B_V,h.  WSVD "Quantization-Aware Training (QAT) en Fused Kernel":
// the reconstruction lives inside the flash-decoding pipeline, never in
// global memory.
//
// Absorbed form: for one (batch, head) the query is moved into the latent
// space once, q~ = B_K,h q (an r-vector, one small kernel per call), so a
// token's score is the r-term dot C_K,t . q~; the latent values are averaged
// with the softmax weights and B_V,h is applied once per (batch, head) by the
// combine kernel.  Work is split over the context (split-K): one CTA per
// (split, head, batch) copies its C_K and C_V chunk into shared memory with
// two bulk asynchronous copies completing on one mbarrier, computes the
// chunk's max, sum and r-dim weighted latent, and writes them; the combine
// kernel merges the splits with the usual log-sum-exp rescaling.  The caches
// are bf16, or int8 with one scale per (batch, head, position) (LASER results:
// the KV cache in 8 bits), applied to the token's score and value weight.
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

// q~ = B_K,h q * scale * log2(e), once per (batch, head) (grid heads x batch):
// the split kernels then read 32 floats instead of recomputing it from B_K.
__global__ void __launch_bounds__(kThreads) latent_kv_qproj_kernel(const __grid_constant__ LatentKvParams P) {
  const int h = blockIdx.x, b = blockIdx.y;
  pdl_launch_dependents();
  pdl_wait();
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
  if (quarter == 0) P.qt[(size_t(b) * P.heads + h) * kR + r] = s * (P.scale * kLog2e);
}

// Eight consecutive latent values of a cached token as fp32 (bf16 codes, or
// int8 codes whose per-position scale is applied by the caller).
template <bool Q8> struct CacheRow;
template <> struct CacheRow<false> {
  using T = __nv_bfloat16;
  static constexpr int kBytes = kR * 2;
  LR_DEV static void load8(const T* row, int part, float* f) {
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + part * 8), f);
  }
};
template <> struct CacheRow<true> {
  using T = int8_t;
  static constexpr int kBytes = kR;
  LR_DEV static void load8(const T* row, int part, float* f) {
    i8x8_to_f32(*reinterpret_cast<const uint2*>(row + part * 8), f);
  }
};

LR_DEV float cache_scale(const void* s, size_t i, bool f16) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(s)[i]) : reinterpret_cast<const float*>(s)[i];
}

template <bool Q8>
__global__ void __launch_bounds__(kThreads) latent_kv_split_kernel(const __grid_constant__ LatentKvParams P) {
  using CR = CacheRow<Q8>;
  using T = typename CR::T;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int TS = P.split_tokens;
  extern __shared__ __align__(128) unsigned char smem[];
  T* ck = reinterpret_cast<T*>(smem);
  T* cv = ck + size_t(TS) * kR;
  float* sc = reinterpret_cast<float*>(cv + size_t(TS) * kR);
  float* sks = sc + TS;   // int8 caches: per-position key scales
  float* svs = sks + TS;  // and value scales
  __shared__ float scratch[kThreads / 32];
  __shared__ float accs[kThreads / 4][kR + 1];
  __shared__ __align__(8) uint64_t bar;

  pdl_launch_dependents();
  pdl_wait();
  int n_ctx = P.seq_lens[b];
  n_ctx = n_ctx < 0 ? 0 : (n_ctx > P.max_ctx ? P.max_ctx : n_ctx);
  const int t0 = split * TS;
  const int n = min(TS, n_ctx - t0);
  float* outp = P.partial + ((size_t(b) * P.heads + h) * P.n_splits + split) * kPart;
  if (n <= 0) {
    if (threadIdx.x < kPart) outp[threadIdx.x] = threadIdx.x == 0 ? -INFINITY : 0.f;
    return;
  }
  const size_t row0 = (size_t(b) * P.heads + h) * P.max_ctx + t0;
  const uint32_t bytes = uint32_t(n) * CR::kBytes;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, 2 * bytes);
    bulk_g2s(ck, reinterpret_cast<const T*>(P.CK) + row0 * kR, bytes, &bar);
    bulk_g2s(cv, reinterpret_cast<const T*>(P.CV) + row0 * kR, bytes, &bar);
  }
  // four lanes per token, eight latent dims each: q~ slice in registers
  const int part = threadIdx.x & 3;
  float q8[8];
  {
    const float* qt = P.qt + (size_t(b) * P.heads + h) * kR + part * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) q8[e] = qt[e];
  }
  const bool f16 = P.cache_scale_f16 != 0;
  if constexpr (Q8) {
    // independent loads, in flight together with the bulk copies
    for (int t = threadIdx.x; t < n; t += kThreads) {
      sks[t] = cache_scale(P.sK, row0 + t, f16);
      svs[t] = cache_scale(P.sV, row0 + t, f16);
    }
    __syncthreads();
  }
  if (!mbar_wait_bounded(&bar, 0, P.err)) {
    // the copies did not land in time (recorded): wait once more before leaving
    mbar_wait_bounded(&bar, 0, P.err);
    if (threadIdx.x < kPart) outp[threadIdx.x] = threadIdx.x == 0 ? -INFINITY : 0.f;
    return;
  }

  // scores
  const int n4 = ((n * 4 + kThreads - 1) / kThreads) * kThreads;
  for (int i = threadIdx.x; i < n4; i += kThreads) {
    const int tk = i >> 2;
    float s = 0.f;
    if (tk < n) {
      float c[8];
      CR::load8(ck + size_t(tk) * kR, part, c);
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(q8[e], c[e], s);
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (part == 0 && tk < n) {
      if constexpr (Q8) s *= sks[tk];
      sc[tk] = s;
    }
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
    float w = p;
    if constexpr (Q8) w *= svs[tk];
    float c[8];
    CR::load8(cv + size_t(tk) * kR, part, c);
#pragma unroll
    for (int e = 0; e < 8; ++e) a8[e] = fmaf(w, c[e], a8[e]);
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
  const bool q8 = p.cache_q8 != 0;
  const size_t row = q8 ? kR : kR * 2;
  const size_t smem = size_t(p.split_tokens) * row * 2 + size_t(p.split_tokens) * 4 * (q8 ? 3 : 1);
  const void* split_fn = q8 ? reinterpret_cast<const void*>(latent_kv_split_kernel<true>)
                            : reinterpret_cast<const void*>(latent_kv_split_kernel<false>);
  cudaError_t e = ensure_smem_fn(split_fn, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c0 = {};
  c0.gridDim = dim3(p.heads, p.batch);
  c0.blockDim = dim3(kThreads);
  c0.stream = s;
  c0.attrs = attr;
  c0.numAttrs = 1;
  e = cudaLaunchKernelEx(&c0, latent_kv_qproj_kernel, p);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c1 = c0;
  c1.gridDim = dim3(p.n_splits, p.heads, p.batch);
  c1.dynamicSmemBytes = smem;
  e = q8 ? cudaLaunchKernelEx(&c1, latent_kv_split_kernel<true>, p)
         : cudaLaunchKernelEx(&c1, latent_kv_split_kernel<false>, p);
  if (e != cudaSuccess) return e;
  return launch_latent_kv_combine(p, s);
}

cudaError_t launch_latent_kv_combine(const LatentKvParams& p, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(p.heads, p.batch);
  c.blockDim = dim3(kThreads);
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, latent_kv_combine_kernel, p);
}

}  // namespace lr
