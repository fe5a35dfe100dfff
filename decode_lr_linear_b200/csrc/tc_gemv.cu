// Batched decode of factorised linears on the tcgen05 tensor cores, sm_100a.
//
// Decode at batch b is y = (x A) B with x [b, d_in]: per weight element it is
// b multiply-adds, so beyond a few tokens the CUDA cores cannot keep pace with
// HBM (2 b flop per 2-byte weight at 6.5 TB/s is 6.5 b TFLOP/s).  Here every
// weight byte streams once per call whatever the batch, through the tensor
// cores with the weights as the M operand and the tokens as N ("swap AB"):
//   GEMM 1  z^T [r, N] = A [r, d_in] . x^T       A latent-major = K-major
//   GEMM 2  y^T [d_out, N] = B^T . z^T           B [r, d_out] = MN-major A operand
// (SAES-SVD technical summary and WSVD "Fine-Grained Per-Head SVD": W ~ A B,
// y = (x A) B without forming W.)
//
// One kernel computes one (weights, activations) product as independent units
// of 128 weight rows x one slice of the reduction (split-K, so that every SM
// streams): warp 0 lane 0 streams 128 x 64 weight tiles with tiled copies
// (128-byte swizzle) through a 4-stage ring, all threads stage the unit's
// activations once as the N x K operand (bf16, same swizzle; an fp32 source is
// split into bf16 high and low parts in separate columns, so the product keeps
// fp32 accuracy), warp 1 lane 0 issues tcgen05.mma kind::f16 into a TMEM
// accumulator, and all four warps add the 128 x N partial product into an fp32
// accumulator in L2 (red.global.add.v4.f32).  A finalize kernel turns the
// accumulators into bf16 outputs and zeroes them.  Every wait is bounded and
// records a device error instead of hanging.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace lr {
namespace {

constexpr int kBM = 128;                 // weight rows per unit (TMEM lanes)
constexpr int kKBytes = 128;             // k-block: one 128-byte swizzle row (64 bf16 or 128 int8)
constexpr int kStages = 4;
constexpr int kThreads = 128;
constexpr int kATile = kBM * kKBytes;    // 16 KiB
constexpr size_t kSmemCap = 200 * 1024;
constexpr int kMaxTokens = 64;           // operand rows (tokens, or high and low parts)

// Byte offset of byte `kb` of row n in a K-major, 128-byte-swizzled operand block
// (rows of 128 bytes; the 16-byte chunk index is XORed with row bits 0..2).
LR_DEV uint32_t sw128_offset(int n, int kb) {
  return uint32_t(n) * 128u + uint32_t((((kb >> 4) ^ (n & 7)) << 4) | (kb & 15));
}

LR_DEV int seg_of(const TcGemvParams& P, int unit) {
  int s = 0;
  while (s + 1 < P.nseg && unit >= P.seg[s + 1].unit0) ++s;
  return s;
}

// 32 lanes x 16 columns of 32-bit accumulators; waits for the load.
LR_DEV void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Element e of a unit's activations for token n at reduction index k (0 outside [.., k1)).
LR_DEV void load_act(const TcSeg& g, int n, int k, int k1, int cnt, float* v) {
  if (g.act_kind == 0) {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(g.act) + size_t(n) * g.act_ld + k;
    if (k + cnt <= k1 && cnt == 8) {
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(src), v);
    } else {
      for (int e = 0; e < cnt; ++e) v[e] = k + e < k1 ? __bfloat162float(src[e]) : 0.f;
    }
  } else {
    const float* src = reinterpret_cast<const float*>(g.act) + size_t(k) * g.act_ld + n;
    for (int e = 0; e < cnt; ++e) v[e] = k + e < k1 ? __ldcg(src + size_t(e) * g.act_ld) : 0.f;
  }
}

// Chunk c of a unit's operand (k-block kb, token n, 16-byte chunk kci of the
// 128-byte row): tokens vary fastest for an fp32 [K, ld] source (a warp then
// reads 32 consecutive tokens of one row), reduction chunks vary fastest for a
// bf16 [nb, K] source (a thread reads 16 contiguous bytes).
LR_DEV void chunk_coords(int c, int nh, int act_kind, int* kb, int* n, int* kci) {
  *kb = c / (nh * 8);
  const int rem = c % (nh * 8);
  if (act_kind == 0) {
    *n = rem / 8;
    *kci = rem % 8;
  } else {
    *kci = rem / nh;
    *n = rem % nh;
  }
}

// I8 = false: bf16 weights, kind::f16, bf16 operand rows (fp32 sources as high +
// low parts).  I8 = true: int8 weights, kind::i8, every activation as two int8
// codes with this unit's per-token scales s1 = max|x| / 127 over the unit's
// reduction slice and s2 = s1 / 254: x ~ s1 hi + s2 lo with |error| <= s1 / 508.
template <bool I8>
__global__ void __launch_bounds__(kThreads) tc_gemv_kernel(const __grid_constant__ TcMaps maps,
                                                           const __grid_constant__ TcGemvParams P) {
  constexpr int kKB = I8 ? 128 : 64;     // elements per k-block
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ __align__(8) uint64_t accum;
  __shared__ uint32_t tmem_slot;
  __shared__ float s_scale[2][kMaxTokens];   // I8: per-token scales of the high and low codes
  __shared__ int s_amax[kMaxTokens];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;      // ring: 1024-byte aligned tiles
  unsigned char* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int s = seg_of(P, blockIdx.x);
  const TcSeg& g = P.seg[s];
  const int u = blockIdx.x - g.unit0;
  const int m_tile = u / g.k_splits, ks = u % g.k_splits;
  const int m0 = m_tile * kBM;
  const int k0 = ks * g.kc;
  const int k1 = min(g.K, k0 + g.kc);
  const int nkb = (k1 - k0 + kKB - 1) / kKB;
  const int N = P.N;
  const int nh = P.hilo ? N / 2 : N;          // token rows; with high/low parts, rows nh.. hold the low parts
  const uint32_t act = base + uint32_t(kStages) * kATile;   // nkb blocks of N rows x 128 B
  unsigned char* act_g = gbase + size_t(kStages) * kATile;
  const CUtensorMap* map = &maps.m[s];

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&accum, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < kMaxTokens) s_amax[threadIdx.x] = 0;
  if (warp == 1) tc::tmem_alloc(&tmem_slot, P.tmem_cols);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_launch_dependents();

  // weights are never written by an earlier kernel: the first stages stream before the dependency wait
  auto load_stage = [&](int kb) {
    const int st = kb % kStages;
    const uint32_t dst = base + uint32_t(st) * kATile;
    mbar_arrive_expect_tx(&full[st], kATile);
    if (!g.a_mn_major) {
      tc::tma_load_2d(dst, map, k0 + kb * kKB, m0, &full[st]);
    } else if (I8) {
      tc::tma_load_2d(dst, map, m0, k0 + kb * kKB, &full[st]);
    } else {
      tc::tma_load_2d(dst, map, m0, k0 + kb * kKB, &full[st]);
      tc::tma_load_2d(dst + kATile / 2, map, m0 + kBM / 2, k0 + kb * kKB, &full[st]);
    }
  };
  if (warp == 0 && lane == 0)
    for (int kb = 0; kb < min(nkb, kStages); ++kb) load_stage(kb);

  // ---- the activations of this unit as the N x K operand (zero outside the data) ----
  pdl_wait();
  if constexpr (!I8) {
    const int chunks = nkb * nh * 8;              // 8 consecutive k (16 bytes) of one token
    for (int c = threadIdx.x; c < chunks; c += kThreads) {
      int kb, n, kci;
      chunk_coords(c, nh, g.act_kind, &kb, &n, &kci);
      const int kc8 = kci * 8;
      const int k = k0 + kb * kKB + kc8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (n < P.nb && k < k1) load_act(g, n, k, k1, 8, v);
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        hi[e] = *reinterpret_cast<const uint32_t*>(&h);
        const float2 hf = __bfloat1622float2(h);
        const __nv_bfloat162 l = __floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
        lo[e] = *reinterpret_cast<const uint32_t*>(&l);
      }
      unsigned char* blk = act_g + size_t(kb) * N * 128;
      *reinterpret_cast<uint4*>(blk + sw128_offset(n, kc8 * 2)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      if (P.hilo) *reinterpret_cast<uint4*>(blk + sw128_offset(nh + n, kc8 * 2)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  } else {
    // pass 1: per-token max |x| over the unit's slice
    const int chunks = nkb * nh * 8;              // 16 consecutive k (16 codes) of one token
    for (int c = threadIdx.x; c < chunks; c += kThreads) {
      int kb, n, kci;
      chunk_coords(c, nh, g.act_kind, &kb, &n, &kci);
      const int k = k0 + kb * kKB + kci * 16;
      if (n < P.nb && k < k1) {
        float v[16];
        load_act(g, n, k, k1, 8, v);
        load_act(g, n, k + 8, k1, 8, v + 8);
        float m = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
        atomicMax(&s_amax[n], __float_as_int(m));
      }
    }
    __syncthreads();
    if (threadIdx.x < nh) {
      const float a = __int_as_float(s_amax[threadIdx.x]);
      const float s1 = a > 0.f ? a / 127.f : 1.f;
      s_scale[0][threadIdx.x] = s1;
      s_scale[1][threadIdx.x] = s1 / 254.f;
    }
    __syncthreads();
    // pass 2: the codes
    for (int c = threadIdx.x; c < chunks; c += kThreads) {
      int kb, n, kci;
      chunk_coords(c, nh, g.act_kind, &kb, &n, &kci);
      const int kc = kci * 16, k = k0 + kb * kKB + kc;
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = 0.f;
      if (n < P.nb && k < k1) {
        load_act(g, n, k, k1, 8, v);
        load_act(g, n, k + 8, k1, 8, v + 8);
      }
      const float s1 = s_scale[0][n], s2 = s_scale[1][n];
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t ph = 0, pl = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = v[4 * w + e];
          const float qh = fminf(fmaxf(rintf(x / s1), -127.f), 127.f);
          const float ql = fminf(fmaxf(rintf((x - qh * s1) / s2), -127.f), 127.f);
          ph |= (uint32_t(int(qh)) & 0xffu) << (8 * e);
          pl |= (uint32_t(int(ql)) & 0xffu) << (8 * e);
        }
        hi[w] = ph;
        lo[w] = pl;
      }
      unsigned char* blk = act_g + size_t(kb) * N * 128;
      *reinterpret_cast<uint4*>(blk + sw128_offset(n, kc)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(blk + sw128_offset(nh + n, kc)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  fence_proxy_async();  // generic-proxy writes of the operand before the tensor cores read it
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = kStages; kb < nkb; ++kb) {
        const int st = kb % kStages;
        if (!mbar_wait_bounded(&empty[st], uint32_t(kb / kStages - 1) & 1u, P.err)) break;
        load_stage(kb);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = I8 ? tc::idesc_i8(kBM, N, false, g.a_mn_major != 0)
                                : tc::idesc_bf16(kBM, N, g.a_mn_major != 0, false);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int st = kb % kStages;
        if (!mbar_wait_bounded(&full[st], uint32_t(kb / kStages) & 1u, P.err)) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t a_base = base + uint32_t(st) * kATile;
        const uint32_t b_base = act + uint32_t(kb) * uint32_t(N) * 128u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {   // four MMAs of 32 bytes of reduction each
          const int kr = I8 ? 32 : 16;     // reduction elements per MMA
          const uint64_t ad = g.a_mn_major ? tc::smem_desc(a_base + kk * kr * 128, kATile / 2, 1024)
                                           : tc::smem_desc(a_base + kk * 32, 16, 1024);
          const uint64_t bd = tc::smem_desc(b_base + kk * 32, 16, 1024);
          if constexpr (I8) tc::mma_i8(tmem, ad, bd, idesc, kb > 0 || kk > 0);
          else tc::mma_f16(tmem, ad, bd, idesc, kb > 0 || kk > 0);
        }
        tc::mma_commit(&empty[st]);
      }
      if (ok) tc::mma_commit(&accum);
    }
  }
  __syncwarp();  // roles end: every warp converges before the warp-wide tensor-memory loads
  // ---- epilogue: lane = weight row, N accumulator columns; add into the fp32 accumulator ----
  const bool have = mbar_wait_bounded(&accum, 0u, P.err);
  tc::fence_after();
  if (have) {
    const int row = m0 + warp * 32 + lane;
    const float rs = (g.row_scale && row < g.M) ? load_scale(g.row_scale, row, g.row_scale_f16 != 0) : 1.f;
    for (int c0 = 0; c0 < nh; c0 += 16) {
      uint32_t v[16], w[16];
      tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(c0), v);
      if (P.hilo) tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(nh + c0), w);
      if (row < g.M) {
        float* out = g.out + size_t(row) * g.out_ld + c0;
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          if (c0 + e < P.nb) {
            float a[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if constexpr (I8) {
                const int n = c0 + e + q;
                a[q] = (float(int(v[e + q])) * s_scale[0][n] + float(int(w[e + q])) * s_scale[1][n]) * rs;
              } else {
                a[q] = (__uint_as_float(v[e + q]) + (P.hilo ? __uint_as_float(w[e + q]) : 0.f)) * rs;
              }
            }
            red_add_f4(out + e, a[0], a[1], a[2], a[3]);
          }
        }
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, P.tmem_cols);
  }
}

// y[n][m] = bf16(acc[m][n]) for every target; then zero the listed accumulator regions.
__global__ void __launch_bounds__(256) tc_finalize_kernel(const __grid_constant__ TcFinalizeParams F) {
  pdl_launch_dependents();
  pdl_wait();
  const int stride = gridDim.x * blockDim.x;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  for (int t = 0; t < F.nt; ++t) {
    const TcFinalTarget& f = F.t[t];
    for (int m = tid; m < f.M; m += stride) {
      float* a = const_cast<float*>(f.acc) + size_t(m) * F.ld;
      __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(f.y) + m;
      for (int n = 0; n < F.nb; ++n) {
        y[size_t(n) * f.M] = __float2bfloat16_rn(__ldcg(a + n));
        if (F.zero_targets) __stcg(a + n, 0.f);   // read and cleared by the same thread
      }
    }
  }
  for (int z = 0; z < F.nz; ++z) {
    float4* p = reinterpret_cast<float4*>(F.zero[z]);
    const size_t n4 = F.zero_floats[z] / 4;
    for (size_t i = tid; i < n4; i += stride) __stcg(p + i, make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

// SwiGLU of the hybrid FFN between its two tensor-core products:
// h[c][n] = silu(g) u for channel c, from the gate/up accumulators of the
// low-rank channels (c < n_lr, rows 2c and 2c+1 of gu) or of the dense ones
// (rows 2(c - n_lr), +1 of dd); each accumulator element is read and cleared by
// the thread that uses it.  Then the listed region (the latent accumulator,
// consumed by the preceding product) is zeroed.
__global__ void __launch_bounds__(256) tc_swiglu_kernel(const __grid_constant__ TcSwigluParams S) {
  pdl_launch_dependents();
  pdl_wait();
  const int stride = gridDim.x * blockDim.x;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int inter = S.n_lr + S.n_dense;
  for (int i = tid; i < inter * S.nb; i += stride) {
    const int c = i / S.nb, n = i % S.nb;
    float* src = c < S.n_lr ? S.gu + size_t(2 * c) * S.cols : S.dd + size_t(2 * (c - S.n_lr)) * S.cols;
    const float gt = __ldcg(src + n), up = __ldcg(src + S.cols + n);
    __stcg(src + n, 0.f);
    __stcg(src + S.cols + n, 0.f);
    S.h[size_t(c) * S.cols + n] = silu(gt) * up;
  }
  if (S.zero) {
    float4* p = reinterpret_cast<float4*>(S.zero);
    for (size_t i = tid; i < S.zero_floats / 4; i += stride) __stcg(p + i, make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

int kb_elems(bool i8) { return i8 ? 128 : 64; }

}  // namespace

int tc_gemv_kc(int K, int k_splits, bool i8) {
  const int e = kb_elems(i8);
  return ((K + k_splits - 1) / k_splits + e - 1) / e * e;
}

size_t tc_gemv_smem(int kc, int N, bool i8) {
  return size_t(kStages) * kATile + size_t(kc / kb_elems(i8)) * N * 128 + 1024;
}

bool tc_gemv_fits(int kc, int N, bool i8) { return N <= kMaxTokens && tc_gemv_smem(kc, N, i8) <= kSmemCap; }

bool tc_make_weight_map(CUtensorMap* m, const void* W, int rows, int cols, int a_mn_major, bool i8) {
  // K-major: W [rows = M, cols = K], box 128 rows x one k-block; MN-major: W [rows = K,
  // cols = M], box one k-block of rows x 128 bytes of columns
  const int e = kb_elems(i8);
  const size_t es = i8 ? 1 : 2;
  return tc::make_map_2d(m, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, uint64_t(rows),
                         uint64_t(cols), uint64_t(cols) * es, a_mn_major ? e : kBM, a_mn_major ? 128 / es : e,
                         CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_tc_gemv(const TcMaps& maps, const TcGemvParams& p, bool i8, cudaStream_t s) {
  int units = 0, kc_max = 0;
  for (int i = 0; i < p.nseg; ++i) {
    units += p.seg[i].m_tiles * p.seg[i].k_splits;
    kc_max = std::max(kc_max, p.seg[i].kc);
  }
  if (!tc_gemv_fits(kc_max, p.N, i8) || (i8 && !p.hilo)) return cudaErrorInvalidValue;
  const size_t smem = tc_gemv_smem(kc_max, p.N, i8);
  auto kern = i8 ? tc_gemv_kernel<true> : tc_gemv_kernel<false>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(units);
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = smem;
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, kern, maps, p);
}

cudaError_t launch_tc_swiglu(const TcSwigluParams& p, int sm_count, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(sm_count);
  c.blockDim = dim3(256);
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, tc_swiglu_kernel, p);
}

cudaError_t launch_tc_finalize(const TcFinalizeParams& f, int sm_count, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(sm_count);
  c.blockDim = dim3(256);
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, tc_finalize_kernel, f);
}

}  // namespace lr
