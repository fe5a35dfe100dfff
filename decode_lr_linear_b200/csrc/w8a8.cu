// W8A8 low-rank linear for prefill on tcgen05 tensor cores, sm_100a.
//
// LASER results (W8A8 setting) and WSVD QAT section (weights and activations
// int8): y = (x A) B with int8 activations (one scale per token), int8
// factors (one scale per output channel), int32 accumulation, and the latent
// requantised per token between the two products:
//   acc1 = x_q A_q                   (tcgen05.mma kind::i8, int32 in TMEM)
//   z    = fp32(fp32(acc1 * s_x[t]) * s_A[j]), per-row max |z|   (epilogue 1)
//   s_z  = max|z| / 127, z_q = clamp(rint(z / s_z))               (requant)
//   acc2 = z_q B_q                   (tcgen05.mma kind::i8)
//   y    = bf16(fp32(fp32(acc2 * s_z[t]) * s_B[k]))                (epilogue 2)
// Every fp32 step is one IEEE operation (__fmul_rn, __fdiv_rn, rintf), so the
// codes match an exact emulation bit for bit.
//
// GEMM kernel: one CTA per 128 x 256 output tile.  Warp 0 issues TMA loads of
// 128-byte-swizzled operand tiles into a 4-stage shared-memory ring; warp 1
// allocates the 256-column TMEM accumulator and one elected thread issues
// the MMAs (four K=32 steps per 128-byte k-block), releasing each stage with
// tcgen05.commit; warps 2..5 (one per TMEM lane quarter) wait for the final
// commit, read the accumulator with tcgen05.ld and run the epilogue.  The
// first factor A_q [r, d_in] is K-major (the B operand of GEMM 1); the second
// factor B_q [r, d_out] is N-contiguous, i.e. an MN-major B operand of GEMM 2.
// Every wait is bounded and records a device error instead of hanging.
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace lr {
namespace {

constexpr int kBM = 128;          // tile rows (tokens)
constexpr int kBN = 256;          // tile columns
constexpr int kBK = 128;          // k-block: 128 int8 = one 128-byte swizzle atom row
constexpr int kStages = 4;
constexpr int kThreads = 192;     // 6 warps
constexpr int kATileBytes = kBM * kBK;         // 16 KB
constexpr int kBTileBytes = kBN * kBK;         // 32 KB
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kTmemCols = 256;
constexpr int kEpiStageBytes = 4 * 32 * 33 * 4;  // a 32 x 32 fp32 chunk per epilogue warp (padded rows)

// 2-D int8 tensor [rows, cols] (row stride `ld` bytes), box [box_rows, box_cols],
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
              uint32_t box_cols) {
  return tc::make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rows, cols, ld, box_rows, box_cols,
                         CU_TENSOR_MAP_SWIZZLE_128B);
}

using tc::fence_after;
using tc::fence_before;
using tc::mma_commit;
using tc::mma_i8;
using tc::smem_desc;
using tc::tma_load_2d;
using tc::tmem_ld32;
LR_DEV void tc_fence_before() { fence_before(); }
LR_DEV void tc_fence_after() { fence_after(); }

struct GemmParams {
  int M, N, K;             // tokens, output columns, reduction length
  int b_mn_major;          // 0: B stored [N, K] (K contiguous); 1: B stored [K, N] (N contiguous)
  int mode;                // 0: latent epilogue (z, row max); 1: output epilogue (bf16 y); 2: raw int32 C
  const float* s_row;      // per-token scale (s_x or s_z)
  const float* s_col;      // per-column scale (s_A or s_B)
  float* z;                // mode 0: [M, N] fp32
  unsigned int* amax;      // mode 0: [M] row max |z| (fp32 bits), zero on entry
  __nv_bfloat16* y;        // mode 1: [M, N]
  int32_t* c;              // mode 2: [M, N]
  int* err;
};

__global__ void __launch_bounds__(kThreads, 1) w8a8_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                                                                const __grid_constant__ CUtensorMap mapB,
                                                                const __grid_constant__ GemmParams P) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ __align__(8) uint64_t accum;
  __shared__ uint32_t tmem_slot;
  // operand tiles must start on 1024-byte boundaries (128-byte swizzle atoms)
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
  const int nk = (P.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(&tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();  // the A operand (activations) may come from the preceding kernel
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages, round = kb / kStages;
        if (round > 0 && !mbar_wait_bounded(&empty[s], uint32_t(round - 1) & 1u, P.err)) break;
        const uint32_t a_dst = base + uint32_t(s) * kStageBytes, b_dst = a_dst + kATileBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(a_dst, &mapA, kb * kBK, m0, &full[s]);
        if (!P.b_mn_major) {
          tma_load_2d(b_dst, &mapB, kb * kBK, n0, &full[s]);
        } else {
          tma_load_2d(b_dst, &mapB, n0, kb * kBK, &full[s]);
          tma_load_2d(b_dst + kBK * 128, &mapB, n0 + 128, kb * kBK, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_i8(kBM, kBN, P.b_mn_major != 0);
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kStages, round = kb / kStages;
        if (!mbar_wait_bounded(&full[s], uint32_t(round) & 1u, P.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_base = base + uint32_t(s) * kStageBytes, b_base = a_base + kATileBytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 32; ++kk) {
          const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024);
          const uint64_t bd = P.b_mn_major ? smem_desc(b_base + kk * 32 * 128, kBK * 128, 1024)
                                           : smem_desc(b_base + kk * 32, 16, 1024);
          mma_i8(tmem, ad, bd, idesc, kb > 0 || kk > 0);
        }
        mma_commit(&empty[s]);
      }
      if (ok) mma_commit(&accum);
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31 (one accumulator row per thread).
    // Its per-token scales, and the row maxima it raises, were written by the
    // preceding kernels: every thread that touches them waits for those first.
    pdl_wait();
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    const bool have = mbar_wait_bounded(&accum, 0u, P.err);
    tc_fence_after();
    if (have) {
      // the raw int32 mode has no scales (s_row, s_col are null there)
      const float sr = (P.mode != 2 && row < P.M) ? P.s_row[row] : 0.f;
      float rmax = 0.f;
      // Each 32 x 32 chunk (lane = row) goes through this warp's shared-memory
      // stage, so that global stores are whole 16-byte pieces of rows (a warp
      // instruction covers 4 rows of fp32 or 8 rows of bf16) instead of one
      // partial 32-byte sector per element.
      float* stage = reinterpret_cast<float*>(smem_raw + (base - smem_u32(smem_raw)) + size_t(kStages) * kStageBytes) +
                     q * 32 * 33;
      const bool vec = (P.N % 8) == 0;
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(c * 32), v);
        const int col0 = n0 + c * 32;
        if (col0 >= P.N) continue;
        float f[32];
        if (P.mode == 2) {
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float sc = col0 + i < P.N ? P.s_col[col0 + i] : 0.f;
            f[i] = __fmul_rn(__fmul_rn(__int2float_rn(int(v[i])), sr), sc);
          }
          if (P.mode == 0 && row < P.M) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i < P.N) rmax = fmaxf(rmax, fabsf(f[i]));
          }
        }
        if (vec && col0 + 32 <= P.N) {
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = f[i];
          __syncwarp();
          const int rbase = m0 + q * 32;
          if (P.mode == 1) {
            // 4 lanes per row, 8 bf16 (16 bytes) each; 8 rows per instruction
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int r = it * 8 + (lane >> 2), cc = (lane & 3) * 8;
              if (rbase + r < P.M) {
                const float* sp = stage + r * 33 + cc;
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const __nv_bfloat162 h = __floats2bfloat162_rn(sp[2 * e], sp[2 * e + 1]);
                  ow[e] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(P.y + size_t(rbase + r) * P.N + col0 + cc) = o;
              }
            }
          } else {
            // 8 lanes per row, 4 words (16 bytes) each; 4 rows per instruction
            uint32_t* dst = P.mode == 0 ? reinterpret_cast<uint32_t*>(P.z) : reinterpret_cast<uint32_t*>(P.c);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int r = it * 4 + (lane >> 3), cc = (lane & 7) * 4;
              if (rbase + r < P.M) {
                const float* sp = stage + r * 33 + cc;
                *reinterpret_cast<uint4*>(dst + size_t(rbase + r) * P.N + col0 + cc) =
                    make_uint4(__float_as_uint(sp[0]), __float_as_uint(sp[1]), __float_as_uint(sp[2]),
                               __float_as_uint(sp[3]));
              }
            }
          }
        } else if (row < P.M) {
          // a ragged last chunk: element stores
          for (int i = 0; i < 32; ++i) {
            if (col0 + i >= P.N) break;
            const size_t o = size_t(row) * P.N + col0 + i;
            if (P.mode == 0) P.z[o] = f[i];
            else if (P.mode == 2) P.c[o] = int32_t(__float_as_uint(f[i]));
            else P.y[o] = __float2bfloat16_rn(f[i]);
          }
        }
      }
      if (P.mode == 0 && row < P.M) atomicMax(reinterpret_cast<int*>(P.amax) + row, __float_as_int(rmax));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Per-token requantisation of the latent: s_z = max|z| / 127 (1 for a zero
// row), z_q = clamp(rint(z / s_z), -127, 127); columns r .. rank_pad-1 of z_q
// are zero; the row max is reset to zero for the next call.
__global__ void __launch_bounds__(256) requant_kernel(const float* __restrict__ z, unsigned int* amax, int r,
                                                      int rank_pad, int8_t* __restrict__ zq, float* __restrict__ sz) {
  const int t = blockIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float s_sc;
  __shared__ int s_zero;
  if (threadIdx.x == 0) {
    const float a = __int_as_float(int(amax[t]));
    float sc = __fdiv_rn(a, 127.0f);
    s_zero = sc == 0.0f;
    if (sc == 0.0f) sc = 1.0f;
    s_sc = sc;
    sz[t] = sc;
  }
  __syncthreads();
  const float sc = s_sc;
  const bool zero = s_zero != 0;
  const float* zr = z + size_t(t) * r;
  int8_t* qr = zq + size_t(t) * rank_pad;
  for (int j = threadIdx.x * 4; j < rank_pad; j += blockDim.x * 4) {
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float q = 0.f;
      if (j + e < r && !zero) q = fminf(fmaxf(rintf(__fdiv_rn(zr[j + e], sc)), -127.f), 127.f);
      w |= (uint32_t(int(q)) & 0xffu) << (8 * e);
    }
    *reinterpret_cast<uint32_t*>(qr + j) = w;
  }
  __syncthreads();
  if (threadIdx.x == 0) amax[t] = 0u;
}

cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p, cudaStream_t s) {
  const size_t smem = size_t(kStages) * kStageBytes + 1024 + kEpiStageBytes;
  cudaError_t e = ensure_smem(w8a8_gemm_kernel, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3((p.N + kBN - 1) / kBN, (p.M + kBM - 1) / kBM);
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = smem;
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, w8a8_gemm_kernel, a, b, p);
}

}  // namespace

size_t w8a8_workspace_bytes(int T, int rank) {
  const size_t rp = (size_t(rank) + 127) / 128 * 128;
  const size_t tp = (size_t(T) + 127) / 128 * 128;
  auto ru = [](size_t v) { return (v + 255) / 256 * 256; };
  return ru(size_t(T) * rank * 4) + ru(tp * rp) + ru(tp * 4) + ru(tp * 4);
}

cudaError_t launch_gemm_s8s32(const int8_t* A, const int8_t* B, int b_kn, int M, int N, int K, int32_t* C,
                              int* err, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, K, kBM, kBK)) return cudaErrorInvalidValue;
  if (!b_kn) {
    if (!make_map(&mb, B, N, K, K, kBN, kBK)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&mb, B, K, N, N, kBK, 128)) return cudaErrorInvalidValue;
  }
  GemmParams g;
  std::memset(&g, 0, sizeof(g));
  g.M = M; g.N = N; g.K = K; g.b_mn_major = b_kn; g.mode = 2; g.c = C; g.err = err;
  return launch_gemm(ma, mb, g, s);
}

cudaError_t launch_w8a8(const W8A8Params& p, int /*sm_count*/, cudaStream_t s) {
  CUtensorMap mx, ma, mz, mb;
  if (!make_map(&mx, p.xq, p.T, p.d_in, p.d_in, kBM, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&ma, p.Aq, p.rank, p.d_in, p.d_in, kBN, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&mz, p.zq, p.T, p.rank_pad, p.rank_pad, kBM, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&mb, p.Bq, p.rank, p.d_out, p.d_out, kBK, 128)) return cudaErrorInvalidValue;

  GemmParams g1;
  std::memset(&g1, 0, sizeof(g1));
  g1.M = p.T; g1.N = p.rank; g1.K = p.d_in; g1.b_mn_major = 0; g1.mode = 0;
  g1.s_row = p.sx; g1.s_col = p.sA; g1.z = p.z; g1.amax = p.amax; g1.err = p.err;
  cudaError_t e = launch_gemm(mx, ma, g1, s);
  if (e != cudaSuccess) return e;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(p.T);
  c.blockDim = dim3(256);
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  e = cudaLaunchKernelEx(&c, requant_kernel, static_cast<const float*>(p.z), p.amax, p.rank, p.rank_pad, p.zq, p.sz);
  if (e != cudaSuccess) return e;

  GemmParams g2;
  std::memset(&g2, 0, sizeof(g2));
  g2.M = p.T; g2.N = p.d_out; g2.K = p.rank; g2.b_mn_major = 1; g2.mode = 1;
  g2.s_row = p.sz; g2.s_col = p.sB; g2.y = reinterpret_cast<__nv_bfloat16*>(p.y); g2.err = p.err;
  return launch_gemm(mz, mb, g2, s);
}

}  // namespace lr
