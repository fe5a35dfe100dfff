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
// fp32 accuracy; for int8 weights, two int8 codes per value with scales from
// the slice's own per-token maxima), warp 1 lane 0 issues tcgen05.mma into a
// TMEM accumulator, and all four warps add the 128 x N partial product into
// an fp32 accumulator in L2.  For a few tokens the hybrid FFN's SwiGLU is
// evaluated while its down projection stages h from the gate/up accumulators
// (no kernel of its own); for more, a SwiGLU kernel writes h once, since every
// tile of the down projection would repeat it.  A finalize kernel turns the accumulators into bf16
// outputs and zeroes them.  Every wait is bounded and records a device error
// instead of hanging.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace lr {
namespace {

constexpr int kBM = 128;                 // weight rows per unit (TMEM lanes)
constexpr int kKBytes = 128;             // k-block: one 128-byte swizzle row (64 bf16 or 128 int8)
constexpr int kStages = 4;                // ring depth, 3 where that keeps two CTAs per SM
constexpr size_t kTwoPerSm = 112 * 1024;  // dynamic shared memory per CTA with two CTAs per SM
constexpr int kThreads = 256;          // 8 warps: all stage the activations; two per TMEM lane quarter in the epilogue
constexpr int kATile = kBM * kKBytes;    // 16 KiB
constexpr size_t kSmemCap = 200 * 1024;
constexpr int kMaxTokens = 64;           // operand rows (tokens, or high and low parts)
constexpr int kSwigluChunk = 1024;       // channels per SwiGLU CTA

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

// Eight activations of token n from reduction index k (0 at k >= k1).  Both
// sources are token-major: bf16 [nb, K] or fp32 [nb, K], row stride act_ld
// (a multiple of 8 elements, so k..k+7 is one aligned 16- or 32-byte piece).
LR_DEV void load_act8(const TcSeg& g, int n, int k, int k1, float* v) {
  if (g.act_kind == 0) {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(g.act) + size_t(n) * g.act_ld + k;
    if (k + 8 <= k1) {
      bf16x8_to_f32(ld_cg_u4(src), v);
    } else {
      for (int e = 0; e < 8; ++e) v[e] = k + e < k1 ? __bfloat162float(src[e]) : 0.f;
    }
  } else {
    const float* src = reinterpret_cast<const float*>(g.act) + size_t(n) * g.act_ld + k;
    if (k + 8 <= k1) {
      const float4 a = ld_cg_f4(src), b = ld_cg_f4(src + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      for (int e = 0; e < 8; ++e) v[e] = k + e < k1 ? __ldcg(src + e) : 0.f;
    }
  }
}

// kPer activations of token n from reduction index k (0 at k >= k1), any
// source kind; k is a multiple of 8.
template <int kPer>
LR_DEV void fetch_act(const TcSeg& g, int n, int k, int k1, float* v) {
  if (g.act_kind != 2) {
#pragma unroll
    for (int h = 0; h < kPer; h += 8) load_act8(g, n, k + h, k1, v + h);
    return;
  }
  const float* gu = reinterpret_cast<const float*>(g.act) + size_t(n) * g.act_ld;
  const float* dd = g.act2 + size_t(n) * g.act2_ld;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int c = k + e;
    v[e] = 0.f;
    if (c < k1) {
      const float2 p = __ldcg(reinterpret_cast<const float2*>(c < g.n_lr ? gu + 2 * c : dd + 2 * (c - g.n_lr)));
      v[e] = silu(p.x) * p.y;
    }
  }
}

LR_DEV void finalize_part(const TcFinalizeParams& F, int part, int parts, int t, int nt);

// I8 = false: bf16 weights, kind::f16, bf16 operand rows (fp32 sources as high +
// low parts).  I8 = true: int8 weights, kind::i8, every activation as two int8
// codes with per-token scales s1 = max|x| / 127 over the unit's slice of the
// token's input and s2 = s1 / 254: x ~ s1 hi + s2 lo with |error| <= s1 / 508.
// Each unit converts its int32 partial product with its own scales before
// adding it into the fp32 accumulator, so no scale is shared between units.
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
  __shared__ float s_inv[2][kMaxTokens];     // and their reciprocals (codes by multiplication)
  __shared__ unsigned int s_amax[kMaxTokens];  // I8: per-token max |x| over the slice (fp32 bits)
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
  const int stages = P.stages;
  const uint32_t act = base + uint32_t(stages) * kATile;   // nkb blocks of N rows x 128 B
  unsigned char* act_g = gbase + size_t(stages) * kATile;
  const CUtensorMap* map = &maps.m[s];

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, P.tmem_cols);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_launch_dependents();

  // weights are never written by an earlier kernel: the first stages stream before the dependency wait
  auto load_stage = [&](int kb) {
    const int st = kb % stages;
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
    for (int kb = 0; kb < min(nkb, stages); ++kb) load_stage(kb);

  // ---- the activations of this unit as the N x K operand (zero outside the data) ----
  pdl_wait();
  // the preceding step's finalize, spread over this launch's units (outputs and clearing)
  if (P.pre.nt > 0 || P.pre.nz > 0) finalize_part(P.pre, blockIdx.x, gridDim.x, threadIdx.x, kThreads);
  {
    // Token n's 16-byte piece kci of k-block kb is chunk c = (kb * nb + n) * 8 + kci
    // (the reduction index varies fastest, so neighbouring threads load
    // neighbouring bytes).  Only real tokens are staged: the accumulator
    // columns of padding tokens are never read.  Pieces past k1 are zero (the
    // weights there are zero-filled, and zero times stale bytes could be NaN).
    // Each thread issues the loads of up to kHold pieces before it uses any.
    constexpr int kPer = I8 ? 16 : 8;   // activations per 16-byte piece of the operand row
    constexpr int kHold = 4;
    const int vchunks = nkb * P.nb * 8;
    const int step = kHold * kThreads;
    float v[kHold][kPer];
    auto piece = [&](int c, int& kb, int& n, int& k) {
      kb = c / (P.nb * 8);
      const int rem = c - kb * P.nb * 8;
      n = rem >> 3;
      k = k0 + kb * kKB + (rem & 7) * kPer;
    };
    auto store = [&](int kb, int n, int kci, const uint32_t* hi, const uint32_t* lo) {
      unsigned char* blk = act_g + size_t(kb) * N * 128;
      *reinterpret_cast<uint4*>(blk + sw128_offset(n, kci * 16)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      if (P.hilo)
        *reinterpret_cast<uint4*>(blk + sw128_offset(nh + n, kci * 16)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    };
    if constexpr (I8) {
      if (threadIdx.x < kMaxTokens) s_amax[threadIdx.x] = 0u;
      __syncthreads();
      // pass 1: the slice's per-token maxima
      for (int c0 = 0; c0 < vchunks; c0 += step) {
#pragma unroll
        for (int i = 0; i < kHold; ++i) {
          const int c = c0 + i * kThreads + threadIdx.x;
          if (c < vchunks) {
            int kb, n, k;
            piece(c, kb, n, k);
            fetch_act<kPer>(g, n, k, k1, v[i]);
          }
        }
#pragma unroll
        for (int i = 0; i < kHold; ++i) {
          const int c = c0 + i * kThreads + threadIdx.x;
          if (c < vchunks) {
            float m = 0.f;
#pragma unroll
            for (int e = 0; e < kPer; ++e) m = fmaxf(m, fabsf(v[i][e]));
            atomicMax(&s_amax[(c % (P.nb * 8)) >> 3], __float_as_uint(m));
          }
        }
      }
      __syncthreads();
      if (threadIdx.x < P.nb) {
        const float a = __uint_as_float(s_amax[threadIdx.x]);
        const float s1 = a > 0.f ? a / 127.f : 1.f;
        s_scale[0][threadIdx.x] = s1;
        s_scale[1][threadIdx.x] = s1 / 254.f;
        s_inv[0][threadIdx.x] = 1.f / s1;
        s_inv[1][threadIdx.x] = 254.f / s1;
      }
      __syncthreads();
      // pass 2: int8 high and low codes; the registers still hold the pieces only when pass 1
      // took a single round, otherwise every round reads its pieces again
      const bool held = vchunks <= step;
      for (int c0 = 0; c0 < vchunks; c0 += step) {
        if (!held) {
#pragma unroll
          for (int i = 0; i < kHold; ++i) {
            const int c = c0 + i * kThreads + threadIdx.x;
            if (c < vchunks) {
              int kb, n, k;
              piece(c, kb, n, k);
              fetch_act<kPer>(g, n, k, k1, v[i]);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < kHold; ++i) {
          const int c = c0 + i * kThreads + threadIdx.x;
          if (c < vchunks) {
            int kb, n, k;
            piece(c, kb, n, k);
            // codes by multiplication with the reciprocal scales: any integer pair whose error
            // against x stays within s2 / 2 plus rounding; the epilogue uses s1, s2 themselves
            const float s1 = s_scale[0][n], i1 = s_inv[0][n], i2 = s_inv[1][n];
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              uint32_t ph = 0, pl = 0;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float x = v[i][4 * w + e];
                const float qh = fminf(fmaxf(rintf(x * i1), -127.f), 127.f);
                const float ql = fminf(fmaxf(rintf(fmaf(-qh, s1, x) * i2), -127.f), 127.f);
                ph |= (uint32_t(int(qh)) & 0xffu) << (8 * e);
                pl |= (uint32_t(int(ql)) & 0xffu) << (8 * e);
              }
              hi[w] = ph;
              lo[w] = pl;
            }
            store(kb, n, (c & 7), hi, lo);
          }
        }
      }
    } else {
      for (int c0 = 0; c0 < vchunks; c0 += step) {
#pragma unroll
        for (int i = 0; i < kHold; ++i) {
          const int c = c0 + i * kThreads + threadIdx.x;
          if (c < vchunks) {
            int kb, n, k;
            piece(c, kb, n, k);
            fetch_act<kPer>(g, n, k, k1, v[i]);
          }
        }
#pragma unroll
        for (int i = 0; i < kHold; ++i) {
          const int c = c0 + i * kThreads + threadIdx.x;
          if (c < vchunks) {
            int kb, n, k;
            piece(c, kb, n, k);
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 h = __floats2bfloat162_rn(v[i][2 * e], v[i][2 * e + 1]);
              hi[e] = *reinterpret_cast<const uint32_t*>(&h);
              const float2 hf = __bfloat1622float2(h);
              const __nv_bfloat162 l = __floats2bfloat162_rn(v[i][2 * e] - hf.x, v[i][2 * e + 1] - hf.y);
              lo[e] = *reinterpret_cast<const uint32_t*>(&l);
            }
            store(kb, n, (c & 7), hi, lo);
          }
        }
      }
    }
  }
  fence_proxy_async();  // generic-proxy writes of the operand before the tensor cores read it
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = stages; kb < nkb; ++kb) {
        const int st = kb % stages;
        if (!mbar_wait_bounded(&empty[st], uint32_t(kb / stages - 1) & 1u, P.err)) break;
        load_stage(kb);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = I8 ? tc::idesc_i8(kBM, N, false, g.a_mn_major != 0)
                                : tc::idesc_bf16(kBM, N, g.a_mn_major != 0, false);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int st = kb % stages;
        if (!mbar_wait_bounded(&full[st], uint32_t(kb / stages) & 1u, P.err)) {
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
  // warps w and w + 4 read TMEM lanes 32 (w % 4) .. + 31 and take alternate groups of 16 columns
  const bool have = mbar_wait_bounded(&accum, 0u, P.err);
  tc::fence_after();
  if (have) {
    const int q = warp & 3;
    const int row = m0 + q * 32 + lane;
    const float rs = (g.row_scale && row < g.M) ? load_scale(g.row_scale, row, g.row_scale_f16 != 0) : 1.f;
    for (int c0 = (warp >> 2) * 16; c0 < nh; c0 += 32) {
      uint32_t v[16], w[16];
      tmem_ld16(tmem + (uint32_t(q * 32) << 16) + uint32_t(c0), v);
      if (P.hilo) tmem_ld16(tmem + (uint32_t(q * 32) << 16) + uint32_t(nh + c0), w);
      if (row < g.M) {
        // token-major accumulator: out[n * out_ld + row]; a warp's 32 rows are contiguous for each n
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int n = c0 + e;
          if (n < P.nb) {
            float a;
            if constexpr (I8) {
              a = (float(int(v[e])) * s_scale[0][n] + float(int(w[e])) * s_scale[1][n]) * rs;
            } else {
              a = (__uint_as_float(v[e]) + (P.hilo ? __uint_as_float(w[e]) : 0.f)) * rs;
            }
            atomicAdd(g.out + size_t(n) * g.out_ld + row, a);
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
// Finalize work for part `part` of `parts` (each part takes its share of every
// target's 8-float chunks and of every zero region), thread `t` of `nt` within
// the part: y[n][m] = bf16(acc[n][m]) for each target (token-major, M a
// multiple of 8), clearing what it read when zero_targets is set; then the
// zero regions, which no part reads.
LR_DEV void finalize_part(const TcFinalizeParams& F, int part, int parts, int t, int nt) {
  for (int q = 0; q < F.nt; ++q) {
    const TcFinalTarget& f = F.t[q];
    float* a = const_cast<float*>(f.acc);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(f.y);
    const long long n8 = (long long)F.nb * f.M / 8;
    const long long c0 = n8 * part / parts, c1 = n8 * (part + 1) / parts;
    for (long long i = c0 + t; i < c1; i += nt) {
      const float4 v0 = ld_cg_f4(a + 8 * i), v1 = ld_cg_f4(a + 8 * i + 4);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
      const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        ow[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(y + 8 * i) = o;
      if (F.zero_targets) {   // read and cleared by the same thread
        st_cg_f4(a + 8 * i, make_float4(0.f, 0.f, 0.f, 0.f));
        st_cg_f4(a + 8 * i + 4, make_float4(0.f, 0.f, 0.f, 0.f));
      }
    }
  }
  for (int z = 0; z < F.nz; ++z) {
    float4* p = reinterpret_cast<float4*>(F.zero[z]);
    const long long n4 = (long long)(F.zero_floats[z] / 4);
    const long long c0 = n4 * part / parts, c1 = n4 * (part + 1) / parts;
    for (long long i = c0 + t; i < c1; i += nt) __stcg(p + i, make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

__global__ void __launch_bounds__(256) tc_finalize_kernel(const __grid_constant__ TcFinalizeParams F) {
  pdl_launch_dependents();
  pdl_wait();
  finalize_part(F, blockIdx.x, gridDim.x, threadIdx.x, blockDim.x);
}

// SwiGLU of the hybrid FFN between its tensor-core products, for passes of
// more tokens than the down projection evaluates while staging (token-major
// accumulators), grid (tokens, channel chunks): h[n][c] = silu(g) u for
// channel c, from the gate/up pair of the low-rank channels (c < n_lr:
// gu[n][2c], gu[n][2c+1]) or of the dense ones (dd[n][2(c - n_lr)], +1); each
// accumulator element is read and cleared by the thread that uses it, and the
// chunk-0 CTA zeroes the token's latent row (consumed by the preceding product).
__global__ void __launch_bounds__(256) tc_swiglu_kernel(const __grid_constant__ TcSwigluParams S) {
  pdl_launch_dependents();
  pdl_wait();
  const int n = blockIdx.x;
  const int inter = S.n_lr + S.n_dense;
  float* gu = S.gu + size_t(n) * 2 * S.n_lr;
  float* dd = S.dd + size_t(n) * 2 * S.n_dense;
  const int c0 = blockIdx.y * kSwigluChunk, c1 = min(inter, c0 + kSwigluChunk);
  for (int c = c0 + int(threadIdx.x); c < c1; c += blockDim.x) {
    float2* src = reinterpret_cast<float2*>(c < S.n_lr ? gu + 2 * c : dd + 2 * (c - S.n_lr));
    const float2 gv = __ldcg(src);
    __stcg(src, make_float2(0.f, 0.f));
    S.h[size_t(n) * S.h_ld + c] = silu(gv.x) * gv.y;
  }
  if (S.zero && blockIdx.y == 0) {
    float* z = S.zero + size_t(n) * S.zero_row;
    for (int i = threadIdx.x; i < S.zero_row; i += blockDim.x) __stcg(z + i, 0.f);
  }
}

// The latent producer's scatter after its tensor-core product: token n's row of
// the token-major fp32 accumulator [nb, 2 H r] (keys then values, head-major)
// goes to the caches at position pos[n] as bf16 and is cleared (read and
// cleared by the same thread); a position outside [0, ctx) writes nothing.
__global__ void __launch_bounds__(256) tc_cache_scatter_kernel(const __grid_constant__ TcScatterParams S) {
  pdl_launch_dependents();
  pdl_wait();
  const int n = blockIdx.y;
  const int hr = S.heads * S.rank, width = 2 * hr;
  const int ps = S.pos[n];
  const bool keep = ps >= 0 && ps < S.ctx;
  float* a = S.acc + size_t(n) * width;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < width; j += gridDim.x * blockDim.x) {
    const float v = __ldcg(a + j);
    __stcg(a + j, 0.f);
    if (keep) {
      const int kv = j >= hr ? 1 : 0, rr = j - kv * hr;
      __nv_bfloat16* c = reinterpret_cast<__nv_bfloat16*>(kv ? S.cache_v : S.cache_k);
      c[((size_t(n) * S.heads + rr / S.rank) * S.ctx + ps) * S.rank + rr % S.rank] = __float2bfloat16_rn(v);
    }
  }
}

int kb_elems(bool i8) { return i8 ? 128 : 64; }

}  // namespace

int tc_gemv_kc(int K, int k_splits, bool i8) {
  const int e = kb_elems(i8);
  return ((K + k_splits - 1) / k_splits + e - 1) / e * e;
}

size_t tc_gemv_smem(int kc, int N, bool i8, int stages) {
  return size_t(stages) * kATile + size_t(kc / kb_elems(i8)) * N * 128 + 1024;
}

bool tc_gemv_fits(int kc, int N, bool i8) { return N <= kMaxTokens && tc_gemv_smem(kc, N, i8, kStages) <= kSmemCap; }

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
  // a 4-stage ring, or 3 stages where that is what keeps two CTAs on an SM (a wide
  // activation operand, many tokens): the second CTA hides the first one's latency
  TcGemvParams q = p;
  q.stages = kStages;
  if (tc_gemv_smem(kc_max, p.N, i8, kStages) > kTwoPerSm && tc_gemv_smem(kc_max, p.N, i8, kStages - 1) <= kTwoPerSm)
    q.stages = kStages - 1;
  const size_t smem = tc_gemv_smem(kc_max, p.N, i8, q.stages);
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
  return cudaLaunchKernelEx(&c, kern, maps, q);
}

cudaError_t launch_tc_cache_scatter(const TcScatterParams& p, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3((2 * p.heads * p.rank + 255) / 256, p.nb);
  c.blockDim = dim3(256);
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, tc_cache_scatter_kernel, p);
}

cudaError_t launch_tc_swiglu(const TcSwigluParams& p, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(p.nb, (p.n_lr + p.n_dense + kSwigluChunk - 1) / kSwigluChunk);
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
