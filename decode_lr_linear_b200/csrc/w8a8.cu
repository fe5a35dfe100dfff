// W8A8 low-rank linear for prefill on tcgen05 tensor cores, sm_100a.
//
// LASER results (W8A8 setting) and WSVD QAT section (weights and activations
// int8): y = (x A) B with int8 activations (one scale per token), int8
// factors (one scale per output channel), int32 accumulation, and the latent
// requantised per token between the two products:
//   acc1 = x_q A_q                   (tcgen05.mma kind::i8, int32 in TMEM)
//   z    = fp32(fp32(acc1 * s_x[t]) * s_A[j])                     (requant)
//   s_z  = max|z| / 127, z_q = clamp(rint(z / s_z))               (requant)
//   acc2 = z_q B_q                   (tcgen05.mma kind::i8)
//   y    = bf16(fp32(fp32(acc2 * s_z[t]) * s_B[k]))                (epilogue)
// Every fp32 step is one IEEE operation (__fmul_rn, the correctly rounded
// quotient, rintf), so the codes match an exact emulation bit for bit.
//
// GEMM kernel: persistent, one CTA per SM, 128 x 256 output tiles.  Warp 0
// issues TMA loads of 128-byte-swizzled operand tiles into a 4-stage
// shared-memory ring; warp 1 allocates two 256-column TMEM accumulators and
// one elected thread issues the MMAs (four K=32 steps per 128-byte k-block),
// releasing each stage with tcgen05.commit; warps 2..5 (one per TMEM lane
// quarter) read a finished accumulator with tcgen05.ld and run the epilogue
// while the next tile accumulates in the other one; the epilogue's results
// leave through swizzled shared-memory buffers and tiled TMA stores.  The first product is
// split along K (stream-K: every CTA takes an equal share of the (tile,
// k-block) space, so a short grid of tiles still fills every SM) and its
// pieces are added into an int32 buffer, which is exact in any order; the
// second product, whose epilogue needs the whole sum, deals whole tiles.
// The first factor A_q [r, d_in] is K-major (the B operand of GEMM 1); the
// second factor B_q [r, d_out] is N-contiguous, i.e. an MN-major B operand of
// GEMM 2.  Every wait is bounded and records a device error instead of
// hanging.
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "quant.cuh"
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
constexpr int kTmemCols = 512;       // two 256-column accumulators
constexpr int kEpiBufBytes = 32 * 128;        // one 32 x 32 chunk of 4-byte values, 128-byte swizzled rows
constexpr int kEpiStageBytes = 4 * 2 * kEpiBufBytes;  // two buffers per epilogue warp

// 2-D int8 tensor [rows, cols] (row stride `ld` bytes), box [box_rows, box_cols],
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows,
              uint32_t box_cols) {
  return tc::make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rows, cols, ld, box_rows, box_cols,
                         CU_TENSOR_MAP_SWIZZLE_128B);
}

// Output maps of the epilogue's tiled stores: 32 x 32 boxes, int32 with
// 128-byte rows (128-byte swizzle) or bf16 with 64-byte rows (64-byte swizzle).
bool make_out_map(CUtensorMap* m, const void* base, bool bf16, uint64_t rows, uint64_t cols, uint64_t ld_bytes) {
  return tc::make_map_2d(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_INT32, base, rows, cols,
                         ld_bytes, 32, 32, bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
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
  int mode;                // 0: int32 partial sums added into acc (K split); 1: bf16 y epilogue; 2: raw int32 C
  const float* s_row;      // mode 1: per-token scale s_z
  const float* s_col;      // mode 1: per-column scale s_B
  int* err;                // the output goes through the map mapC: mode 0 int32 acc [M, N] (zero on
                           // entry), mode 1 bf16 y [M, N], mode 2 int32 C [M, N]
};

// One piece of a CTA's work: output tile (m0, n0) over k-blocks [kb0, kb1).
struct Seg {
  int m0, n0, kb0, kb1;
};

// The persistent schedule.  Mode 0 splits the linear (tile, k-block) space
// into gridDim.x contiguous ranges (stream-K): a range may start or end in
// the middle of a tile, and the pieces of a tile meet in the int32 buffer
// (integer addition, so the order does not matter).  Modes 1 and 2 need the
// whole sum in one place and deal whole tiles round robin.  Producer, MMA
// issuer and epilogue walk the same sequence.
struct Walker {
  long long u, hi;
  int tile, tiles, ntn, nk, mode;
  LR_DEV void init(const GemmParams& P) {
    ntn = (P.N + kBN - 1) / kBN;
    tiles = ntn * ((P.M + kBM - 1) / kBM);
    nk = (P.K + kBK - 1) / kBK;
    mode = P.mode;
    const long long total = (long long)tiles * nk;
    u = total * blockIdx.x / gridDim.x;
    hi = total * (blockIdx.x + 1) / gridDim.x;
    tile = blockIdx.x;
  }
  LR_DEV bool next(Seg& s) {
    int t;
    if (mode == 0) {
      if (u >= hi) return false;
      t = int(u / nk);
      s.kb0 = int(u - (long long)t * nk);
      const long long left = hi - u;
      s.kb1 = left < (long long)(nk - s.kb0) ? s.kb0 + int(left) : nk;
      u += s.kb1 - s.kb0;
    } else {
      if (tile >= tiles) return false;
      t = tile;
      tile += gridDim.x;
      s.kb0 = 0;
      s.kb1 = nk;
    }
    s.m0 = (t / ntn) * kBM;
    s.n0 = (t % ntn) * kBN;
    return true;
  }
};

// Tiled stores from shared memory (bulk async-group completion): a plain
// store, or an element-wise atomic add into global memory (the int32 type of
// the map).  Boxes that reach past the tensor are clipped by the copy engine.
LR_DEV void tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(src) : "memory");
}
LR_DEV void tma_reduce_add_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(src) : "memory");
}
LR_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most one group still reading its shared-memory source
LR_DEV void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every group complete (writes performed)
LR_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
LR_DEV void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) w8a8_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                                                                const __grid_constant__ CUtensorMap mapB,
                                                                const __grid_constant__ CUtensorMap mapC,
                                                                const __grid_constant__ GemmParams P) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  __shared__ __align__(8) uint64_t tfull[2];   // accumulator b holds a finished segment
  __shared__ __align__(8) uint64_t tempty[2];  // accumulator b has been read by the four epilogue warps
  __shared__ uint32_t tmem_slot;
  // operand tiles must start on 1024-byte boundaries (128-byte swizzle atoms)
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
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
  Walker w;
  w.init(P);

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();  // the A operand (activations) may come from the preceding kernel
      uint32_t g = 0;
      bool ok = true;
      Seg sg;
      while (ok && w.next(sg)) {
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++g) {
          const uint32_t s = g % kStages, round = g / kStages;
          if (round > 0 && !mbar_wait_bounded(&empty[s], (round - 1) & 1u, P.err)) { ok = false; break; }
          const uint32_t a_dst = base + s * kStageBytes, b_dst = a_dst + kATileBytes;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(a_dst, &mapA, kb * kBK, sg.m0, &full[s]);
          if (!P.b_mn_major) {
            tma_load_2d(b_dst, &mapB, kb * kBK, sg.n0, &full[s]);
          } else {
            tma_load_2d(b_dst, &mapB, sg.n0, kb * kBK, &full[s]);
            tma_load_2d(b_dst + kBK * 128, &mapB, sg.n0 + 128, kb * kBK, &full[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_i8(kBM, kBN, P.b_mn_major != 0);
      uint32_t g = 0;
      bool ok = true;
      Seg sg;
      for (int j = 0; ok && w.next(sg); ++j) {
        const int b = j & 1;
        if (j >= 2) {
          if (!mbar_wait_bounded(&tempty[b], uint32_t((j >> 1) - 1) & 1u, P.err)) break;
          tc_fence_after();
        }
        const uint32_t d = tmem + uint32_t(b * kBN);
        for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++g) {
          const uint32_t s = g % kStages, round = g / kStages;
          if (!mbar_wait_bounded(&full[s], round & 1u, P.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = base + s * kStageBytes, b_base = a_base + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 32; ++kk) {
            const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = P.b_mn_major ? smem_desc(b_base + kk * 32 * 128, kBK * 128, 1024)
                                             : smem_desc(b_base + kk * 32, 16, 1024);
            mma_i8(d, ad, bd, idesc, kb > sg.kb0 || kk > 0);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tfull[b]);
      }
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31 (one accumulator row per thread).
    // The per-token scales of mode 1 were written by the preceding kernel:
    // every thread that reads them waits for it first.
    pdl_wait();
    const int q = warp & 3;
    // Each 32 x 32 chunk (lane = row) is written into one of this warp's two
    // swizzled shared-memory buffers and leaves through the copy engine: a
    // tiled store of bf16 y (64-byte rows, 64-byte swizzle) or int32 C, or a
    // tiled atomic add of the int32 partial sums (128-byte rows, 128-byte
    // swizzle); the swizzle keeps the row-per-lane writes free of bank
    // conflicts.  One lane issues the copies and keeps one in flight per buffer.
    const uint32_t stage0 = base + uint32_t(kStages * kStageBytes + q * 2 * kEpiBufBytes);
    uint32_t nst = 0;
    Seg sg;
    for (int j = 0; w.next(sg); ++j) {
      const int b = j & 1;
      if (!mbar_wait_bounded(&tfull[b], uint32_t(j >> 1) & 1u, P.err)) break;
      tc_fence_after();
      const int row = sg.m0 + q * 32 + lane;
      const int rbase = sg.m0 + q * 32;
      const float sr = (P.mode == 1 && row < P.M) ? P.s_row[row] : 0.f;
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(b * kBN + c * 32), v);
        if (c == kBN / 32 - 1) {
          // the accumulator is in registers: hand it back to the MMA issuer
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        }
        const int col0 = sg.n0 + c * 32;
        if (col0 >= P.N || rbase >= P.M) continue;
        const uint32_t buf = stage0 + (nst & 1u) * kEpiBufBytes;
        if (lane == 0) bulk_wait_read_1();  // the copy issued two chunks ago from this buffer has read it
        __syncwarp();
        if (P.mode == 1) {
          // y = bf16(fp32(fp32(acc * s_z[t]) * s_B[k])); N is a multiple of 16, so
          // every group of four column scales is wholly inside or outside the row
          const float4* sc4 = reinterpret_cast<const float4*>(P.s_col + col0);
          uint32_t wds[16];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 sc = col0 + 4 * g < P.N ? __ldg(sc4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float f0 = __fmul_rn(__fmul_rn(__int2float_rn(int(v[4 * g + 0])), sr), sc.x);
            const float f1 = __fmul_rn(__fmul_rn(__int2float_rn(int(v[4 * g + 1])), sr), sc.y);
            const float f2 = __fmul_rn(__fmul_rn(__int2float_rn(int(v[4 * g + 2])), sr), sc.z);
            const float f3 = __fmul_rn(__fmul_rn(__int2float_rn(int(v[4 * g + 3])), sr), sc.w);
            const __nv_bfloat162 h0 = __floats2bfloat162_rn(f0, f1), h1 = __floats2bfloat162_rn(f2, f3);
            wds[2 * g] = *reinterpret_cast<const uint32_t*>(&h0);
            wds[2 * g + 1] = *reinterpret_cast<const uint32_t*>(&h1);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k)
            st_shared_v4(buf + uint32_t(lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)), wds[4 * k], wds[4 * k + 1],
                         wds[4 * k + 2], wds[4 * k + 3]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(buf + uint32_t(lane * 128 + ((k ^ (lane & 7)) << 4)), v[4 * k], v[4 * k + 1], v[4 * k + 2],
                         v[4 * k + 3]);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          if (P.mode == 0) tma_reduce_add_2d(&mapC, col0, rbase, buf);
          else tma_store_2d(&mapC, col0, rbase, buf);
          bulk_commit();
        }
        ++nst;
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Per-token requantisation of the latent, from the int32 sums of the first
// product (row stride rank_pad): z_j = fp32(fp32(acc_j * s_x) * s_A[j]), s_z =
// max_j |z_j| / 127 (1 for a zero row), z_q = clamp(rint(z / s_z), -127, 127);
// columns r .. rank_pad-1 of z_q are zero (their sums are zero: the first
// product never writes them).  The sums are reset to zero for the next call.
// One CTA per token, four columns per access (16-byte loads of the sums, four
// codes per store); the first kHeldGroups groups of each thread stay in
// registers between the row maximum and the quantisation.
constexpr int kReqThreads = 256;
constexpr int kHeldGroups = 4;

__global__ void __launch_bounds__(kReqThreads) requant_kernel(int32_t* __restrict__ acc, const float* __restrict__ sx,
                                                              const float* __restrict__ sA, int r, int rank_pad,
                                                              int8_t* __restrict__ zq, float* __restrict__ sz) {
  __shared__ float red[kReqThreads / 32];
  const int t = blockIdx.x;
  pdl_launch_dependents();
  pdl_wait();
  int32_t* ar = acc + size_t(t) * rank_pad;
  const int ng = rank_pad >> 2;
  const float sr = sx[t];
  // z of the four columns of group g (scales past r are not read: their sums are zero)
  auto zgroup = [&](int g, float* z) {
    const int4 a = *reinterpret_cast<const int4*>(ar + 4 * g);
    const int j = 4 * g;
    float s4[4];
    if (j + 4 <= r) {
      const float4 f = *reinterpret_cast<const float4*>(sA + j);
      s4[0] = f.x; s4[1] = f.y; s4[2] = f.z; s4[3] = f.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) s4[e] = j + e < r ? sA[j + e] : 0.f;
    }
    z[0] = __fmul_rn(__fmul_rn(__int2float_rn(a.x), sr), s4[0]);
    z[1] = __fmul_rn(__fmul_rn(__int2float_rn(a.y), sr), s4[1]);
    z[2] = __fmul_rn(__fmul_rn(__int2float_rn(a.z), sr), s4[2]);
    z[3] = __fmul_rn(__fmul_rn(__int2float_rn(a.w), sr), s4[3]);
  };
  float z[kHeldGroups][4];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < kHeldGroups; ++i) {
    const int g = threadIdx.x + i * kReqThreads;
    if (g < ng) {
      zgroup(g, z[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) m = fmaxf(m, fabsf(z[i][e]));
    }
  }
  for (int g = threadIdx.x + kHeldGroups * kReqThreads; g < ng; g += kReqThreads) {
    float w[4];
    zgroup(g, w);
#pragma unroll
    for (int e = 0; e < 4; ++e) m = fmaxf(m, fabsf(w[e]));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int k = 1; k < kReqThreads / 32; ++k) m = fmaxf(m, red[k]);
  float sc = __fdiv_rn(m, 127.0f);
  const bool zero = sc == 0.0f;
  if (zero) sc = 1.0f;
  if (threadIdx.x == 0) sz[t] = sc;
  uint32_t* qr = reinterpret_cast<uint32_t*>(zq + size_t(t) * rank_pad);
  const float inv = __frcp_rn(sc);
  auto put = [&](int g, const float* w) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float c = zero ? 0.f : quant_code(w[e], sc, inv);
      word |= (uint32_t(int(c)) & 0xffu) << (8 * e);
    }
    qr[g] = word;
    *reinterpret_cast<int4*>(ar + 4 * g) = make_int4(0, 0, 0, 0);
  };
#pragma unroll
  for (int i = 0; i < kHeldGroups; ++i) {
    const int g = threadIdx.x + i * kReqThreads;
    if (g < ng) put(g, z[i]);
  }
  for (int g = threadIdx.x + kHeldGroups * kReqThreads; g < ng; g += kReqThreads) {
    float w[4];
    zgroup(g, w);
    put(g, w);
  }
}

// Persistent grid: one CTA per SM at most (the shared-memory ring keeps it
// to one), fewer when there is less work; mode 0 gives every CTA at least
// four k-blocks so that its partial sums are worth their atomic traffic.
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& out, const GemmParams& p,
                        int sm_count, cudaStream_t s) {
  const size_t smem = size_t(kStages) * kStageBytes + 1024 + kEpiStageBytes;
  cudaError_t e = ensure_smem(w8a8_gemm_kernel, smem);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)((p.N + kBN - 1) / kBN) * ((p.M + kBM - 1) / kBM);
  long long units = tiles;
  if (p.mode == 0) units = tiles * ((p.K + kBK - 1) / kBK) / 4;
  if (units < 1) units = 1;
  const int grid = int(units < sm_count ? units : sm_count);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(grid);
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = smem;
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, w8a8_gemm_kernel, a, b, out, p);
}

}  // namespace

size_t w8a8_workspace_bytes(int T, int rank) {
  const size_t rp = (size_t(rank) + 127) / 128 * 128;
  const size_t tp = (size_t(T) + 127) / 128 * 128;
  auto ru = [](size_t v) { return (v + 255) / 256 * 256; };
  return ru(size_t(T) * rp * 4) + ru(tp * rp) + ru(tp * 4);
}

cudaError_t launch_gemm_s8s32(const int8_t* A, const int8_t* B, int b_kn, int M, int N, int K, int32_t* C,
                              int* err, int sm_count, cudaStream_t s) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, K, kBM, kBK)) return cudaErrorInvalidValue;
  if (!b_kn) {
    if (!make_map(&mb, B, N, K, K, kBN, kBK)) return cudaErrorInvalidValue;
  } else {
    if (!make_map(&mb, B, K, N, N, kBK, 128)) return cudaErrorInvalidValue;
  }
  CUtensorMap mc;
  if (!make_out_map(&mc, C, false, M, N, uint64_t(N) * 4)) return cudaErrorInvalidValue;
  GemmParams g;
  std::memset(&g, 0, sizeof(g));
  g.M = M; g.N = N; g.K = K; g.b_mn_major = b_kn; g.mode = 2; g.err = err;
  return launch_gemm(ma, mb, mc, g, sm_count, s);
}

cudaError_t launch_w8a8(const W8A8Params& p, int sm_count, cudaStream_t s) {
  CUtensorMap mx, ma, mz, mb, macc, my;
  if (!make_map(&mx, p.xq, p.T, p.d_in, p.d_in, kBM, kBK)) return cudaErrorInvalidValue;
  if (!make_out_map(&macc, p.acc, false, p.T, p.rank, uint64_t(p.rank_pad) * 4)) return cudaErrorInvalidValue;
  if (!make_out_map(&my, p.y, true, p.T, p.d_out, uint64_t(p.d_out) * 2)) return cudaErrorInvalidValue;
  if (!make_map(&ma, p.Aq, p.rank, p.d_in, p.d_in, kBN, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&mz, p.zq, p.T, p.rank_pad, p.rank_pad, kBM, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&mb, p.Bq, p.rank, p.d_out, p.d_out, kBK, 128)) return cudaErrorInvalidValue;

  GemmParams g1;
  std::memset(&g1, 0, sizeof(g1));
  g1.M = p.T; g1.N = p.rank; g1.K = p.d_in; g1.b_mn_major = 0; g1.mode = 0;
  g1.err = p.err;
  cudaError_t e = launch_gemm(mx, ma, macc, g1, sm_count, s);
  if (e != cudaSuccess) return e;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(p.T);
  c.blockDim = dim3(kReqThreads);
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  e = cudaLaunchKernelEx(&c, requant_kernel, p.acc, p.sx, p.sA, p.rank, p.rank_pad, p.zq, p.sz);
  if (e != cudaSuccess) return e;

  GemmParams g2;
  std::memset(&g2, 0, sizeof(g2));
  g2.M = p.T; g2.N = p.d_out; g2.K = p.rank; g2.b_mn_major = 1; g2.mode = 1;
  g2.s_row = p.sz; g2.s_col = p.sB; g2.err = p.err;
  return launch_gemm(mz, mb, my, g2, sm_count, s);
}

}  // namespace lr
