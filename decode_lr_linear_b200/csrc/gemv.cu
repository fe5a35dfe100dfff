// Decode-time (small batch) kernels for factorised linears and the hybrid
// SwiGLU FFN on CUDA cores, sm_100a.
//
// A factorised linear y = (x A) B is evaluated as a sum of rank-1 terms,
// y = sum_j z_j b_j with z_j = x . a_j, where a_j / b_j are the latent-major
// rows of the two factors.  Each CTA owns a contiguous block of latent rows:
// it streams its rows of A (phase A, z_j kept in shared memory), then its rows
// of B (phase B), and adds its partial y into an fp32 accumulator in L2 with
// vector reductions.  The last CTA to arrive (atomic ticket, no waiting)
// converts the accumulator to the output type and zeroes it again.  Both
// factor streams are read exactly once, coalesced, 8 elements per lane.
//
// The same building blocks evaluate the hybrid FFN of LASER ("Hybrid
// SVD-Quantization for FFNs", "System Implementation") in two launches:
//   phase 1: low-rank branch  z = x A', [g_S,u_S] += z_j b'_j  (reduction)
//            dense branch     [g_D,u_D] = x D' row dots, SwiGLU in the epilogue
//   phase 2: h = [silu(g_S) u_S, h_D]; y += h_c w_c over input channels of
//            W_down (reduction), last CTA applies the output scales.
#include "common.cuh"
#include "internal.h"

namespace lr {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kLine = 256;          // elements covered by one warp-wide chunk load
constexpr int kMaxRowsCta = 96;     // latent rows owned by one CTA, at most
// independent chunk loads in flight per lane (fewer for wide batches: registers)
template <int NB> constexpr int unroll_for() { return NB >= 8 ? 2 : (NB >= 4 ? 4 : 8); }

struct SmemLayout {
  // part [rows][kWarps][NB] fp32, z [rows][NB] fp32, row pointers, row projections
  static size_t bytes(int rows, int nb) {
    return size_t(rows) * kWarps * nb * 4 + size_t(rows) * nb * 4 + size_t(rows) * 8 + size_t(rows) * 4 + 64;
  }
};

// Phase A: part[r][warp][b] = sum over this warp's lines of a_r . x_b.
template <typename WT, typename XT, int NB, int kUnroll = unroll_for<NB>()>
LR_DEV void phase_dot(const WT* const* arow, int nr, int d_in, const XT* x, int nb, float* part) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = lane; i < nr * NB; i += 32) part[(i / NB) * kWarps * NB + warp * NB + (i % NB)] = 0.f;
  __syncwarp();
  const int nlines = (d_in + kLine - 1) / kLine;
  for (int l = warp; l < nlines; l += kWarps) {
    const int col = l * kLine + lane * 8;
    const bool cv = col < d_in;
    float xr[NB][8];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (cv && b < nb) load_act8(x + size_t(b) * d_in + col, xr[b]);
      else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xr[b][e] = 0.f;
      }
    }
    for (int r = 0; r < nr; r += kUnroll) {
      float w[kUnroll][8];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (cv && r + u < nr) Chunk<WT>::load(arow[r + u] + col, w[u]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) w[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float s = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) s = fmaf(w[u][e], xr[b][e], s);
          s = warp_sum(s);
          if (lane == 0 && r + u < nr) part[(r + u) * kWarps * NB + warp * NB + b] += s;
        }
      }
    }
  }
}

// z[r][b] = sum_w part[r][w][b] (fixed order) times an optional row scale.
template <int NB>
LR_DEV void reduce_parts(const float* part, int nr, float* zs, const void* sA, const int* srow, bool f16) {
  for (int i = threadIdx.x; i < nr * NB; i += kThreads) {
    const int r = i / NB, b = i % NB;
    float s = 0.f;
#pragma unroll 4
    for (int w = 0; w < kWarps; ++w) s += part[r * kWarps * NB + w * NB + b];
    if (sA) s *= load_scale(sA, srow[r], f16);
    zs[r * NB + b] = s;
  }
}

// Phase B: acc[b][k] += sum_r z[r][b] * B0[r][k] over nr consecutive rows of B.
template <typename WT, int NB, int kUnroll = unroll_for<NB>()>
LR_DEV void phase_rank1(const WT* B0, int d_out, int nr, const float* zs, float* acc, int nb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nlines = (d_out + kLine - 1) / kLine;
  for (int l = warp; l < nlines; l += kWarps) {
    const int col = l * kLine + lane * 8;
    const bool cv = col < d_out;
    float a[NB][8];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) a[b][e] = 0.f;
    for (int r = 0; r < nr; r += kUnroll) {
      float w[kUnroll][8];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (cv && r + u < nr) Chunk<WT>::load(B0 + size_t(r + u) * d_out + col, w[u]);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) w[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int rr = (r + u < nr) ? (r + u) : r;  // w is zero when out of range
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float zb = zs[rr * NB + b];
#pragma unroll
          for (int e = 0; e < 8; ++e) a[b][e] = fmaf(zb, w[u][e], a[b][e]);
        }
      }
    }
    if (cv) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < nb) {
          float* p = acc + size_t(b) * d_out + col;
          red_add_f4(p, a[b][0], a[b][1], a[b][2], a[b][3]);
          red_add_f4(p + 4, a[b][4], a[b][5], a[b][6], a[b][7]);
        }
      }
    }
  }
}

// Arrival ticket: returns true in exactly one CTA, the last one to arrive,
// after every CTA's reductions are visible to it.
LR_DEV bool last_cta_arrives(unsigned int* ticket) {
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(ticket, 1u);
    s_last = (prev == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return false;
  __threadfence();
  return true;
}

// y[b][k] = acc[b][k] * scale[k] (optional) in the output type; acc := 0.
template <typename YT>
LR_DEV void finalize(float* acc, YT* y, int nb, int d_out, const void* scale, bool f16) {
  const int n = nb * d_out;
  for (int i = threadIdx.x * 8; i < n; i += kThreads * 8) {
    const int k = i % d_out;
    float4 v0 = ld_cg_f4(acc + i), v1 = ld_cg_f4(acc + i + 4);
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    if (scale) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= load_scale(scale, k + e, f16);
    }
    if constexpr (sizeof(YT) == 2) {
      uint4 o;
      __nv_bfloat162 h[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
      o.x = *reinterpret_cast<uint32_t*>(&h[0]); o.y = *reinterpret_cast<uint32_t*>(&h[1]);
      o.z = *reinterpret_cast<uint32_t*>(&h[2]); o.w = *reinterpret_cast<uint32_t*>(&h[3]);
      *reinterpret_cast<uint4*>(y + i) = o;
    } else {
      *reinterpret_cast<float4*>(y + i) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(y + i + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    st_cg_f4(acc + i, zero);
    st_cg_f4(acc + i + 4, zero);
  }
}

LR_DEV void block_rows(int total, int* r0, int* r1) {
  *r0 = int((long long)total * blockIdx.x / gridDim.x);
  *r1 = int((long long)total * (blockIdx.x + 1) / gridDim.x);
}

// ---------------------------------------------------------------------------
// Factorised linear (grouped): one launch for up to kMaxGroup projections.
// ---------------------------------------------------------------------------
template <typename WT, typename XT, typename YT, int NB>
__global__ void __launch_bounds__(kThreads, 1) lr_rank1_kernel(const __grid_constant__ Rank1Params P) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  int r0, r1;
  block_rows(P.total_rows, &r0, &r1);
  const int nr = r1 - r0;
  float* part = reinterpret_cast<float*>(smem_raw);
  float* zs = part + size_t(nr) * kWarps * NB;
  const WT** arow = reinterpret_cast<const WT**>(zs + size_t(nr) * NB + (nr & 1) * NB);
  int* srow = reinterpret_cast<int*>(arow + nr);
  __shared__ int s_proj_of_row[kMaxRowsCta];

  pdl_launch_dependents();
  for (int i = threadIdx.x; i < nr; i += kThreads) {
    const int g = r0 + i;
    int p = 0;
#pragma unroll
    for (int q = 1; q < kMaxGroup; ++q)
      if (q < P.n_proj && g >= P.proj[q].row_begin) p = q;
    const int j = g - P.proj[p].row_begin;
    arow[i] = reinterpret_cast<const WT*>(P.proj[p].A) + size_t(j) * P.d_in;
    srow[i] = j;
    s_proj_of_row[i] = p;
  }
  __syncthreads();
  // Weights are never written by an earlier kernel: start their DRAM reads
  // before waiting for the producer of x.
  if (threadIdx.x < nr) {
    const size_t bytes = size_t(P.d_in) * sizeof(WT);
    if ((bytes & 15) == 0) prefetch_l2_bulk(arow[threadIdx.x], uint32_t(bytes));
  }
  pdl_wait();

  phase_dot<WT, XT, NB>(arow, nr, P.d_in, reinterpret_cast<const XT*>(P.x), P.nb, part);
  __syncthreads();
  // scale of A depends on the row's projection; all projections share scale dtype
  for (int i = threadIdx.x; i < nr * NB; i += kThreads) {
    const int r = i / NB, b = i % NB;
    float s = 0.f;
#pragma unroll 4
    for (int w = 0; w < kWarps; ++w) s += part[r * kWarps * NB + w * NB + b];
    const void* sA = P.proj[s_proj_of_row[r]].sA;
    if (sA) s *= load_scale(sA, srow[r], P.scale_f16 != 0);
    zs[r * NB + b] = s;
  }
  __syncthreads();

  // phase B over the segments of rows that belong to one projection
  int sa = 0;
  while (sa < nr) {
    const int p = s_proj_of_row[sa];
    int sb = sa + 1;
    while (sb < nr && s_proj_of_row[sb] == p) ++sb;
    const Rank1Proj& pr = P.proj[p];
    const WT* B0 = reinterpret_cast<const WT*>(pr.B) + size_t(srow[sa]) * pr.d_out;
    phase_rank1<WT, NB>(B0, pr.d_out, sb - sa, zs + sa * NB, pr.acc, P.nb);
    sa = sb;
  }

  if (!last_cta_arrives(P.ticket)) return;
  for (int p = 0; p < P.n_proj; ++p)
    finalize<YT>(P.proj[p].acc, reinterpret_cast<YT*>(P.proj[p].y), P.nb, P.proj[p].d_out, P.proj[p].sB,
                 P.scale_f16 != 0);
  if (threadIdx.x == 0) *P.ticket = 0u;
}

template <typename WT, typename XT, typename YT, int NB>
cudaError_t launch_rank1_t(const Rank1Params& p, int sm_count, cudaStream_t s) {
  int grid = sm_count;
  if (grid > p.total_rows) grid = p.total_rows;
  const int need = (p.total_rows + kMaxRowsCta - 1) / kMaxRowsCta;
  if (grid < need) grid = need;
  const int rows_max = (p.total_rows + grid - 1) / grid;
  const size_t smem = SmemLayout::bytes(rows_max, NB);
  auto kern = lr_rank1_kernel<WT, XT, YT, NB>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <typename WT, typename XT, typename YT>
cudaError_t launch_rank1_nb(const Rank1Params& p, int sm_count, cudaStream_t s) {
  if (p.nb <= 1) return launch_rank1_t<WT, XT, YT, 1>(p, sm_count, s);
  if (p.nb <= 2) return launch_rank1_t<WT, XT, YT, 2>(p, sm_count, s);
  if (p.nb <= 4) return launch_rank1_t<WT, XT, YT, 4>(p, sm_count, s);
  return launch_rank1_t<WT, XT, YT, 8>(p, sm_count, s);
}

// ---------------------------------------------------------------------------
// Hybrid SwiGLU FFN.
// ---------------------------------------------------------------------------
template <int NB>
__global__ void __launch_bounds__(kThreads, 1) ffn_phase1_kernel(const __grid_constant__ FfnParams P, int g_lr) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const bool f16 = P.scale_f16 != 0;
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(P.x);
  pdl_launch_dependents();
  if (int(blockIdx.x) < g_lr) {
    // low-rank branch: rows of A' (latent channels) then rows of B'
    const int r0 = int((long long)P.rank * blockIdx.x / g_lr), r1 = int((long long)P.rank * (blockIdx.x + 1) / g_lr);
    const int nr = r1 - r0;
    float* part = reinterpret_cast<float*>(smem_raw);
    float* zs = part + size_t(nr) * kWarps * NB;
    const int8_t** arow = reinterpret_cast<const int8_t**>(zs + size_t(nr) * NB + (nr & 1) * NB);
    int* srow = reinterpret_cast<int*>(arow + nr);
    for (int i = threadIdx.x; i < nr; i += kThreads) {
      arow[i] = P.A + size_t(r0 + i) * P.hidden;
      srow[i] = r0 + i;
    }
    __syncthreads();
    if (threadIdx.x < nr && (P.hidden & 15) == 0) prefetch_l2_bulk(arow[threadIdx.x], uint32_t(P.hidden));
    pdl_wait();
    phase_dot<int8_t, __nv_bfloat16, NB>(arow, nr, P.hidden, x, P.nb, part);
    __syncthreads();
    reduce_parts<NB>(part, nr, zs, P.sA, srow, f16);
    __syncthreads();
    phase_rank1<int8_t, NB>(P.B + size_t(r0) * (2 * P.n_lr), 2 * P.n_lr, nr, zs, P.gu_acc, P.nb);
  } else {
    // dense branch: row pairs (gate_c, up_c) of D, SwiGLU in the epilogue
    const int gd = gridDim.x - g_lr, c = blockIdx.x - g_lr;
    const int p0 = int((long long)P.n_dense * c / gd), p1 = int((long long)P.n_dense * (c + 1) / gd);
    const int nr = 2 * (p1 - p0);
    float* part = reinterpret_cast<float*>(smem_raw);
    float* zs = part + size_t(nr) * kWarps * NB;
    const int8_t** arow = reinterpret_cast<const int8_t**>(zs + size_t(nr) * NB);
    int* srow = reinterpret_cast<int*>(arow + nr);
    for (int i = threadIdx.x; i < nr; i += kThreads) {
      arow[i] = P.D + size_t(2 * p0 + i) * P.hidden;
      srow[i] = 2 * p0 + i;
    }
    __syncthreads();
    if (threadIdx.x < nr && (P.hidden & 15) == 0) prefetch_l2_bulk(arow[threadIdx.x], uint32_t(P.hidden));
    pdl_wait();
    phase_dot<int8_t, __nv_bfloat16, NB>(arow, nr, P.hidden, x, P.nb, part);
    __syncthreads();
    reduce_parts<NB>(part, nr, zs, P.sD, srow, f16);
    __syncthreads();
    for (int i = threadIdx.x; i < (p1 - p0) * NB; i += kThreads) {
      const int pp = i / NB, b = i % NB;
      if (b < P.nb) {
        const float g = zs[(2 * pp) * NB + b], u = zs[(2 * pp + 1) * NB + b];
        P.h_dense[size_t(b) * P.n_dense + p0 + pp] = silu(g) * u;
      }
    }
  }
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1) ffn_phase2_kernel(const __grid_constant__ FfnParams P) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const bool f16 = P.scale_f16 != 0;
  int c0, c1;
  block_rows(P.inter, &c0, &c1);
  const int nr = c1 - c0;
  float* hs = reinterpret_cast<float*>(smem_raw);  // [nr][NB]
  pdl_launch_dependents();
  if (threadIdx.x < nr) {
    const size_t bytes = size_t(P.hidden);
    const int8_t* row = P.Wd + size_t(c0 + threadIdx.x) * P.hidden;
    if ((bytes & 15) == 0) prefetch_l2_bulk(row, uint32_t(bytes));
  }
  pdl_wait();
  const int two_n = 2 * P.n_lr;
  for (int i = threadIdx.x; i < nr * NB; i += kThreads) {
    const int r = i / NB, b = i % NB, ch = c0 + r;
    float h = 0.f;
    if (b < P.nb) {
      if (ch < P.n_lr) {
        float* gp = P.gu_acc + size_t(b) * two_n + 2 * ch;
        float g, u;
        asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(g) : "l"(gp) : "memory");
        asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(u) : "l"(gp + 1) : "memory");
        g *= load_scale(P.sB, 2 * ch, f16);
        u *= load_scale(P.sB, 2 * ch + 1, f16);
        h = silu(g) * u;
        asm volatile("st.global.cg.f32 [%0], %1;" :: "l"(gp), "f"(0.f) : "memory");
        asm volatile("st.global.cg.f32 [%0], %1;" :: "l"(gp + 1), "f"(0.f) : "memory");
      } else {
        h = P.h_dense[size_t(b) * P.n_dense + (ch - P.n_lr)];
      }
    }
    hs[r * NB + b] = h;
  }
  __syncthreads();
  phase_rank1<int8_t, NB>(P.Wd + size_t(c0) * P.hidden, P.hidden, nr, hs, P.y_acc, P.nb);
  if (!last_cta_arrives(P.ticket)) return;
  finalize<__nv_bfloat16>(P.y_acc, reinterpret_cast<__nv_bfloat16*>(P.y), P.nb, P.hidden, P.sd, f16);
  if (threadIdx.x == 0) *P.ticket = 0u;
}

cudaLaunchConfig_t pdl_config(int grid, size_t smem, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int NB>
cudaError_t launch_ffn_t(const FfnParams& p, int sm_count, cudaStream_t s) {
  // split phase-1 CTAs between the branches in proportion to their bytes
  const double lr_bytes = double(p.rank) * (p.hidden + 2.0 * p.n_lr);
  const double dn_bytes = 2.0 * p.n_dense * p.hidden;
  int g_lr = 0, g_d = 0;
  if (p.n_lr > 0 && p.n_dense > 0) {
    g_lr = int(sm_count * lr_bytes / (lr_bytes + dn_bytes) + 0.5);
    if (g_lr < 1) g_lr = 1;
    if (g_lr > sm_count - 1) g_lr = sm_count - 1;
    g_d = sm_count - g_lr;
  } else if (p.n_lr > 0) {
    g_lr = sm_count;
  } else {
    g_d = sm_count;
  }
  if (g_lr > p.rank) g_lr = p.rank;
  if (g_lr > 0 && (p.rank + g_lr - 1) / g_lr > kMaxRowsCta) g_lr = (p.rank + kMaxRowsCta - 1) / kMaxRowsCta;
  if (g_d > p.n_dense) g_d = p.n_dense;
  if (g_d > 0 && 2 * ((p.n_dense + g_d - 1) / g_d) > kMaxRowsCta) g_d = (2 * p.n_dense + kMaxRowsCta - 1) / kMaxRowsCta;
  const int rows1 = std::max(g_lr ? (p.rank + g_lr - 1) / g_lr : 0, g_d ? 2 * ((p.n_dense + g_d - 1) / g_d) : 0);
  const size_t smem1 = SmemLayout::bytes(rows1 + 1, NB);
  cudaLaunchAttribute attr[1];
  auto k1 = ffn_phase1_kernel<NB>;
  cudaError_t e = ensure_smem(k1, smem1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c1 = pdl_config(g_lr + g_d, smem1, s, attr);
  e = cudaLaunchKernelEx(&c1, k1, p, g_lr);
  if (e != cudaSuccess) return e;

  int g2 = std::min(sm_count, p.inter);
  if ((p.inter + g2 - 1) / g2 > kMaxRowsCta) g2 = (p.inter + kMaxRowsCta - 1) / kMaxRowsCta;
  const size_t smem2 = size_t((p.inter + g2 - 1) / g2) * NB * 4 + 64;
  auto k2 = ffn_phase2_kernel<NB>;
  e = ensure_smem(k2, smem2);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t c2 = pdl_config(g2, smem2, s, attr);
  return cudaLaunchKernelEx(&c2, k2, p);
}

}  // namespace

cudaError_t launch_lr_rank1(const Rank1Params& p, lr_dtype_t w_dtype, int sm_count, cudaStream_t s) {
  switch (w_dtype) {
    case LR_F32: return launch_rank1_nb<float, float, float>(p, sm_count, s);
    case LR_BF16: return launch_rank1_nb<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(p, sm_count, s);
    case LR_I8: return launch_rank1_nb<int8_t, __nv_bfloat16, __nv_bfloat16>(p, sm_count, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_ffn(const FfnParams& p, int sm_count, cudaStream_t s) {
  if (p.nb <= 1) return launch_ffn_t<1>(p, sm_count, s);
  if (p.nb <= 2) return launch_ffn_t<2>(p, sm_count, s);
  if (p.nb <= 4) return launch_ffn_t<4>(p, sm_count, s);
  return launch_ffn_t<8>(p, sm_count, s);
}

}  // namespace lr
