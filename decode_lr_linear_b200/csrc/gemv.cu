// Decode-time (small batch) hybrid SwiGLU FFN on CUDA cores, sm_100a: LASER
// ("Hybrid SVD-Quantization for FFNs", "System Implementation").
//
// One streaming engine runs both launches.  Each CTA owns a contiguous block
// of weight rows; one producer warp streams them through a ring of
// shared-memory stages with bulk asynchronous copies (cp.async.bulk,
// completing on mbarriers), and sixteen consumer warps compute from shared
// memory:
//   phase 1: low-rank branch  z = x A', [g_S,u_S] += z_j b'_j (fp32 vector
//            reductions into L2, red.global.add.v4.f32);
//            dense branch     [g_D,u_D] = x D' row dots, SwiGLU in the epilogue
//   phase 2: h = [silu(g_S) u_S, h_D]; y += h_c w_c over input channels of
//            W_down (reduction); after a grid barrier each CTA applies the
//            output scales to its slice of y and zeroes the accumulator.
// Each weight byte is read once per launch; the weight copies are issued
// before the programmatic-dependent-launch wait, so they overlap the tail of
// the preceding kernel.  The factorised linears themselves run in chain.cu.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace lr {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + one producer warp
constexpr int kLineElems = 256;            // elements of one warp-wide chunk (8 per lane)
constexpr int kStageBytes = 32 * 1024;
constexpr int kMaxStages = 4;
// A CTA that fits in this much shared memory can share its SM with the next
// kernel's CTA, whose producer then streams while this one drains.
constexpr size_t kCoResidentSmem = 108 * 1024;
constexpr int kRowGroup = 4;               // rows reduced together in phase A (ILP)
constexpr int kMaxSegs = 2 * kMaxGroup;
constexpr size_t kSmemLimit = 227 * 1024;

enum Mode : int { kFfn1 = 1, kFfn2 = 2, kDense = 3 };
enum SegKind : int { kDot = 0, kRank1 = 1 };

struct Seg {
  const unsigned char* src;  // first byte of the segment's first row
  int row_bytes;
  int rows;
  int rps;                   // rows per ring stage
  int kind;                  // kDot: row . x ; kRank1: acc += z_row * row
  int zrow0;                 // CTA-local index of the first row (into part / z)
};

struct Plan {
  Seg seg[kMaxSegs];
  int nseg;
  int nrows;
  int row_base;              // first global row of the CTA (scales, channel ids)
  int role;                  // kFfn1: 0 low-rank branch, 1 dense branch
};

struct KParams {
  FfnParams f;
  int g_lr;                  // kFfn1: CTAs of the low-rank branch
  int stages;                // ring stages in use
  int rows_cap;              // rows per CTA the shared-memory layout holds
  int x_elems;               // elements of one staged activation row (0: none)
  int* err;
};

struct Layout {
  size_t ring, x, part, z, total;
};

LR_HD_INLINE size_t round16(size_t v) { return (v + 15) & ~size_t(15); }

template <int NB>
LR_HD_INLINE Layout layout_for(int stages, int x_elems, int x_esize, int rows_cap) {
  Layout L;
  L.ring = 0;
  L.x = size_t(stages) * kStageBytes;
  L.part = L.x + round16(size_t(NB) * x_elems * x_esize);
  L.z = L.part + round16(size_t(rows_cap) * kConsumerWarps * NB * 4);
  L.total = L.z + round16(size_t(rows_cap) * NB * 4);
  return L;
}

// ---- shared-memory chunk loads (8 elements) --------------------------------
template <typename T> struct SChunk;
template <> struct SChunk<__nv_bfloat16> {
  LR_DEV static void load(const unsigned char* p, float* f) { bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f); }
};
template <> struct SChunk<int8_t> {
  LR_DEV static void load(const unsigned char* p, float* f) { i8x8_to_f32(*reinterpret_cast<const uint2*>(p), f); }
};

LR_DEV void consumer_sync() { asm volatile("bar.sync 1, %0;" :: "r"(kConsumers) : "memory"); }

// Sum of four per-lane values over the warp for each of the four, with six
// shuffles: after the two exchange steps lane l holds a partial of value
// ((l >> 3) & 3) over lanes {l, l^8, l^16, l^24}; three more steps finish it.
// Lanes 0, 8, 16 and 24 return the totals of values 0, 1, 2 and 3.
LR_DEV float warp_sum4(float v0, float v1, float v2, float v3, int lane) {
  const bool hi = (lane & 16) != 0, mid = (lane & 8) != 0;
  const float r0 = __shfl_xor_sync(0xffffffffu, hi ? v0 : v2, 16);
  const float r1 = __shfl_xor_sync(0xffffffffu, hi ? v1 : v3, 16);
  const float k0 = (hi ? v2 : v0) + r0, k1 = (hi ? v3 : v1) + r1;
  const float r = __shfl_xor_sync(0xffffffffu, mid ? k0 : k1, 8);
  float t = (mid ? k1 : k0) + r;
  t += __shfl_xor_sync(0xffffffffu, t, 4);
  t += __shfl_xor_sync(0xffffffffu, t, 2);
  t += __shfl_xor_sync(0xffffffffu, t, 1);
  return t;
}

// ---- phase A: part[row][warp][b] = sum over this warp's lines of row . x_b --
// Every (row, warp) slot is written exactly once (a row lives in one stage and
// all of a warp's lines of that row are summed here), so part needs no zeroing.
// When a row has at most kConsumerWarps lines, warp w only ever touches line w
// and its x chunk comes from registers (xr), loaded once per kernel.
template <typename WT, typename XT, int NB>
LR_DEV void consume_dot(const unsigned char* stage, int k, int d_in, const XT* xs, const float (&xr)[NB][8],
                        bool x_in_regs, float* part, int zrow, int cw, int lane) {
  const int lines = (d_in + kLineElems - 1) / kLineElems;
  for (int r0 = 0; r0 < k; r0 += kRowGroup) {
    float s[kRowGroup][NB];
#pragma unroll
    for (int u = 0; u < kRowGroup; ++u)
#pragma unroll
      for (int b = 0; b < NB; ++b) s[u][b] = 0.f;
    for (int line = cw; line < lines; line += kConsumerWarps) {
      const int col = line * kLineElems + lane * 8;
      if (col < d_in) {
        float xv[NB][8];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (NB <= 2 && x_in_regs) {
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[b][e] = xr[b][e];
          } else {
            SChunk<XT>::load(reinterpret_cast<const unsigned char*>(xs + size_t(b) * d_in + col), xv[b]);
          }
        }
        float w[kRowGroup][8];
#pragma unroll
        for (int u = 0; u < kRowGroup; ++u) {
          const int rr = min(r0 + u, k - 1);  // rows past k load a valid row, masked below
          SChunk<WT>::load(stage + (size_t(rr) * d_in + col) * sizeof(WT), w[u]);
        }
#pragma unroll
        for (int u = 0; u < kRowGroup; ++u) {
          const float m = (r0 + u < k) ? 1.f : 0.f;
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              a0 = fmaf(w[u][e], xv[b][e], a0);
              a1 = fmaf(w[u][e + 1], xv[b][e + 1], a1);
            }
            s[u][b] = fmaf(m, a0 + a1, s[u][b]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float t = warp_sum4(s[0][b], s[1][b], s[2][b], s[3][b], lane);
      const int u = lane >> 3;
      if ((lane & 7) == 0 && r0 + u < k) part[(size_t(zrow + r0 + u) * kConsumerWarps + cw) * NB + b] = t;
    }
  }
}

// ---- phase B: acc[li][b][e] += z[row][b] * row[col+e] ----------------------
template <typename WT, int NB, int LPW>
LR_DEV void consume_rank1(const unsigned char* stage, int k, int d_out, const float* z, int zrow,
                          float (&acc)[LPW][NB][8], int cw, int lane) {
  const int lines = (d_out + kLineElems - 1) / kLineElems;
#pragma unroll
  for (int li = 0; li < LPW; ++li) {
    const int line = cw + li * kConsumerWarps;
    const int col = line * kLineElems + lane * 8;
    if (line < lines && col < d_out) {
#pragma unroll 4
      for (int i = 0; i < k; ++i) {
        float w[8];
        SChunk<WT>::load(stage + (size_t(i) * d_out + col) * sizeof(WT), w);
        const float* zr = z + size_t(zrow + i) * NB;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float zb = zr[b];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[li][b][e] = fmaf(zb, w[e], acc[li][b][e]);
        }
      }
    }
  }
}

template <int NB, int LPW>
LR_DEV void flush_rank1(float (&acc)[LPW][NB][8], float* dst, int d_out, int nb, int cw, int lane) {
  const int lines = (d_out + kLineElems - 1) / kLineElems;
#pragma unroll
  for (int li = 0; li < LPW; ++li) {
    const int line = cw + li * kConsumerWarps;
    const int col = line * kLineElems + lane * 8;
    if (line < lines && col < d_out) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < nb) {
          float* p = dst + size_t(b) * d_out + col;
          red_add_f4(p, acc[li][b][0], acc[li][b][1], acc[li][b][2], acc[li][b][3]);
          red_add_f4(p + 4, acc[li][b][4], acc[li][b][5], acc[li][b][6], acc[li][b][7]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[li][b][e] = 0.f;
  }
}

// ---- producer: stream every segment's rows through the ring ---------------
LR_DEV void produce(const Plan& pl, unsigned char* ring, uint64_t* full, uint64_t* empty, int stages, int* err) {
  // Start the DRAM reads of the CTA's whole working set at once (into L2); the
  // ring copies below then mostly hit L2, and DRAM streaming does not wait for
  // consumer progress or for the preceding kernel.
  for (int s = 0; s < pl.nseg; ++s) {
    const Seg& g = pl.seg[s];
    const size_t total = size_t(g.rows) * g.row_bytes;
    for (size_t off = 0; off < total; off += kStageBytes)
      prefetch_l2_bulk(g.src + off, uint32_t(total - off < size_t(kStageBytes) ? total - off : kStageBytes));
  }
  int st = 0;
  for (int s = 0; s < pl.nseg; ++s) {
    const Seg& g = pl.seg[s];
    for (int r = 0; r < g.rows; r += g.rps) {
      const int k = min(g.rps, g.rows - r);
      const int slot = st % stages, round = st / stages;
      if (round > 0 && !mbar_wait_bounded(&empty[slot], uint32_t(round - 1) & 1u, err)) return;
      const uint32_t bytes = uint32_t(k) * uint32_t(g.row_bytes);
      mbar_arrive_expect_tx(&full[slot], bytes);
      bulk_g2s(ring + size_t(slot) * kStageBytes, g.src + size_t(r) * g.row_bytes, bytes, &full[slot]);
      ++st;
    }
  }
}

// Barrier over the CTAs of one launch.  The grid never exceeds the CTAs that
// can be resident at once (one per SM at most, checked before the launch),
// so every CTA gets to arrive.  words[0] counts arrivals, words[1] is a
// generation number: the last CTA to arrive resets the count and bumps the
// generation; the others wait until the generation changes (bounded: after
// wait_ns the wait gives up and sets the device error word).  All threads of
// the CTA call it; on return every CTA's earlier global writes and
// reductions are visible.
LR_DEV void grid_barrier(unsigned int* words, unsigned long long wait_ns, int* err) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned gen = ld_acquire_u32(words + 1);
    __threadfence();  // after the CTA barrier: covers every thread's earlier writes
    const unsigned prev = atomicAdd(words, 1u);
    if (prev == gridDim.x - 1) {
      atomicExch(words, 0u);
      __threadfence();
      atomicAdd(words + 1, 1u);
    } else {
      const uint64_t t0 = global_ns();
      while (ld_acquire_u32(words + 1) == gen) {
        if (global_ns() - t0 > wait_ns) {
          set_device_error(err, kErrGridBarrier);
          break;
        }
      }
    }
  }
  __syncthreads();
}

// One output of a split reduction: y[b][k] = acc[b][k] * scale[k] (optional).
struct FinalTarget {
  float* acc;
  void* y;
  const void* scale;
  int n;       // nb * d_out
  int d_out;
};

template <typename YT>
LR_DEV void finalize_chunk(const FinalTarget& t, int i, bool f16) {
  const float4 v0 = ld_cg_f4(t.acc + i), v1 = ld_cg_f4(t.acc + i + 4);
  const int k = i % t.d_out;
  float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  if (t.scale) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] *= load_scale(t.scale, k + e, f16);
  }
  YT* y = reinterpret_cast<YT*>(t.y);
  if constexpr (sizeof(YT) == 2) {
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
      ow[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(y + i) = o;
  } else {
    *reinterpret_cast<float4*>(y + i) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(y + i + 4) = make_float4(v[4], v[5], v[6], v[7]);
  }
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  st_cg_f4(t.acc + i, zero);
  st_cg_f4(t.acc + i + 4, zero);
}

// After the grid barrier: this CTA converts its 1/gridDim share of all the
// targets' 8-element chunks (targets concatenated) and zeroes them in acc.
template <typename YT, int NT>
LR_DEV void finalize_slice(const FinalTarget (&t)[NT], int nt, bool f16) {
  int total = 0;
#pragma unroll
  for (int q = 0; q < NT; ++q)
    if (q < nt) total += t[q].n / 8;
  const int c0 = int((long long)total * blockIdx.x / gridDim.x);
  const int c1 = int((long long)total * (blockIdx.x + 1) / gridDim.x);
  for (int c = c0 + int(threadIdx.x); c < c1; c += kThreads) {
    int off = c;
#pragma unroll
    for (int q = 0; q < NT; ++q) {
      if (q < nt) {
        const int nq = t[q].n / 8;
        if (off >= 0 && off < nq) finalize_chunk<YT>(t[q], off * 8, f16);
        off -= nq;
      }
    }
  }
}

LR_DEV void split_range(long long total, int part, int parts, int* a, int* b) {
  *a = int(total * part / parts);
  *b = int(total * (part + 1) / parts);
}

LR_DEV int rows_per_stage(int row_bytes) { return max(1, kStageBytes / row_bytes); }

// Build this CTA's segment list (thread 0 only).
template <typename WT, int MODE>
LR_DEV void build_plan(const KParams& K, Plan& pl) {
  pl.nseg = 0;
  pl.role = 0;
  auto add = [&](const void* base, size_t row0, int row_bytes, int rows, int kind, int zrow0, int proj) {
    if (rows <= 0) return;
    Seg& g = pl.seg[pl.nseg++];
    g.src = reinterpret_cast<const unsigned char*>(base) + row0 * size_t(row_bytes);
    g.row_bytes = row_bytes;
    g.rows = rows;
    g.rps = rows_per_stage(row_bytes);
    g.kind = kind;
    g.zrow0 = zrow0;
  };
  if constexpr (MODE == kFfn1) {
    const FfnParams& F = K.f;
    if (int(blockIdx.x) < K.g_lr) {
      int r0, r1;
      split_range(F.rank, blockIdx.x, K.g_lr, &r0, &r1);
      pl.nrows = r1 - r0;
      pl.row_base = r0;
      add(F.A, size_t(r0), F.hidden, r1 - r0, kDot, 0, 0);
      add(F.B, size_t(r0), 2 * F.n_lr, r1 - r0, kRank1, 0, 0);
    } else {
      int p0, p1;
      split_range(F.n_dense, blockIdx.x - K.g_lr, gridDim.x - K.g_lr, &p0, &p1);
      pl.role = 1;
      pl.nrows = 2 * (p1 - p0);
      pl.row_base = 2 * p0;
      add(F.D, size_t(2 * p0), F.hidden, 2 * (p1 - p0), kDot, 0, 0);
    }
  } else if constexpr (MODE == kDense) {
    // dense output-major rows W [d_out, d_in]: f.D = W, f.n_dense = d_out, f.hidden = d_in
    const FfnParams& F = K.f;
    int c0, c1;
    split_range(F.n_dense, blockIdx.x, gridDim.x, &c0, &c1);
    pl.role = 2;
    pl.nrows = c1 - c0;
    pl.row_base = c0;
    add(F.D, size_t(c0), F.hidden * int(sizeof(WT)), c1 - c0, kDot, 0, 0);
  } else {
    const FfnParams& F = K.f;
    int c0, c1;
    split_range(F.inter, blockIdx.x, gridDim.x, &c0, &c1);
    pl.nrows = c1 - c0;
    pl.row_base = c0;
    add(F.Wd, size_t(c0), F.hidden, c1 - c0, kRank1, 0, 0);
  }
}

// Scale of CTA-local row r after phase A (per latent / output channel).
template <int MODE>
LR_DEV float row_scale(const KParams& K, const Plan& pl, int r) {
  const bool f16 = K.f.scale_f16 != 0;
  {
    if (pl.role == 0) return load_scale(K.f.sA, pl.row_base + r, f16);
    if (pl.role == 2 && !K.f.sD) return 1.f;
    return load_scale(K.f.sD, pl.row_base + r, f16);
  }
}

template <typename WT, typename XT, typename YT, int NB, int LPW, int MODE>
__global__ void __launch_bounds__(kThreads, (NB <= 1 && LPW <= 2 ? 2 : 1)) stream_kernel(const __grid_constant__ KParams K) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ Plan pl;
  __shared__ __align__(8) uint64_t full[kMaxStages];
  __shared__ __align__(8) uint64_t empty[kMaxStages];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Layout L = layout_for<NB>(K.stages, K.x_elems, int(sizeof(XT)), K.rows_cap);
  unsigned char* ring = smem;
  XT* xs = reinterpret_cast<XT*>(smem + L.x);
  float* part = reinterpret_cast<float*>(smem + L.part);
  float* zs = reinterpret_cast<float*>(smem + L.z);

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    build_plan<WT, MODE>(K, pl);
    for (int s = 0; s < K.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // weights are never written by an earlier kernel: no dependency wait here
    if (lane == 0) produce(pl, ring, full, empty, K.stages, K.err);
  } else {
    const int cw = warp;
    const int nb = K.f.nb;
    pdl_wait();
    if constexpr (MODE != kFfn2) {
      const uint4* xg = reinterpret_cast<const uint4*>(K.f.x);
      const int n16 = int(size_t(NB) * K.x_elems * sizeof(XT) / 16);
      const int valid16 = int(size_t(nb) * K.x_elems * sizeof(XT) / 16);
      for (int i = threadIdx.x; i < n16; i += kConsumers)
        reinterpret_cast<uint4*>(xs)[i] = i < valid16 ? xg[i] : make_uint4(0u, 0u, 0u, 0u);
    } else {
      const FfnParams& F = K.f;
      const bool f16 = F.scale_f16 != 0;
      const int two_n = 2 * F.n_lr;
      for (int i = threadIdx.x; i < pl.nrows * NB; i += kConsumers) {
        const int r = i / NB, b = i % NB, ch = pl.row_base + r;
        float h = 0.f;
        if (b < nb) {
          if (ch < F.n_lr) {
            float* gp = F.gu_acc + size_t(b) * two_n + 2 * ch;
            float g, u;
            asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(g) : "l"(gp) : "memory");
            asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(u) : "l"(gp + 1) : "memory");
            g *= load_scale(F.sB, 2 * ch, f16);
            u *= load_scale(F.sB, 2 * ch + 1, f16);
            h = silu(g) * u;
            asm volatile("st.global.cg.f32 [%0], %1;" :: "l"(gp), "f"(0.f) : "memory");
            asm volatile("st.global.cg.f32 [%0], %1;" :: "l"(gp + 1), "f"(0.f) : "memory");
          } else {
            h = F.h_dense[size_t(b) * F.n_dense + (ch - F.n_lr)];
          }
        }
        zs[r * NB + b] = h;
      }
    }
    consumer_sync();

    // this warp's x chunk, when each warp owns a single line of every row
    float xr[NB][8];
    const bool x_in_regs = NB <= 2 && MODE != kFfn2 && (K.x_elems + kLineElems - 1) / kLineElems <= kConsumerWarps;
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) xr[b][e] = 0.f;
    if constexpr (MODE != kFfn2) {
      const int col = cw * kLineElems + lane * 8;
      if (x_in_regs && col < K.x_elems) {
#pragma unroll
        for (int b = 0; b < NB; ++b)
          SChunk<XT>::load(reinterpret_cast<const unsigned char*>(xs + size_t(b) * K.x_elems + col), xr[b]);
      }
    }

    float acc[LPW][NB][8];
#pragma unroll
    for (int li = 0; li < LPW; ++li)
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[li][b][e] = 0.f;
    bool zready = (MODE == kFfn2), failed = false;
    int st = 0;
    for (int s = 0; s < pl.nseg; ++s) {
      const Seg& g = pl.seg[s];
      if (g.kind == kRank1 && !zready) {
        consumer_sync();
        for (int i = threadIdx.x; i < pl.nrows * NB; i += kConsumers) {
          const int r = i / NB, b = i % NB;
          float v = 0.f;
#pragma unroll 4
          for (int w = 0; w < kConsumerWarps; ++w) v += part[(r * kConsumerWarps + w) * NB + b];
          zs[r * NB + b] = v * row_scale<MODE>(K, pl, r);
        }
        consumer_sync();
        zready = true;
      }
      const int elems = g.row_bytes / int(sizeof(WT));
      for (int r = 0; r < g.rows; r += g.rps) {
        const int k = min(g.rps, g.rows - r);
        const int slot = st % K.stages, round = st / K.stages;
        // after a first timeout: stop computing, keep to the protocol with a
        // short bound so that no issued copy is left in flight
        if (!failed) {
          if (!mbar_wait_bounded(&full[slot], uint32_t(round) & 1u, K.err)) failed = true;
        } else {
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(&full[slot], uint32_t(round) & 1u) && global_ns() - t0 < kDegradedMbarNs) {
          }
        }
        if (!failed) {
          const unsigned char* stage = ring + size_t(slot) * kStageBytes;
          if (g.kind == kDot)
            consume_dot<WT, XT, NB>(stage, k, elems, xs, xr, x_in_regs, part, g.zrow0 + r, cw, lane);
          else consume_rank1<WT, NB, LPW>(stage, k, elems, zs, g.zrow0 + r, acc, cw, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        ++st;
      }
      if (g.kind == kRank1 && !failed) {
        float* dst;
        if constexpr (MODE == kFfn1) dst = K.f.gu_acc;
        else dst = K.f.y_acc;
        flush_rank1<NB, LPW>(acc, dst, elems, nb, cw, lane);
      }
    }
    if constexpr (MODE == kDense) {
      // y[b][row] = row . x_b * scale[row]
      consumer_sync();
      for (int i = threadIdx.x; i < pl.nrows * NB; i += kConsumers) {
        const int r = i / NB, b = i % NB;
        if (b < nb) {
          float v = 0.f;
#pragma unroll 4
          for (int w = 0; w < kConsumerWarps; ++w) v += part[(r * kConsumerWarps + w) * NB + b];
          const __nv_bfloat16 o = __float2bfloat16_rn(v * row_scale<MODE>(K, pl, r));
          const int row = pl.row_base + r;
          if (!K.f.cache_k) {
            reinterpret_cast<__nv_bfloat16*>(K.f.y)[size_t(b) * K.f.n_dense + row] = o;
          } else {
            // latent producer: row (kv, head, j) of token b goes to its cache position
            const int hr = K.f.cache_heads * K.f.cache_rank, ps = K.f.cache_pos[b];
            const int kv = row >= hr ? 1 : 0, rr = row - kv * hr;
            if (ps >= 0 && ps < K.f.cache_ctx) {
              __nv_bfloat16* c = reinterpret_cast<__nv_bfloat16*>(kv ? K.f.cache_v : K.f.cache_k);
              c[((size_t(b) * K.f.cache_heads + rr / K.f.cache_rank) * K.f.cache_ctx + ps) * K.f.cache_rank +
                rr % K.f.cache_rank] = o;
            }
          }
        }
      }
    }
    if constexpr (MODE == kFfn1) {
      if (pl.role == 1) {
        // dense branch: g, u of each channel pair, SwiGLU, h_D
        consumer_sync();
        for (int i = threadIdx.x; i < pl.nrows * NB; i += kConsumers) {
          const int r = i / NB, b = i % NB;
          float v = 0.f;
#pragma unroll 4
          for (int w = 0; w < kConsumerWarps; ++w) v += part[(r * kConsumerWarps + w) * NB + b];
          zs[r * NB + b] = v * row_scale<MODE>(K, pl, r);
        }
        consumer_sync();
        const FfnParams& F = K.f;
        for (int i = threadIdx.x; i < (pl.nrows / 2) * NB; i += kConsumers) {
          const int pp = i / NB, b = i % NB;
          if (b < nb) {
            const float g = zs[(2 * pp) * NB + b], u = zs[(2 * pp + 1) * NB + b];
            F.h_dense[size_t(b) * F.n_dense + pl.row_base / 2 + pp] = silu(g) * u;
          }
        }
      }
    }
  }

  if constexpr (MODE == kFfn1 || MODE == kDense) {
    return;
  } else {
    unsigned int* words = K.f.ticket;
    grid_barrier(words, K.f.wait_ns, K.err);
    {
      FinalTarget t[1] = {FinalTarget{K.f.y_acc, K.f.y, K.f.sd, K.f.nb * K.f.hidden, K.f.hidden}};
      finalize_slice<__nv_bfloat16, 1>(t, 1, K.f.scale_f16 != 0);
    }
  }
}

// ---------------------------------------------------------------------------
// Launch helpers
// ---------------------------------------------------------------------------
template <typename WT, typename XT, typename YT, int NB, int LPW, int MODE>
cudaError_t launch_stream(KParams K, int grid, int sm_count, cudaStream_t s) {
  // Three stages when that lets two CTAs share an SM (the next kernel's
  // producer then streams during this kernel's tail); otherwise the most
  // stages that fit.
  size_t bytes = layout_for<NB>(3, K.x_elems, int(sizeof(XT)), K.rows_cap).total;
  K.stages = 3;
  if (bytes > kCoResidentSmem) {
    for (K.stages = kMaxStages; K.stages >= 2; --K.stages) {
      bytes = layout_for<NB>(K.stages, K.x_elems, int(sizeof(XT)), K.rows_cap).total;
      if (bytes <= kSmemLimit - 2048) break;
    }
    if (bytes > kSmemLimit - 2048) return cudaErrorInvalidValue;
  }
  auto kern = stream_kernel<WT, XT, YT, NB, LPW, MODE>;
  cudaError_t e = ensure_smem(kern, bytes);
  if (e != cudaSuccess) return e;
  if (MODE == kFfn2) {  // the finalize barrier needs every CTA resident
    e = check_resident(reinterpret_cast<const void*>(kern), kThreads, bytes, grid, sm_count);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, K);
}

int lpw_for(int d_out) {
  const int lines = (d_out + kLineElems - 1) / kLineElems;
  const int need = (lines + kConsumerWarps - 1) / kConsumerWarps;
  return need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : need <= 8 ? 8 : 0;
}

// Pick the (NB, LPW) instantiation: NB is the smallest power of two >= nb
// with NB * LPW <= 8 (accumulator registers).
template <typename WT, typename XT, typename YT, int MODE>
cudaError_t dispatch(const KParams& K, int nb, int lpw, int grid, int sm_count, cudaStream_t s) {
#define LR_CASE(NB_, LPW_) \
  if (lpw == LPW_ && nb <= NB_) return launch_stream<WT, XT, YT, NB_, LPW_, MODE>(K, grid, sm_count, s);
  LR_CASE(1, 1) LR_CASE(2, 1) LR_CASE(4, 1) LR_CASE(8, 1)
  LR_CASE(1, 2) LR_CASE(2, 2) LR_CASE(4, 2)
  LR_CASE(1, 4) LR_CASE(2, 4)
  LR_CASE(1, 8)
#undef LR_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_ffn_impl(const FfnParams& p0, int sm_count, cudaStream_t s) {
  const int lpw1 = p0.n_lr > 0 ? lpw_for(2 * p0.n_lr) : 1;
  const int lpw2 = lpw_for(p0.hidden);
  if (lpw1 == 0 || lpw2 == 0) return cudaErrorInvalidValue;
  if (2 * p0.n_lr > kStageBytes || p0.hidden > kStageBytes) return cudaErrorInvalidValue;
  // split phase-1 CTAs between the branches in proportion to their bytes
  const double lr_bytes = double(p0.rank) * (p0.hidden + 2.0 * p0.n_lr);
  const double dn_bytes = 2.0 * p0.n_dense * p0.hidden;
  int g_lr = 0, g_d = 0;
  if (p0.n_lr > 0 && p0.n_dense > 0) {
    g_lr = int(sm_count * lr_bytes / (lr_bytes + dn_bytes) + 0.5);
    g_lr = std::min(std::max(g_lr, 1), sm_count - 1);
    g_d = sm_count - g_lr;
  } else if (p0.n_lr > 0) {
    g_lr = sm_count;
  } else {
    g_d = sm_count;
  }
  if (g_lr > 0) g_lr = std::min(g_lr, p0.rank);
  if (g_d > 0) g_d = std::min(g_d, p0.n_dense);
  // one CTA per SM at most: the finalize barrier of phase 2 needs every CTA resident
  const int g2 = std::min(sm_count, p0.inter);

  KParams K1, K2;
  std::memset(&K1, 0, sizeof(K1));
  std::memset(&K2, 0, sizeof(K2));
  K1.err = K2.err = p0.err;
  K1.g_lr = g_lr;
  K1.rows_cap = std::max(g_lr ? (p0.rank + g_lr - 1) / g_lr : 0, g_d ? 2 * ((p0.n_dense + g_d - 1) / g_d) : 0);
  K1.x_elems = p0.hidden;
  K2.rows_cap = (p0.inter + g2 - 1) / g2;
  K2.x_elems = 0;
  // Each phase takes as many batch rows per launch as its accumulator
  // registers allow (8 / lines per warp; at most 4 in phase 2, whose 8-row
  // instantiation spills).  Phase 1 writes every row of the intermediate
  // gate/up accumulator and h_D first, so phase 2 streams W_down once per
  // group of up to 4 rows even when phase 1 needs more launches.
  const int nb1 = 8 / lpw1, nb2 = std::min(4, 8 / lpw2);
  for (int b0 = 0; b0 < p0.nb; b0 += nb1) {
    FfnParams f = p0;
    f.nb = std::min(nb1, p0.nb - b0);
    f.x = reinterpret_cast<const __nv_bfloat16*>(p0.x) + size_t(b0) * p0.hidden;
    f.gu_acc = p0.gu_acc + size_t(b0) * 2 * p0.n_lr;
    f.h_dense = p0.h_dense + size_t(b0) * p0.n_dense;
    K1.f = f;
    cudaError_t e = dispatch<int8_t, __nv_bfloat16, __nv_bfloat16, kFfn1>(K1, f.nb, lpw1, g_lr + g_d, sm_count, s);
    if (e != cudaSuccess) return e;
  }
  for (int b0 = 0; b0 < p0.nb; b0 += nb2) {
    FfnParams f = p0;
    f.nb = std::min(nb2, p0.nb - b0);
    f.y = reinterpret_cast<__nv_bfloat16*>(p0.y) + size_t(b0) * p0.hidden;
    f.gu_acc = p0.gu_acc + size_t(b0) * 2 * p0.n_lr;
    f.h_dense = p0.h_dense + size_t(b0) * p0.n_dense;
    f.y_acc = p0.y_acc + size_t(b0) * p0.hidden;
    K2.f = f;
    cudaError_t e = dispatch<int8_t, __nv_bfloat16, __nv_bfloat16, kFfn2>(K2, f.nb, lpw2, g2, sm_count, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Dense GEMV: every CTA owns a block of output rows; no reduction, no barrier.
template <typename WT>
cudaError_t launch_dense_impl(const FfnParams& p0, int sm_count, cudaStream_t s) {
  if (p0.hidden * int(sizeof(WT)) > kStageBytes) return cudaErrorInvalidValue;
  const int grid = std::min(sm_count, p0.n_dense);
  KParams K;
  std::memset(&K, 0, sizeof(K));
  K.err = p0.err;
  K.rows_cap = (p0.n_dense + grid - 1) / grid;
  K.x_elems = p0.hidden;
  for (int b0 = 0; b0 < p0.nb; b0 += kMaxDecodeChunk) {
    FfnParams f = p0;
    f.nb = std::min(kMaxDecodeChunk, p0.nb - b0);
    f.x = reinterpret_cast<const __nv_bfloat16*>(p0.x) + size_t(b0) * p0.hidden;
    if (p0.cache_k) {
      const size_t per_b = size_t(p0.cache_heads) * p0.cache_ctx * p0.cache_rank;
      f.cache_k = reinterpret_cast<__nv_bfloat16*>(p0.cache_k) + size_t(b0) * per_b;
      f.cache_v = reinterpret_cast<__nv_bfloat16*>(p0.cache_v) + size_t(b0) * per_b;
      f.cache_pos = p0.cache_pos + b0;
    } else {
      f.y = reinterpret_cast<__nv_bfloat16*>(p0.y) + size_t(b0) * p0.n_dense;
    }
    K.f = f;
    cudaError_t e = dispatch<WT, __nv_bfloat16, __nv_bfloat16, kDense>(K, f.nb, 1, grid, sm_count, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_ffn(const FfnParams& p, int sm_count, cudaStream_t s) { return launch_ffn_impl(p, sm_count, s); }

cudaError_t launch_dense(const FfnParams& p, lr_dtype_t w_dtype, int sm_count, cudaStream_t s) {
  return w_dtype == LR_BF16 ? launch_dense_impl<__nv_bfloat16>(p, sm_count, s)
                            : launch_dense_impl<int8_t>(p, sm_count, s);
}

}  // namespace lr
