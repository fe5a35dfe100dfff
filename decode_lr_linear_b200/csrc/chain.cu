// Chains of dependent factorised linears in one persistent launch, sm_100a.
//
// A chain is a list of steps.  Step s evaluates up to four factorised linears
// y_p = (x_s A_p) B_p ("Low-Rank Approximation of Large Language Models",
// factorised layer W ~ A B) that share their input x_s: the chain input, the
// fp32 result of the previous step, or the stored output of an older step.
// Factors are stored latent-major (A as [rank, d_in], B as [rank, d_out]), so
// y_p = sum_j (x_s . a_j) b_j and a prefix of the rows is a lower-rank model.
//
// One CTA per SM at most (all resident).  Each CTA owns a contiguous block of
// the step's latent rows (the projections' rows concatenated).  A producer
// warp streams the CTA's rows of every step, A rows then B rows, through a
// ring of shared-memory stages with bulk copies (cp.async.bulk completing on
// mbarriers).  It never waits for a step boundary, only for a free stage, so
// DRAM keeps streaming the next steps' rows while the CTA waits for an input.
// Sixteen consumer warps, per step:
//   input    wait until every CTA has finished the step this one reads (one
//            completion counter per step, bounded in time; every CTA is
//            resident, which the launch checks), then load x in fp32: the
//            chain input, or the input step's fp32 accumulator;
//   phase A  z_j = x_s . a_j: warp w takes line w (512 bytes) of every row in
//            a stage, keeps x in registers, reduces the stage's rows with one
//            butterfly and adds its line sums into z in shared memory;
//   phase B  y_p += z_j b_j: warp w takes line w of every B row and keeps the
//            output line in registers, adding it into the step's own fp32
//            accumulator (red.global.add.v4.f32) when a projection's rows end;
//   done     thread 0 adds one to the step's completion counter (release).
// A step waits only for the step it reads: a step whose input is already
// complete (for example K and Q next to V, which O reads) starts at once, so
// independent work covers the hand-off of a dependent one.  Every step keeps
// its own accumulators, so nothing is reused within a launch; after the last
// step each CTA writes its share of every step's outputs and clears those
// accumulators, and the last CTA to leave resets the counters, so the
// workspace is all zero between calls.
#include <algorithm>
#include <cstring>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace lr {
namespace {

constexpr int kWarps = 16;                 // consumer warps
constexpr int kConsumers = kWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + the producer warp
constexpr int kLineBytes = 512;            // one warp-wide line: 16 bytes per lane
constexpr int kStageBytes = 64 * 1024;
constexpr int kStages = 3;
constexpr size_t kSmemLimit = 227 * 1024;

// 16 bytes of weights -> fp32.
template <typename WT> struct Lane16;
template <> struct Lane16<__nv_bfloat16> {
  static constexpr int kElems = 8;
  LR_DEV static void cvt(const uint4 v, float* f) { bf16x8_to_f32(v, f); }
};
template <> struct Lane16<float> {
  static constexpr int kElems = 4;
  LR_DEV static void cvt(const uint4 v, float* f) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
};
template <> struct Lane16<int8_t> {
  static constexpr int kElems = 16;
  LR_DEV static void cvt(const uint4 v, float* f) {
    i8x8_to_f32(make_uint2(v.x, v.y), f);
    i8x8_to_f32(make_uint2(v.z, v.w), f + 8);
  }
};

// Compile-time shape of one instantiation: NB batch rows, up to L lines of a
// row per warp.  A stage holds at most GR rows; GR * NB <= 16 values are
// reduced by one butterfly.
template <typename WT, int NB, int L>
struct Cfg {
  static constexpr int EPC = Lane16<WT>::kElems;
  static constexpr int GR0 = 8 / L < 16 / NB ? 8 / L : 16 / NB;
  static constexpr int GR = GR0 < 1 ? 1 : GR0;
};

LR_HD_INLINE int ceil_div(int a, int b) { return (a + b - 1) / b; }

// [a, b) of `total` items for part `part` of `parts` (total * parts < 2^31:
// rows and 8-float chunks of one step over at most one CTA per SM).
LR_DEV void split_range(int total, int part, int parts, int* a, int* b) {
  *a = int(unsigned(total) * unsigned(part) / unsigned(parts));
  *b = int(unsigned(total) * unsigned(part + 1) / unsigned(parts));
}

// How the warps cover rows of `row_bytes`: wpr warps per row (a power of two,
// at most kWarps) and rs = kWarps / wpr rows side by side.  Warp w reads lines
// line0 + wpr * i of the stage's rows slot, slot + rs, ...
struct WarpMap {
  int wpr, rs, slot, line0;
};

LR_DEV WarpMap warp_map(int row_bytes) {
  const int lines = ceil_div(row_bytes, kLineBytes);
  int wpr = 1;
  while (wpr < lines && wpr < kWarps) wpr <<= 1;
  const int warp = threadIdx.x >> 5;
  WarpMap m;
  m.wpr = wpr;
  m.rs = kWarps / wpr;
  m.slot = warp / wpr;
  m.line0 = warp % wpr;
  return m;
}

LR_DEV void consumer_sync() { asm volatile("bar.sync 1, %0;" :: "r"(kConsumers) : "memory"); }

LR_DEV uint4 lds128(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }

LR_DEV void red_release_add(unsigned int* p, unsigned int v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

LR_DEV int acc_offset(const ChainStep& st, int p, int nb) {
  int o = 0;
  for (int q = 0; q < p; ++q) o += nb * st.p[q].d_out;
  return o;
}


// This CTA's segments of step S for one kind (0: A rows, 1: B rows), in
// projection order: f(p, src, row_bytes, z0, j0, rows) with z0 the CTA-local
// index of the first row and j0 its index within projection p.
template <typename WT, class F>
LR_DEV void for_segments(const ChainStep& S, int kind, F&& f) {
  int r0, r1;
  split_range(S.total_rows, blockIdx.x, gridDim.x, &r0, &r1);
  int begin = 0;
  for (int p = 0; p < S.n; ++p) {
    const ChainProj& pr = S.p[p];
    const int a = max(r0, begin), b = min(r1, begin + pr.rows);
    if (a < b) {
      const int row_bytes = (kind == 0 ? S.d_in : pr.d_out) * int(sizeof(WT));
      const unsigned char* src =
          reinterpret_cast<const unsigned char*>(kind == 0 ? pr.A : pr.B) + size_t(a - begin) * row_bytes;
      f(p, src, row_bytes, a - r0, a - begin, b - a);
    }
    begin += pr.rows;
  }
}

LR_HD_INLINE int stage_rows(int row_bytes, int gr) {
  const int r = kStageBytes / row_bytes;
  return r < 1 ? 1 : (r < gr ? r : gr);
}

// Producer: every stage of every step, in the consumers' order.
template <typename WT, int GR>
LR_DEV void produce(const ChainParams& P, unsigned char* ring, uint64_t* full, uint64_t* empty) {
  int st = 0;
  bool ok = true;
  for (int s = 0; s < P.n_steps && ok; ++s) {
    for (int kind = 0; kind < 2 && ok; ++kind) {
      for_segments<WT>(P.step[s], kind, [&](int, const unsigned char* src, int row_bytes, int, int, int rows) {
        const int rps = stage_rows(row_bytes, GR);
        for (int r = 0; r < rows && ok; r += rps) {
          const int k = min(rps, rows - r);
          const int slot = st % kStages, round = st / kStages;
          if (round > 0 && !mbar_wait_bounded(&empty[slot], uint32_t(round - 1) & 1u, P.err)) {
            ok = false;
            return;
          }
          const uint32_t bytes = uint32_t(k) * uint32_t(row_bytes);
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_g2s(ring + size_t(slot) * kStageBytes, src + size_t(r) * row_bytes, bytes, &full[slot]);
          ++st;
        }
      });
    }
  }
}

// ---- butterfly reduction of V values over the warp ------------------------
// Each exchange halves the values a lane holds: the lane whose bit m is set
// keeps the upper half and sends the lower one (its partner the reverse), so
// after log2(V) exchanges a lane holds one value summed over the lanes that
// differ in those bits; plain xor steps finish the sum.  Returns the total of
// value bfly_index<V>(lane); lanes with (lane & (32 / V - 1)) == 0 report it.
template <int V> struct Log2 { static constexpr int value = 1 + Log2<V / 2>::value; };
template <> struct Log2<1> { static constexpr int value = 0; };

template <int V>
LR_DEV float warp_reduce_scatter(float (&v)[V], int lane) {
  constexpr int S = Log2<V>::value;
#pragma unroll
  for (int st = 0; st < S; ++st) {
    const int m = 16 >> st;
    const int half = V >> (st + 1);
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
  float t = v[0];
#pragma unroll
  for (int m = 16 >> S; m > 0; m >>= 1) t += __shfl_xor_sync(0xffffffffu, t, m);
  return t;
}

template <int V>
LR_DEV int bfly_index(int lane) {
  constexpr int S = Log2<V>::value;
  int vi = 0;
#pragma unroll
  for (int st = 0; st < S; ++st) vi |= ((lane >> (4 - st)) & 1) << (S - 1 - st);
  return vi;
}

// ---- the step's input for this lane's columns (fp32 registers) ------------
// Chain input: the caller's x (bf16, or fp32 for fp32 weights).  An earlier
// step: its fp32 accumulator (times the int8 output scale).
template <typename WT, int NB, int L>
LR_DEV void load_x(const ChainParams& P, int s, const WarpMap& m, float (&xr)[L][NB][Lane16<WT>::kElems],
                   int lane) {
  using XT = typename std::conditional<sizeof(WT) == 4, float, __nv_bfloat16>::type;
  constexpr int EPC = Lane16<WT>::kElems;
  const ChainStep& S = P.step[s];
  const int d_in = S.d_in;
  const bool f16 = P.scale_f16 != 0;
#pragma unroll
  for (int li = 0; li < L; ++li) {
    const int off = (m.line0 + m.wpr * li) * kLineBytes + lane * 16;
    const int col = off / int(sizeof(WT));
    const bool valid = off < d_in * int(sizeof(WT));
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float* f = xr[li][b];
#pragma unroll
      for (int e = 0; e < EPC; ++e) f[e] = 0.f;
      if (!valid || b >= P.nb) continue;
      const size_t idx = size_t(b) * d_in + col;
      if (S.input_step >= 0) {
        const ChainStep& I = P.step[S.input_step];
        const float* a = P.acc + I.acc_off + acc_offset(I, S.input_proj, P.nb) + idx;
#pragma unroll
        for (int q = 0; q < EPC; q += 4) {
          const float4 v = ld_cg_f4(a + q);
          f[q] = v.x; f[q + 1] = v.y; f[q + 2] = v.z; f[q + 3] = v.w;
        }
        const void* sB = I.p[S.input_proj].sB;
        if (sB) {
#pragma unroll
          for (int e = 0; e < EPC; ++e) f[e] *= load_scale(sB, col + e, f16);
        }
      } else {
        const XT* src = reinterpret_cast<const XT*>(P.x);
        if constexpr (sizeof(XT) == 4) {
          const float4 v = ld_cg_f4(src + idx);
          f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
#pragma unroll
          for (int q = 0; q < EPC; q += 8) bf16x8_to_f32(ld_cg_u4(src + idx + q), f + q);
        }
      }
    }
  }
}

// ---- outputs of step t: this CTA's 1/gridDim share of the 8-float chunks ----
LR_DEV void out_range(const ChainParams& P, int t, int* c0, int* c1) {
  const ChainStep& S = P.step[t];
  split_range(acc_offset(S, S.n, P.nb) / 8, blockIdx.x, gridDim.x, c0, c1);
}

// Accumulator address of chunk c of step t and its projection / offset.
LR_DEV float* out_locate(const ChainParams& P, int t, int c, int* p_out, int* off_out) {
  const ChainStep& S = P.step[t];
  const int nb = P.nb;
  int off = c * 8, p = 0, base = 0;
  while (p < S.n - 1 && off >= nb * S.p[p].d_out) {
    off -= nb * S.p[p].d_out;
    base += nb * S.p[p].d_out;
    ++p;
  }
  *p_out = p;
  *off_out = off;
  return P.acc + S.acc_off + base + off;
}

// This CTA's share of step t's outputs: scale, round, store; clear the accumulators read.
template <typename YT>
LR_DEV void write_outputs(const ChainParams& P, int t) {
  const bool f16 = P.scale_f16 != 0;
  int c0, c1;
  out_range(P, t, &c0, &c1);
  for (int c = c0 + int(threadIdx.x); c < c1; c += kConsumers) {
    int p, off;
    float* a = out_locate(P, t, c, &p, &off);
    const ChainProj& pr = P.step[t].p[p];
    const float4 v0 = ld_cg_f4(a), v1 = ld_cg_f4(a + 4);
    float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    if (pr.sB) {
      const int k = off % pr.d_out;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= load_scale(pr.sB, k + e, f16);
    }
    YT* y = reinterpret_cast<YT*>(pr.y) + off;
    if constexpr (sizeof(YT) == 2) {
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        ow[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(y) = o;
    } else {
      *reinterpret_cast<float4*>(y) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(y + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
    st_cg_f4(a, make_float4(0.f, 0.f, 0.f, 0.f));
    st_cg_f4(a + 4, make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

// Add this warp's output lines of one projection into its accumulator.
template <typename WT, int NB, int L>
LR_DEV void flush_lines(float (&acc)[L][NB][Lane16<WT>::kElems], float* dst, int bbytes, int nb, const WarpMap& m,
                        int lane) {
  constexpr int EPC = Lane16<WT>::kElems;
  const int d_out = bbytes / int(sizeof(WT));
#pragma unroll
  for (int li = 0; li < L; ++li) {
    const int off = (m.line0 + m.wpr * li) * kLineBytes + lane * 16;
    if (off < bbytes) {
      const int col = off / int(sizeof(WT));
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < nb) {
#pragma unroll
          for (int q = 0; q < EPC; q += 4)
            red_add_f4(dst + size_t(b) * d_out + col + q, acc[li][b][q], acc[li][b][q + 1], acc[li][b][q + 2],
                       acc[li][b][q + 3]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < EPC; ++e) acc[li][b][e] = 0.f;
  }
}

// Wait for a ring stage.  After a first mbarrier timeout the CTA stops
// computing but keeps to the protocol, with a short bound per stage, so that
// no copy it issued is left in flight into its shared memory.
LR_DEV const unsigned char* stage_acquire(unsigned char* ring, uint64_t* full, int st, bool* failed, int* err) {
  const int slot = st % kStages;
  const uint32_t parity = uint32_t(st / kStages) & 1u;
  if (!*failed) {
    if (!mbar_wait_bounded(&full[slot], parity, err)) *failed = true;
  } else {
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(&full[slot], parity) && global_ns() - t0 < kDegradedMbarNs) {
    }
  }
  return ring + size_t(slot) * kStageBytes;
}

LR_DEV void stage_release(uint64_t* empty, int st) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[st % kStages]);
}

template <typename WT, int NB, int L>
__global__ void __launch_bounds__(kThreads, 1) chain_kernel(const __grid_constant__ ChainParams P, int rows_cap) {
  using C = Cfg<WT, NB, L>;
  using YT = typename std::conditional<sizeof(WT) == 4, float, __nv_bfloat16>::type;
  constexpr int EPC = C::EPC, GR = C::GR, V = GR * NB;
  static_assert(V <= 32, "butterfly width");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t empty[kStages];
  unsigned char* ring = smem;
  float* zs = reinterpret_cast<float*>(smem + size_t(kStages) * kStageBytes);  // [rows_cap][NB]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = P.nb;
  const bool f16 = P.scale_f16 != 0;

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < rows_cap * NB; i += kThreads) zs[i] = 0.f;
  __syncthreads();

  if (warp == kWarps) {
    // weights are not written by the preceding kernel: no dependency wait
    if (lane == 0) produce<WT, GR>(P, ring, full, empty);
    return;
  }

  pdl_wait();
  int st = 0;
  bool failed = false;
  for (int s = 0; s < P.n_steps; ++s) {
    const ChainStep& S = P.step[s];
    // ---- the step's input: wait for the step it reads, then load it ----
    if (S.input_step >= 0) {
      if (threadIdx.x == 0) wait_counter_geq(P.bar + S.input_step, gridDim.x, P.wait_ns, P.err);
      consumer_sync();
    }
    const WarpMap ma = warp_map(S.d_in * int(sizeof(WT)));
    float xr[L][NB][EPC];
    load_x<WT, NB, L>(P, s, ma, xr, lane);

    // ---- phase A: z_j = x . a_j ----
    for_segments<WT>(S, 0, [&](int p, const unsigned char*, int row_bytes, int z0, int j0, int rows) {
      const int rps = stage_rows(row_bytes, GR);
      const void* sA = S.p[p].sA;
      for (int r = 0; r < rows; r += rps) {
        const int k = min(rps, rows - r);
        const unsigned char* stage = stage_acquire(ring, full, st, &failed, P.err);
        if (!failed) {
          float v[V];
#pragma unroll
          for (int i = 0; i < V; ++i) v[i] = 0.f;
#pragma unroll
          for (int uu = 0; uu < GR; ++uu) {
            const int u = ma.slot + ma.rs * uu;
            if (u < k) {
#pragma unroll
              for (int li = 0; li < L; ++li) {
                const int off = (ma.line0 + ma.wpr * li) * kLineBytes + lane * 16;
                if (off < row_bytes) {
                  float w[EPC];
                  Lane16<WT>::cvt(lds128(stage + size_t(u) * row_bytes + off), w);
#pragma unroll
                  for (int b = 0; b < NB; ++b) {
                    float a0 = 0.f, a1 = 0.f;
#pragma unroll
                    for (int e = 0; e < EPC; e += 2) {
                      a0 = fmaf(w[e], xr[li][b][e], a0);
                      a1 = fmaf(w[e + 1], xr[li][b][e + 1], a1);
                    }
                    v[uu * NB + b] += a0 + a1;
                  }
                }
              }
            }
          }
          const float t = warp_reduce_scatter<V>(v, lane);
          const int vi = bfly_index<V>(lane);
          const int u = ma.slot + ma.rs * (vi / NB), b = vi % NB;
          if ((lane & (32 / V - 1)) == 0 && u < k && b < nb) {
            const float sc = sA ? load_scale(sA, j0 + r + u, f16) : 1.f;
            atomicAdd(zs + (z0 + r + u) * NB + b, t * sc);
          }
        }
        stage_release(empty, st);
        ++st;
      }
    });
    consumer_sync();  // z complete

    // ---- phase B: y += z_j b_j ----
    float* acc_set = P.acc + S.acc_off;
    for_segments<WT>(S, 1, [&](int p, const unsigned char*, int row_bytes, int z0, int, int rows) {
      const WarpMap mb = warp_map(row_bytes);
      const int rps = stage_rows(row_bytes, GR);
      float acc[L][NB][EPC];
#pragma unroll
      for (int li = 0; li < L; ++li)
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int e = 0; e < EPC; ++e) acc[li][b][e] = 0.f;
      for (int r = 0; r < rows; r += rps) {
        const int k = min(rps, rows - r);
        const unsigned char* stage = stage_acquire(ring, full, st, &failed, P.err);
        if (!failed) {
#pragma unroll
          for (int uu = 0; uu < GR; ++uu) {
            const int u = mb.slot + mb.rs * uu;
            if (u < k) {
              float zb[NB];
#pragma unroll
              for (int b = 0; b < NB; ++b) zb[b] = zs[(z0 + r + u) * NB + b];
#pragma unroll
              for (int li = 0; li < L; ++li) {
                const int off = (mb.line0 + mb.wpr * li) * kLineBytes + lane * 16;
                if (off < row_bytes) {
                  float w[EPC];
                  Lane16<WT>::cvt(lds128(stage + size_t(u) * row_bytes + off), w);
#pragma unroll
                  for (int b = 0; b < NB; ++b)
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[li][b][e] = fmaf(zb[b], w[e], acc[li][b][e]);
                }
              }
            }
          }
        }
        stage_release(empty, st);
        ++st;
      }
      if (!failed) flush_lines<WT, NB, L>(acc, acc_set + acc_offset(S, p, nb), row_bytes, nb, mb, lane);
    });

    // ---- step s done: all of this CTA's partial outputs of step s are issued ----
    consumer_sync();
    for (int i = threadIdx.x; i < rows_cap * NB; i += kConsumers) zs[i] = 0.f;
    if (threadIdx.x == 0) red_release_add(P.bar + s, 1u);
    consumer_sync();
  }

  // ---- every step's outputs (the last step completes after all others); clear ----
  if (threadIdx.x == 0) wait_counter_geq(P.bar + (P.n_steps - 1), gridDim.x, P.wait_ns, P.err);
  consumer_sync();
  for (int t = 0; t < P.n_steps; ++t) write_outputs<YT>(P, t);
  consumer_sync();
  if (threadIdx.x == 0) {
    __threadfence();
    unsigned int* exit_count = P.bar + P.n_steps;
    const unsigned prev = atomicAdd(exit_count, 1u);
    if (prev == gridDim.x - 1) {
      for (int t = 0; t <= P.n_steps; ++t) atomicExch(P.bar + t, 0u);
    }
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int NB>
size_t chain_smem(int rows_cap) {
  return size_t(kStages) * kStageBytes + size_t(rows_cap) * NB * sizeof(float);
}

template <typename WT, int NB, int L>
cudaError_t launch_chain_t(const ChainParams& p, int grid, int rows_cap, int sm_count, cudaStream_t s) {
  const size_t bytes = chain_smem<NB>(rows_cap);
  if (bytes > kSmemLimit - 1024) return cudaErrorInvalidValue;
  auto kern = chain_kernel<WT, NB, L>;
  cudaError_t e = ensure_smem(kern, bytes);
  if (e != cudaSuccess) return e;
  e = check_resident(reinterpret_cast<const void*>(kern), kThreads, bytes, grid, sm_count);
  if (e != cudaSuccess) return e;
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
  return cudaLaunchKernelEx(&cfg, kern, p, rows_cap);
}

// Largest batch rows one launch takes for L lines per warp: NB * L <= 8 and
// at most 64 fp32 accumulator registers (NB * L * elements per lane).
template <typename WT>
constexpr int nb_max_for(int L) {
  const int a = 8 / L, b = 64 / (L * Lane16<WT>::kElems);
  const int m = a < b ? a : b;
  return m >= 8 ? 8 : m >= 4 ? 4 : m >= 2 ? 2 : 1;
}

template <typename WT, int L>
cudaError_t launch_chain_nb(const ChainParams& p, int grid, int rows_cap, int sm_count, cudaStream_t s) {
  constexpr int kMaxNb = nb_max_for<WT>(L);
  if (p.nb <= 1) return launch_chain_t<WT, 1, L>(p, grid, rows_cap, sm_count, s);
  if (p.nb <= 2 && kMaxNb >= 2) return launch_chain_t<WT, (kMaxNb >= 2 ? 2 : 1), L>(p, grid, rows_cap, sm_count, s);
  if (p.nb <= 4 && kMaxNb >= 4) return launch_chain_t<WT, (kMaxNb >= 4 ? 4 : 1), L>(p, grid, rows_cap, sm_count, s);
  if (p.nb <= 8 && kMaxNb >= 8) return launch_chain_t<WT, (kMaxNb >= 8 ? 8 : 1), L>(p, grid, rows_cap, sm_count, s);
  return cudaErrorInvalidValue;
}

template <typename WT>
cudaError_t launch_chain_w(const ChainParams& p0, int sm_count, cudaStream_t s) {
  using XT = typename std::conditional<sizeof(WT) == 4, float, __nv_bfloat16>::type;
  int max_lines = 1, max_rows = 0, x_width = 0;
  for (int i = 0; i < p0.n_steps; ++i) {
    const ChainStep& st = p0.step[i];
    max_lines = std::max(max_lines, ceil_div(st.d_in * int(sizeof(WT)), kLineBytes));
    for (int q = 0; q < st.n; ++q)
      max_lines = std::max(max_lines, ceil_div(st.p[q].d_out * int(sizeof(WT)), kLineBytes));
    max_rows = std::max(max_rows, st.total_rows);
    if (st.input_step < 0) x_width = st.d_in;
  }
  const int lpw = ceil_div(max_lines, kWarps);
  const int L = lpw <= 1 ? 1 : lpw <= 2 ? 2 : lpw <= 4 ? 4 : 0;
  if (L == 0) return cudaErrorInvalidValue;
  const int grid = std::min(sm_count, std::max(max_rows, 1));
  const int rows_cap = std::max(1, ceil_div(max_rows, grid));
  const int piece = L == 1 ? nb_max_for<WT>(1) : L == 2 ? nb_max_for<WT>(2) : nb_max_for<WT>(4);
  static ChainParams P;  // large; launches are issued under the caller's lock
  for (int b0 = 0; b0 < p0.nb; b0 += piece) {
    std::memcpy(&P, &p0, sizeof(P));
    P.nb = std::min(piece, p0.nb - b0);
    P.x = reinterpret_cast<const XT*>(p0.x) + size_t(b0) * x_width;
    for (int i = 0; i < P.n_steps; ++i)
      for (int q = 0; q < P.step[i].n; ++q)
        P.step[i].p[q].y = reinterpret_cast<XT*>(p0.step[i].p[q].y) + size_t(b0) * p0.step[i].p[q].d_out;
    cudaError_t e = L == 1   ? launch_chain_nb<WT, 1>(P, grid, rows_cap, sm_count, s)
                    : L == 2 ? launch_chain_nb<WT, 2>(P, grid, rows_cap, sm_count, s)
                             : launch_chain_nb<WT, 4>(P, grid, rows_cap, sm_count, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace


cudaError_t launch_chain(const ChainParams& p, lr_dtype_t w_dtype, int sm_count, cudaStream_t s) {
  switch (w_dtype) {
    case LR_F32: return launch_chain_w<float>(p, sm_count, s);
    case LR_BF16: return launch_chain_w<__nv_bfloat16>(p, sm_count, s);
    case LR_I8: return launch_chain_w<int8_t>(p, sm_count, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lr
