// Latent-KV flash decoding with the keys reconstructed on chip (tensor cores),
// so that a rotary position embedding can act on them, sm_100a.
//
// WSVD "Fine-Grained Per-Head SVD": the cache of head h keeps the latent
// C_K,t (rank r) instead of the key, K_t = C_K,t B_K,h.  WSVD "Quantization-
// Aware Training (QAT) en Fused Kernel": the reconstruction runs inside the
// flash-decoding pipeline and K never reaches global memory.  With a rotary
// embedding (the LLaMA convention of the pages' models: dimension i turns with
// i + 64 by pos * theta_i) the score of token t is
//   s_t = RoPE(q, p) . RoPE(K_t, t) = sum_i cos(d theta_i) P_i + sin(d theta_i) Q_i,
//   d = t - p,  P_i = q_i k_i + q_{i+64} k_{i+64},  Q_i = q_{i+64} k_i - q_i k_{i+64},
// which depends on t through the rotation, so the query cannot be absorbed
// into B_K once for all tokens.  The kernel reconstructs, per tile of 128
// cached tokens, G = C_K,tile U'^T on the tensor cores (tcgen05.mma kind::f16,
// M = 128 tokens, N = 128, K = r = 32, fp32 accumulator in tensor memory),
// where U' is B_K with the query pairs and the tile's base rotation folded in
// (rows u'_i = C0_i u_i + S0_i w_i and w'_i = C0_i w_i - S0_i u_i, with
// u_i = q_i B_K[:, i] + q_{i+64} B_K[:, i+64], w_i = q_{i+64} B_K[:, i] -
// q_i B_K[:, i+64], (C0_i, S0_i) = cos/sin((t0 - p) theta_i)); then the
// thread that owns token t0 + j finishes the rotation with its own
// coefficients: s_t = sum_i cos(j theta_i) G[i] + sin(j theta_i) G[64 + i].
// Values carry no rotation: the softmax-weighted latent values are averaged
// on CUDA cores and B_V is applied once per (batch, head) by the combine
// kernel of the absorbed path.
//
// Persistent CTAs (two per SM) each take a contiguous range of work items
// (batch, head, 256-token split), so the query folded into B_K is recomputed
// only when the (batch, head) pair changes; only the tile's base rotation is
// new per item.  Thread 0 keeps one item ahead in a two-stage ring: each stage
// holds the item's C_K tiles (tiled copies with the 64-byte swizzle the MMA
// operand descriptor expects) and its C_V rows (one bulk copy), completing on
// one mbarrier.  Every wait is bounded and records a device error instead of
// hanging.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace lr {
namespace {

constexpr int kR = 32;                       // latent rank per head
constexpr int kD = 128;                      // head dim
constexpr int kHalf = kD / 2;                // rotary frequencies
constexpr int kTile = 128;                   // tokens per MMA (tensor-memory lanes)
constexpr int kSplit = 2 * kTile;            // tokens per work item
constexpr int kStages = 2;
constexpr int kThreads = 128;
constexpr int kTileBytes = kTile * kR * 2;   // 8 KiB: one C_K tile, or one U' tile (128 rows of 64 B)
constexpr int kCkBytes = 2 * kTileBytes;
constexpr int kCvBytes = kSplit * kR * 2;
constexpr int kStageBytes = kCkBytes + kCvBytes;
constexpr int kUBytes = 2 * kTileBytes;
constexpr int kTmemCols = 2 * kTile;         // one 128-column fp32 accumulator per tile
constexpr int kPart = kR + 2;                // m, l, acc[r]
constexpr float kLog2e = 1.4426950408889634f;
constexpr size_t kDynSmem = size_t(kStages) * kStageBytes + kUBytes + 1024;

struct Item {
  int b, h, split, n_ctx, n;  // n: tokens of the item that are in the context (<= 0: none)
};

LR_DEV Item item_at(const LatentKvParams& P, int item) {
  Item it;
  it.split = item % P.n_splits;
  const int bh = item / P.n_splits;
  it.h = bh % P.heads;
  it.b = bh / P.heads;
  int n_ctx = P.seq_lens[it.b];
  it.n_ctx = n_ctx < 0 ? 0 : (n_ctx > P.max_ctx ? P.max_ctx : n_ctx);
  it.n = min(kSplit, it.n_ctx - it.split * kSplit);
  return it;
}

// Byte offset of the 16-byte chunk `c` (0..3) of row `row` in a 64-byte-swizzled
// K-major operand tile (rows of 64 bytes; the chunk index is XORed with bits 1..2
// of the row, the layout the tensor copy writes and the descriptor reads).
LR_DEV uint32_t sw64_offset(int row, int c) { return uint32_t(row) * 64u + uint32_t((c ^ ((row >> 1) & 3)) * 16); }

__global__ void __launch_bounds__(kThreads, 2) latent_kv_rope_kernel(const __grid_constant__ CUtensorMap mapK,
                                                                     const __grid_constant__ KvRopeParams R) {
  const LatentKvParams& P = R.p;
  extern __shared__ unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ float sc[kSplit];
  __shared__ float base_cs[2][2][kHalf];     // [tile][cos, sin][i]
  __shared__ float accs[kThreads / 4][kR + 1];
  __shared__ float red[kThreads / 32];

  // operand tiles on 1024-byte boundaries (the swizzle pattern repeats every 512 bytes)
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  const uint32_t ubuf = base + uint32_t(kStages) * kStageBytes;
  unsigned char* ubuf_g = gbase + size_t(kStages) * kStageBytes;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    mbar_init(&mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_launch_dependents();

  // The rotation of a token by its offset j inside a tile: cf[i] = cos(j theta_i),
  // cf[64 + i] = sin(j theta_i), in the order of the accumulator columns.
  const int j = warp * 32 + lane;   // this thread's tensor-memory lane = token offset in a tile
  float cf[kD];
#pragma unroll
  for (int i = 0; i < kHalf; ++i) sincosf(float(j) * R.theta_f[i], &cf[kHalf + i], &cf[i]);

  const int n_items = P.batch * P.heads * P.n_splits;
  const int item_lo = int((long long)n_items * blockIdx.x / gridDim.x);
  const int item_hi = int((long long)n_items * (blockIdx.x + 1) / gridDim.x);
  const uint32_t idesc = tc::idesc_bf16(kTile, kD, false, false);

  // q, the caches and the lengths may come from the preceding kernel
  pdl_wait();

  // ---- producer state (thread 0): the next item to load and the loads issued ----
  int pc = item_lo, issued = 0;
  auto issue_next = [&]() {
    while (pc < item_hi) {
      const int item = pc++;
      const Item it = item_at(P, item);
      if (it.n <= 0) continue;
      const int st = issued % kStages;
      const size_t row0 = (size_t(it.b) * P.heads + it.h) * P.max_ctx + size_t(it.split) * kSplit;
      const uint32_t ck = base + uint32_t(st) * kStageBytes;
      mbar_arrive_expect_tx(&full[st], uint32_t(kCkBytes + it.n * kR * 2));
      tc::tma_load_2d(ck, &mapK, 0, int(row0), &full[st]);
      tc::tma_load_2d(ck + kTileBytes, &mapK, 0, int(row0 + kTile), &full[st]);
      bulk_g2s(gbase + size_t(st) * kStageBytes + kCkBytes,
               reinterpret_cast<const __nv_bfloat16*>(P.CV) + row0 * kR, uint32_t(it.n * kR * 2), &full[st]);
      ++issued;
      return;
    }
  };
  if (tid == 0) issue_next();

  int L = 0;  // loading items consumed
  bool failed = false;
  int cur_bh = -1;  // the (batch, head) whose query factors uu, ww hold
  const int fi = tid & (kHalf - 1), kh = tid >> 6;  // frequency i, latent dims [16 kh, 16 kh + 16)
  float uu[16], ww[16];
  for (int item = item_lo; item < item_hi; ++item) {
    const Item it = item_at(P, item);
    float* outp = P.partial + size_t(item) * kPart;
    if (it.n <= 0) {
      if (tid < kPart) outp[tid] = tid == 0 ? -INFINITY : 0.f;
      continue;
    }
    const int st = L % kStages;
    const uint32_t par = uint32_t(L / kStages) & 1u;
    // the stage of the item after this one was released at the end of the previous item
    if (tid == 0) issue_next();

    // ---- base rotations of the two tiles, and this thread's query factors ----
    const int p = it.n_ctx - 1;  // the query sits at the newest cached position
    {
      // angle (t0 - p) theta_i, reduced to [-pi, pi] in double, then the fp32 sine and cosine
      const int i = tid & (kHalf - 1), u = tid >> 6;
      constexpr double kTwoPi = 6.283185307179586;
      const double a = double(it.split * kSplit + u * kTile - p) * R.theta_d[i];
      const float ar = float(a - rint(a * (1.0 / kTwoPi)) * kTwoPi);
      float sn, cs;
      sincosf(ar, &sn, &cs);
      base_cs[u][0][i] = cs;
      base_cs[u][1][i] = sn;
    }
    const int bh = it.b * P.heads + it.h;
    if (bh != cur_bh) {
      cur_bh = bh;
      const __nv_bfloat16* qv = reinterpret_cast<const __nv_bfloat16*>(P.q) + (size_t(it.b) * P.heads + it.h) * kD;
      const float qs = P.scale * kLog2e;
      const float q1 = __bfloat162float(qv[fi]) * qs, q2 = __bfloat162float(qv[fi + kHalf]) * qs;
      const __nv_bfloat16* bk = reinterpret_cast<const __nv_bfloat16*>(P.BK) + size_t(it.h) * kR * kD;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int k = kh * 16 + e;
        const float b1 = __bfloat162float(bk[k * kD + fi]), b2 = __bfloat162float(bk[k * kD + fi + kHalf]);
        uu[e] = fmaf(q1, b1, q2 * b2);
        ww[e] = fmaf(q2, b1, -(q1 * b2));
      }
    }
    __syncthreads();
    // ---- U' of both tiles: rows fi (u') and 64 + fi (w'), two 16-byte chunks each ----
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float C = base_cs[u][0][fi], S = base_cs[u][1][fi];
      unsigned char* ut = ubuf_g + u * kTileBytes;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pu[4], pw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int a = c * 8 + 2 * e;
          __nv_bfloat162 hu = __floats2bfloat162_rn(fmaf(C, uu[a], S * ww[a]), fmaf(C, uu[a + 1], S * ww[a + 1]));
          __nv_bfloat162 hw = __floats2bfloat162_rn(fmaf(C, ww[a], -(S * uu[a])), fmaf(C, ww[a + 1], -(S * uu[a + 1])));
          pu[e] = *reinterpret_cast<uint32_t*>(&hu);
          pw[e] = *reinterpret_cast<uint32_t*>(&hw);
        }
        const int chunk = kh * 2 + c;
        *reinterpret_cast<uint4*>(ut + sw64_offset(fi, chunk)) = make_uint4(pu[0], pu[1], pu[2], pu[3]);
        *reinterpret_cast<uint4*>(ut + sw64_offset(fi + kHalf, chunk)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
    }
    fence_proxy_async();  // the generic-proxy writes of U' before the tensor cores read them
    // ---- the stage has landed (every thread: its C_V rows are read below) ----
    if (__syncthreads_or(!mbar_wait_bounded(&full[st], par, P.err))) {
      failed = true;
      break;
    }
    if (tid == 0) {
      tc::fence_after();
      const uint32_t ck = base + uint32_t(st) * kStageBytes;
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int kk = 0; kk < kR / 16; ++kk) {
          const uint64_t ad = tc::smem_desc(ck + u * kTileBytes + kk * 32, 16, 512, tc::kSwizzle64B);
          const uint64_t bd = tc::smem_desc(ubuf + u * kTileBytes + kk * 32, 16, 512, tc::kSwizzle64B);
          tc::mma_f16(tmem + uint32_t(u * kTile), ad, bd, idesc, kk > 0);
        }
      tc::mma_commit(&mma_done);
    }
    // ---- scores: this thread's token of each tile ----
    const bool mma_ok = mbar_wait_bounded(&mma_done, uint32_t(L) & 1u, P.err);
    tc::fence_after();
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t ta = tmem + (uint32_t(warp * 32) << 16) + uint32_t(u * kTile);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t v[32];
        tc::tmem_ld32(ta + uint32_t(c * 32), v);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          s0 = fmaf(cf[c * 32 + e], __uint_as_float(v[e]), s0);
          s1 = fmaf(cf[c * 32 + e + 1], __uint_as_float(v[e + 1]), s1);
        }
      }
      const int tk = u * kTile + j;
      sc[tk] = tk < it.n ? s0 + s1 : -INFINITY;
    }
    tc::fence_before();
    if (__syncthreads_or(!mma_ok)) {
      failed = true;
      break;
    }

    // ---- softmax over the item and the weighted latent value ----
    float m = warp_max(fmaxf(sc[tid], sc[tid + kThreads]));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const int tg = tid >> 2, part = tid & 3;
    const __nv_bfloat16* cv =
        reinterpret_cast<const __nv_bfloat16*>(gbase + size_t(st) * kStageBytes + kCkBytes);
    float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float lsum = 0.f;
    for (int tk = tg; tk < it.n; tk += kThreads / 4) {
      const float w = exp2f(sc[tk] - m);
      lsum += w;
      float c[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(cv + size_t(tk) * kR + part * 8), c);
#pragma unroll
      for (int e = 0; e < 8; ++e) a8[e] = fmaf(w, c[e], a8[e]);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) accs[tg][part * 8 + e] = a8[e];
    if (part == 0) accs[tg][kR] = lsum;
    __syncthreads();
    if (tid < kR + 1) {
      float s = 0.f;
      for (int g = 0; g < kThreads / 4; ++g) s += accs[g][tid];
      if (tid < kR) outp[2 + tid] = s;
      else outp[1] = s;
    }
    if (tid == 0) outp[0] = m;
    __syncthreads();  // the stage, the scores and the sums are free again
    ++L;
  }

  if (failed && tid == 0) {
    // a wait gave up (recorded): let every issued copy land before the CTA exits
    for (int k = L; k < issued; ++k) {
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(&full[k % kStages], uint32_t(k / kStages) & 1u) && global_ns() - t0 < kDegradedMbarNs) {
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_latent_kv_rope(const KvRopeParams& r, int sm_count, cudaStream_t s) {
  const LatentKvParams& p = r.p;
  CUtensorMap mk;
  const uint64_t rows = uint64_t(p.batch) * p.heads * p.max_ctx;
  if (!tc::make_map_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.CK, rows, kR, kR * 2, kTile, kR,
                       CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem(latent_kv_rope_kernel, kDynSmem);
  if (e != cudaSuccess) return e;
  const int n_items = p.batch * p.heads * p.n_splits;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c = {};
  c.gridDim = dim3(std::min(n_items, 2 * sm_count));
  c.blockDim = dim3(kThreads);
  c.dynamicSmemBytes = kDynSmem;
  c.stream = s;
  c.attrs = attr;
  c.numAttrs = 1;
  e = cudaLaunchKernelEx(&c, latent_kv_rope_kernel, mk, r);
  if (e != cudaSuccess) return e;
  return launch_latent_kv_combine(p, s);
}

int latent_kv_rope_split() { return kSplit; }

}  // namespace lr
