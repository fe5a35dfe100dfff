// Internal launch interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/lr.h"

namespace lr {

// Device address of the library's error word on the current device.
int* device_error_word();

// Bound of waits on the other CTAs of a persistent grid (lr_set_wait_timeout_us), in nanoseconds.
unsigned long long grid_wait_ns();

// The CTAs of a persistent grid wait for one another, so all of them must be
// resident at once: cudaSuccess when `grid` CTAs of `threads` threads and
// `smem` bytes of dynamic shared memory fit the device together, else
// cudaErrorCooperativeLaunchTooLarge (cached per kernel and size).
cudaError_t check_resident(const void* fn, int threads, size_t smem, int grid, int sm_count);

constexpr int kMaxGroup = LR_MAX_GROUP;

// Workspace element shared by the split-reduction kernels: one arrival counter
// padded to 256 bytes, followed by fp32 accumulators.
constexpr size_t kTicketBytes = 256;

// Batch rows handled by one launch of the CUDA-core decode kernels.
constexpr int kMaxDecodeChunk = 8;

// ---- factorised-linear chains (lr_linear, lr_linear_grouped, lr_linear_chain) ----
constexpr int kMaxChain = LR_MAX_CHAIN;

struct ChainProj {
  const void* A;      // [rank, d_in]
  const void* B;      // [rank, d_out]
  const void* sA;     // int8: [rank]
  const void* sB;     // int8: [d_out]
  void* y;            // [batch, d_out], offset to the batch chunk
  int d_out;
  int rows;           // active latent rows
};

struct ChainStep {
  ChainProj p[kMaxGroup];
  int n;
  int d_in;
  int total_rows;
  int input_step;     // -1: chain input
  int input_proj;
  int acc_off;        // first float of this step's accumulators in ChainParams::acc
};

struct ChainParams {
  ChainStep step[kMaxChain];
  int n_steps;
  int nb;             // batch rows in this launch (<= kMaxDecodeChunk)
  const void* x;      // chain input [nb, d_in of step 0], offset to the chunk
  float* acc;         // every step's fp32 output accumulators (zero on entry and exit)
  unsigned int* bar;  // n_steps completion counters + one exit counter (zero on entry and exit)
  int scale_f16;
  int* err;
  unsigned long long wait_ns;  // bound of the waits on other CTAs
};

static_assert(sizeof(ChainParams) < 32000, "chain parameters must fit the kernel parameter space");
// Bytes of the chain's counters (the accumulators follow them in the workspace).
inline size_t chain_counter_bytes(int n_steps) { return (size_t(n_steps + 1) * 4 + 255) / 256 * 256; }
cudaError_t launch_chain(const ChainParams& p, lr_dtype_t w_dtype, int sm_count, cudaStream_t s);

struct FfnParams {
  int hidden, inter, n_lr, n_dense, rank;
  int nb;
  int scale_f16;
  const int8_t* A; const void* sA;
  const int8_t* B; const void* sB;
  const int8_t* D; const void* sD;
  const int8_t* Wd; const void* sd;
  const void* x;      // bf16 [nb, hidden]
  void* y;            // bf16 [nb, hidden]
  float* gu_acc;      // [nb, 2*n_lr]  (zero on entry and exit)
  float* h_dense;     // [nb, n_dense]
  float* y_acc;       // [nb, hidden]  (zero on entry and exit)
  unsigned int* ticket;
  unsigned long long wait_ns;  // bound of the grid-barrier wait
  int* err;                    // device error word
  // dense mode only: when cache_k is set, output row j of token b is not written
  // to y but to the latent caches [batch, heads, ctx, rank] at position cache_pos[b]
  // (rows [0, heads*rank) -> cache_k, the next heads*rank rows -> cache_v), bf16
  void* cache_k;
  void* cache_v;
  const int* cache_pos;
  int cache_heads, cache_rank, cache_ctx;
};

cudaError_t launch_ffn(const FfnParams& p, int sm_count, cudaStream_t s);
// Dense GEMV y = x W^T for output-major W [n_dense rows, hidden] in p.D (bf16 or
// int8 with per-row scales p.sD, or none); p.x, p.y, p.nb as for the FFN.
cudaError_t launch_dense(const FfnParams& p, lr_dtype_t w_dtype, int sm_count, cudaStream_t s);

struct LatentKvParams {
  int batch, heads, head_dim, rank, max_ctx;
  int split_tokens, n_splits;
  float scale;
  const void* q; const void* CK; const void* CV;
  const void* BK; const void* BV;
  const int* seq_lens;
  void* out;
  float* partial;     // [batch, heads, n_splits, rank + 2]
  float* qt;          // [batch, heads, rank]: B_K q * scale * log2(e)
  int mode;
  int cache_q8;       // 1: int8 caches with per-position scales sK, sV
  int cache_scale_f16;
  const void* sK; const void* sV;   // [batch, heads, max_ctx]
  int* err;           // device error word
};

cudaError_t launch_latent_kv(const LatentKvParams& p, cudaStream_t s);
// The merge of the splits and o = a B_V (the last launch of launch_latent_kv).
cudaError_t launch_latent_kv_combine(const LatentKvParams& p, cudaStream_t s);

// Keys reconstructed on chip, with an optional rotary embedding: p.split_tokens
// must be latent_kv_rope_split(); theta = 0 everywhere means no rotation.
struct KvRopeParams {
  LatentKvParams p;
  float theta_f[64];   // rotary frequencies theta_i = base^(-2i/head_dim)
  double theta_d[64];
};
int latent_kv_rope_split();
cudaError_t launch_latent_kv_rope(const KvRopeParams& r, int sm_count, cudaStream_t s);

// ---- batched decode on the tensor cores (tc_gemv.cu) ----
// One product out[m][n] += sum_k W[m][k] act[n][k] over up to four weight
// matrices ("segments"), each split into units of 128 rows x kc of the reduction.
struct TcSeg {
  int M, K;           // weight rows (outputs) and reduction length
  int a_mn_major;     // 0: W stored [M, K]; 1: W stored [K, M] (its tensor map in TcMaps)
  int m_tiles, k_splits, kc, unit0;
  // The activations, token-major [nb, K] with row stride act_ld (a multiple of 8):
  // act_kind 0 bf16, 1 fp32; act_kind 2 the SwiGLU of the hybrid FFN, h[n][c] =
  // silu(g) u with the interleaved gate/up pair of channel c from the fp32
  // accumulators act [nb, 2 n_lr] (c < n_lr, row stride act_ld) or act2
  // [nb, 2 (K - n_lr)] (the dense channels, row stride act2_ld).
  const void* act;
  int act_kind, act_ld;
  const float* act2;
  int act2_ld, n_lr;
  float* out;         // token-major fp32 [nb, out_ld], out[n][m] += product
  int out_ld;
  const void* row_scale;  // int8 weights: one scale per weight row (output channel), or null
  int row_scale_f16;
};
struct TcFinalTarget {
  const float* acc;   // token-major fp32 [nb, M]
  void* y;            // bf16 [nb, M]
  int M;              // a multiple of 8
};
struct TcFinalizeParams {
  TcFinalTarget t[4];
  int nt;
  int nb;
  int zero_targets;   // clear each accumulator element after reading it
  float* zero[3];
  size_t zero_floats[3];  // multiples of 4
  int nz;
};
// i8: int8 weights (kind::i8, activations as high and low int8 codes; hilo must be set)
struct TcGemvParams {
  TcSeg seg[4];
  int nseg;
  int N;              // MMA N: token rows of the operand (x2 with hilo)
  int nb;             // tokens
  int hilo;           // split each fp32 activation into bf16 high and low parts (rows nb.. of the operand)
  int tmem_cols;
  int stages;         // weight ring depth (set by launch_tc_gemv)
  int* err;
  TcFinalizeParams pre;  // finalize work of the preceding step, spread over the units (after the dependency wait)
};
struct alignas(64) TcMaps {
  CUtensorMap m[4];
};
int tc_gemv_kc(int K, int k_splits, bool i8);
size_t tc_gemv_smem(int kc, int N, bool i8, int stages);
bool tc_gemv_fits(int kc, int N, bool i8);
bool tc_make_weight_map(CUtensorMap* m, const void* W, int rows, int cols, int a_mn_major, bool i8);
cudaError_t launch_tc_gemv(const TcMaps& maps, const TcGemvParams& p, bool i8, cudaStream_t s);
cudaError_t launch_tc_finalize(const TcFinalizeParams& f, int sm_count, cudaStream_t s);
struct TcSwigluParams {
  float* gu;          // token-major [nb, 2 n_lr] gate/up accumulators of the low-rank channels (interleaved)
  float* dd;          // token-major [nb, 2 n_dense] of the dense channels
  float* h;           // token-major [nb, h_ld], h_ld >= n_lr + n_dense
  int h_ld;
  int n_lr, n_dense, nb;
  float* zero;        // token-major rows of zero_row floats zeroed afterwards (or null)
  int zero_row;
};
cudaError_t launch_tc_swiglu(const TcSwigluParams& p, cudaStream_t s);
struct TcScatterParams {
  float* acc;         // token-major fp32 [nb, 2 heads rank], cleared
  void* cache_k;      // bf16 [nb, heads, ctx, rank], offset to the pass's first sequence
  void* cache_v;
  const int* pos;     // [nb]
  int nb, heads, rank, ctx;
};
cudaError_t launch_tc_cache_scatter(const TcScatterParams& p, cudaStream_t s);

// Full-K/V flash decoding (the uncompressed baseline).
struct FlashParams {
  int batch, heads, max_ctx;
  int split_tokens, n_splits;
  float scale;
  const void* q; const void* K; const void* V;   // bf16 [batch, heads, (max_ctx,) 128]
  const int* seq_lens;
  void* out;          // bf16 [batch, heads, 128]
  float* partial;     // [batch, heads, n_splits, 130]
  int* err;
};

size_t flash_partial_floats();
cudaError_t launch_flash(const FlashParams& p, cudaStream_t s);

cudaError_t launch_quantize_per_token(const void* x, int rows, int cols, int8_t* xq, float* s,
                                      cudaStream_t st);

struct W8A8Params {
  int T, d_in, d_out, rank;
  const int8_t* xq; const float* sx;
  const int8_t* Aq; const float* sA;
  const int8_t* Bq; const float* sB;
  void* y;            // bf16 [T, d_out]
  int32_t* acc;       // [T, rank_pad] int32 sums of the first product (zero between calls)
  int8_t* zq;         // [T, rank_pad] int8 workspace
  float* sz;          // [T]
  int rank_pad;
  int* err;           // device error word
};

size_t w8a8_workspace_bytes(int T, int rank);
cudaError_t launch_gemm_s8s32(const int8_t* A, const int8_t* B, int b_kn, int M, int N, int K, int32_t* C,
                              int* err, int sm_count, cudaStream_t s);
cudaError_t launch_w8a8(const W8A8Params& p, int sm_count, cudaStream_t s);

}  // namespace lr
