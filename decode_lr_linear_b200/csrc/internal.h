// Internal launch interface between the C ABI (api.cu) and the kernel files.
#pragma once

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
};

struct ChainParams {
  ChainStep step[kMaxChain];
  int n_steps;
  int nb;             // batch rows in this launch (<= kMaxDecodeChunk)
  const void* x;      // chain input [nb, d_in of step 0], offset to the chunk
  float* acc;         // 3 accumulator sets of acc_set floats (zero on entry and exit)
  int acc_set;        // floats per set
  unsigned int* bar;  // 2 barrier counters (zero on entry and exit)
  int scale_f16;
  int* err;
  unsigned long long wait_ns;  // bound of the grid-barrier waits
};

static_assert(sizeof(ChainParams) < 32000, "chain parameters must fit the kernel parameter space");
size_t chain_workspace_bytes(const ChainParams& p);
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
  float* z;           // [T, rank] fp32 workspace
  int8_t* zq;         // [T, rank_pad] int8 workspace
  float* sz;          // [T]
  unsigned int* amax; // [T] row max |z| as fp32 bits (zero between calls)
  int rank_pad;
  int* err;           // device error word
};

size_t w8a8_workspace_bytes(int T, int rank);
cudaError_t launch_gemm_s8s32(const int8_t* A, const int8_t* B, int b_kn, int M, int N, int K, int32_t* C,
                              int* err, cudaStream_t s);
cudaError_t launch_w8a8(const W8A8Params& p, int sm_count, cudaStream_t s);

}  // namespace lr
