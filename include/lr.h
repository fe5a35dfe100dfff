/*
 * lr.h -- C ABI of the B200 (sm_100a) low-rank decode library.
 *
 * The library executes truncated-SVD-factorised layers at decode time without
 * ever forming the full weight: a weight W (d_in x d_out, y = x W) is replaced
 * by factors A (d_in x r) and B (r x d_out) and the layer computes
 * y = (x A) B.  Three families of calls are provided:
 *   - lr_linear / lr_linear_grouped: factorised linears (Q/K/V/O projections;
 *     the grouped form shares one input between several projections),
 *   - lr_swiglu_ffn: the hybrid SwiGLU FFN whose gate/up channels are split
 *     into SVD-compressed channels (sharing one latent) and dense channels,
 *     int8 round-to-nearest weights with per-output-channel scales,
 *   - lr_latent_kv_decode: single-query flash-decoding attention over
 *     per-head rank-r latent K/V caches,
 * plus per-token int8 quantisation for the W8A8 prefill path.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers unless a parameter says "host".
 *     The caller owns every buffer, including the workspace; the library never
 *     allocates, frees or synchronises (except lr_check_device_error, whose job
 *     is to synchronise).  Descriptors are read during the call and not kept.
 *   - Tensors are dense and row-major; every device pointer must be 16-byte
 *     aligned (LR_ERR_MISALIGNED otherwise).
 *   - Every call is asynchronous on the given stream (NULL = legacy default).
 *   - Arguments are validated before any launch; nothing is launched when a
 *     call returns an error.  A failed kernel launch returns LR_ERR_CUDA.
 *   - There is no host fallback: every step runs in this library's kernels.
 *   - Workspaces: a call that takes one needs at least the bytes reported by
 *     its *_workspace_size function.  A workspace must be zero-filled once
 *     (lr_workspace_init) before its first use; every call leaves it zeroed
 *     again on completion.  Two calls that may run concurrently must not share
 *     a workspace.
 *
 * Factor storage ("latent-major"): both factors hold one contiguous row per
 * latent component j,
 *     A_store [rank, d_in]   row j = column j of A,
 *     B_store [rank, d_out]  row j = row j of B,
 * so y = sum_j (x . A_store[j]) B_store[j].  The leading rows are the leading
 * singular components, so a shorter active rank uses a prefix of both.
 */
#ifndef LR_DECODE_H
#define LR_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LR_API __attribute__((visibility("default")))
#else
#define LR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* lr_stream_t;

typedef enum {
  LR_OK = 0,
  LR_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, inconsistent shape */
  LR_ERR_UNSUPPORTED = 2,    /* valid but not implemented combination (dtype, shape) */
  LR_ERR_MISALIGNED = 3,     /* a device pointer is not 16-byte aligned */
  LR_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
  LR_ERR_CUDA = 5,           /* a CUDA runtime call or kernel launch failed */
  LR_ERR_DEVICE_TIMEOUT = 6  /* a kernel gave up a bounded wait (see lr_check_device_error) */
} lr_status_t;

typedef enum { LR_F32 = 0, LR_BF16 = 1, LR_F16 = 2, LR_I8 = 3, LR_I32 = 4 } lr_dtype_t;

/* ------------------------------------------------------------------------ */
/* Factorised linear                                                        */
/* ------------------------------------------------------------------------ */

/*
 * One truncated-SVD factor pair.  The factor pair replaces the weight
 * (SAES-SVD technical summary, CEALC: the local term || A_l B_l X_l - W_l X_l ||;
 * WSVD "Fine-Grained Per-Head SVD": W_Kh = A_Kh B_Kh); per-projection ranks are
 * free (LASER "Loss-Aware Cross-Layer Rank Allocation", FLRC "Fisher-based
 * layer-wise rank allocation": non-uniform ranks across layers and projections).
 *
 *   A            [rank, d_in]  latent-major first factor (see file header)
 *   B            [rank, d_out] latent-major second factor
 *   rank         stored rank (rows of A and B), >= 1
 *   active_rank  0 (or rank): use every component; 1..rank-1: use only the
 *                first active_rank components (FLRC "progressive low-rank
 *                decoding", r(t) <= r); bytes read scale with it
 *   w_dtype      LR_F32, LR_BF16 or LR_I8
 *   scale_A      LR_I8 only: [rank] scale of row j of A (per latent channel)
 *   scale_B      LR_I8 only: [d_out] scale of column k of B (per output channel)
 *   scale_dtype  LR_I8 only: LR_F16 or LR_F32
 * An int8 factor dequantises as A[i][j] = A_store[j][i] * scale_A[j] and
 * B[j][k] = B_store[j][k] * scale_B[k] (LASER "Hybrid SVD-Quantization for
 * FFNs": RTN quantisation of the factors).
 */
typedef struct lr_factor_desc {
  const void* A;
  const void* B;
  int d_in;
  int d_out;
  int rank;
  int active_rank;
  lr_dtype_t w_dtype;
  lr_dtype_t scale_dtype;
  const void* scale_A;
  const void* scale_B;
} lr_factor_desc_t;

/*
 * y = (x A) B for `batch` tokens (rows of x).
 *
 * Weight-only paths (x_scale == NULL):
 *   w_dtype LR_F32:  x f32 [batch, d_in]  -> y f32 [batch, d_out]
 *   w_dtype LR_BF16: x bf16 [batch, d_in] -> y bf16 [batch, d_out]
 *   w_dtype LR_I8:   x bf16 [batch, d_in] -> y bf16 [batch, d_out]
 *   accumulation in fp32; the r-dim latent z = x A stays on chip in fp32.
 *   Below batch 4 (and always for f32 weights) the CUDA cores stream the
 *   factors; from batch 4 (lr_set_tensor_core_min_batch) bf16 and int8
 *   factors run on the tensor cores (tcgen05, weights as the M operand,
 *   tokens as N), streaming every factor once per pass of up to 32 tokens;
 *   there the latent goes through an fp32 accumulator in the workspace and
 *   enters the second product as bf16 high and low parts (bf16 factors,
 *   fp32 accuracy) or as int8 high and low codes with per-token scales
 *   taken over each tensor-core unit's slice of the reduction (int8 factors,
 *   error within the slice's max|z| / 64516 per element).
 * W8A8 path (x_scale != NULL; w_dtype LR_I8, scale_dtype LR_F32):
 *   x int8 [batch, d_in] with per-token scales x_scale f32 [batch] (from
 *   lr_quantize_per_token), y bf16 [batch, d_out]; int8 x int8 -> int32 tensor
 *   core products; the latent is requantised per token in between:
 *     acc1 = x_q A_q (int32);  z = fp32(fp32(acc1 * x_scale[t]) * scale_A[j])
 *     s_z  = max_j |z| / 127;  z_q = clamp(rint(z / s_z), -127, 127)
 *     acc2 = z_q B_q (int32);  y = bf16(fp32(fp32(acc2 * s_z[t]) * scale_B[k]))
 *   (LASER results, W8A8 setting; WSVD "Quantization-Aware Training",
 *   weights and activations quantised, e.g. W8A8).
 *   Workspace (lr_linear_workspace_size with w8a8 = 1; rp = r rounded up
 *   to 128, bp = batch rounded up to 128, each part rounded up to 256
 *   bytes): the int32 sums of the first product [batch, rp] (batch * rp * 4
 *   bytes; zero on entry and left zero: the first product adds its K-split
 *   pieces into it), then the requantised latent int8 [bp, rp] and its
 *   scales f32 [bp], which each call overwrites and leaves behind.
 * Weight-only limits: d_in and d_out multiples of 8 (of 16 for int8 weights)
 * and at most 32 KiB per factor row (d <= 16384 for bf16, 8192 for f32).
 * ws: workspace of at least lr_linear_workspace_size(...) bytes: 256 +
 * 8-rounded(min(batch, 8) * d_out) * 4, and for bf16 or int8 factors on the
 * tensor-core path at least 256 + (2 r8 + 2 d_out) * c * 4 with c = 8-rounded
 * min(batch, 32) and r8 the 8-rounded active rank.  Zero on entry
 * (lr_workspace_init); every call leaves it zero.
 * Errors: LR_ERR_INVALID_ARG (null pointers, batch < 1, bad shape or rank),
 * LR_ERR_UNSUPPORTED (dtype combination), LR_ERR_MISALIGNED,
 * LR_ERR_WORKSPACE, LR_ERR_CUDA.
 */
LR_API lr_status_t lr_linear(const lr_factor_desc_t* desc, const void* x, const float* x_scale, int batch,
                      void* y, void* ws, size_t ws_bytes, lr_stream_t stream);

LR_API lr_status_t lr_linear_workspace_size(const lr_factor_desc_t* desc, int batch, int w8a8,
                                     size_t* bytes);

/*
 * Several factorised linears that share one input x (e.g. Q, K and V), in one
 * launch: y_p = (x A_p) B_p for p < n (1 <= n <= LR_MAX_GROUP).  All
 * descriptors must have the same d_in, w_dtype and scale_dtype; ranks and
 * d_out may differ.  `descs` is a host array of n descriptors and `ys` a host
 * array of n device output pointers.  Weight-only paths only, any batch >= 1.
 * LASER "System Implementation" fuses the input projection with the latent
 * activation; sharing x across Q/K/V reads it once.
 */
#define LR_MAX_GROUP 4
LR_API lr_status_t lr_linear_grouped(const lr_factor_desc_t* descs, int n, const void* x, int batch,
                              void* const* ys, void* ws, size_t ws_bytes, lr_stream_t stream);

LR_API lr_status_t lr_linear_grouped_workspace_size(const lr_factor_desc_t* descs, int n, int batch,
                                             size_t* bytes);

/*
 * A chain of grouped factorised linears in one launch: the projections of a
 * decode stack (for example Q, K, V of a layer, then O, then the next layer)
 * where a step's input is the chain input or an output of an earlier step.
 * Step s computes y[s][p] = (x_s A[s][p]) B[s][p] for p < n, with
 *   x_s = x                      when input_step < 0,
 *   x_s = y[input_step][input_proj] otherwise (input_step < s).
 * An input taken from an earlier step is read at fp32 (its accumulator times
 * the int8 output scale, before the output rounding to bf16).  Every step's
 * outputs are written.  A step waits only for the step it reads, so steps
 * whose inputs are ready (for example Q and K next to V, which O reads)
 * overlap the hand-off of a dependent one.  All
 * descriptors of a step share d_in, which must equal d_out of the projection
 * its input comes from; all steps share w_dtype (weight-only paths) and
 * scale_dtype; any batch >= 1 (one launch per 8 rows or fewer, depending on
 * the widest row); at most LR_MAX_CHAIN steps.
 * bf16 and int8 factors from batch 4 run on the tensor cores instead (as
 * lr_linear: two launches per step and pass of up to 32 tokens, plus one at
 * the end; there the
 * step right before is read at fp32 from its accumulator and an older step
 * from its stored output).
 * On the CUDA-core path, one persistent CTA per SM (all resident: checked before the
 * launch, LR_ERR_UNSUPPORTED otherwise) streams the factors of all steps back
 * to back through shared memory, so the loads of later steps proceed while a
 * step waits for its input; that wait on the CTAs producing the input is
 * bounded in time (lr_set_wait_timeout_us).  LASER "System Implementation" fuses the stages
 * of a layer to cut memory movement and kernel-launch overhead; this is that
 * fusion across consecutive factorised projections.
 */
#define LR_MAX_CHAIN 128
typedef struct lr_chain_step {
  int n;
  int input_step;
  int input_proj;
  lr_factor_desc_t proj[LR_MAX_GROUP];
  void* y[LR_MAX_GROUP];
} lr_chain_step_t;

LR_API lr_status_t lr_linear_chain(const lr_chain_step_t* steps, int n_steps, const void* x, int batch, void* ws,
                                   size_t ws_bytes, lr_stream_t stream);

LR_API lr_status_t lr_linear_chain_workspace_size(const lr_chain_step_t* steps, int n_steps, int batch,
                                                  size_t* bytes);

/*
 * Rank vectors: one rank per projection, in chain order (step 0's projections,
 * then step 1's, ...).  `ranks` is a host array of n entries, read during the
 * call and not kept.
 */
typedef struct lr_rank_vec {
  int n;
  const int* ranks;
} lr_rank_vec_t;

/*
 * FLRC rank allocation (FLRC "Fisher-based layer-wise rank allocation":
 * r_{l,p} = round(alpha_{l,p} / S * R_budget), S the total importance; FLRC
 * "progressive low-rank decoding": the same rule per token t with a
 * non-increasing budget R_budget(t)).  Host-only, no device work:
 *   alpha      host array of n importances (> 0, finite)
 *   r_budget   total rank budget (>= 0)
 *   cap        the stored ranks (cap->n == n); each result is clamped to
 *              [1, cap->ranks[p]] (a rank of 0 would drop the projection)
 *   ranks_out  host array of n results
 * S is summed in index order, alpha_p / S * r_budget is evaluated in double
 * and rounded to nearest, ties to even.  Errors: LR_ERR_INVALID_ARG.
 */
LR_API lr_status_t lr_rank_allocate(const double* alpha, int n, double r_budget, const lr_rank_vec_t* cap,
                                    int* ranks_out);

/*
 * lr_linear_chain with the active rank of every projection taken from a rank
 * vector (active->n = total projections of the chain, entry p in [0, rank];
 * 0 = every stored component), e.g. the per-token ranks of FLRC progressive
 * decoding from lr_rank_allocate.  The factors are SVD-ordered, so a lower
 * active rank streams a prefix of each factor and the bytes read fall with it.
 * Everything else as lr_linear_chain (the descriptors' own active_rank fields
 * are ignored); the workspace of lr_linear_chain_workspace_size suffices.
 */
LR_API lr_status_t lr_linear_chain_ranked(const lr_chain_step_t* steps, int n_steps, const lr_rank_vec_t* active,
                                          const void* x, int batch, void* ws, size_t ws_bytes, lr_stream_t stream);

/*
 * lr_linear without a caller-provided workspace (the pages have no
 * counterpart to this call; it exists for integration).
 *
 * Some callers cannot allocate device memory at all: a plugin running inside
 * a host framework that owns every device allocation, or a serving loop that
 * has to stay allocation-free after start-up because cudaMalloc can
 * synchronise the device and stall other work.  This call does what lr_linear
 * does on its weight-only paths (x_scale must be absent: f32, bf16 and int8
 * weights) but takes its scratch from a fixed array inside the library of
 * LR_NOALLOC_SCRATCH_BYTES bytes per device, which every GPU that loads the
 * library keeps until the process exits.  The caller still passes x and y.
 *
 *   - The scratch a call needs is 256 + 8-rounded(min(batch, 8) * d_out) * 4
 *     bytes (this call stays on the CUDA-core path at every batch); a call that needs
 *     more returns LR_ERR_WORKSPACE and launches nothing.  Shapes lr_linear
 *     refuses are refused the same way (LR_ERR_UNSUPPORTED) before that.
 *   - The first call on a device (in a CUDA context) looks the array up and
 *     zero-fills it on `stream`; make that first call before any stream
 *     capture.  Every call leaves the array zeroed again, except a call whose
 *     kernel gave up a bounded wait: once lr_check_device_error has reported
 *     that, the next call zero-fills the array again before it launches.
 *   - All calls on one device share the array: calls that may overlap on the
 *     GPU (different streams without ordering between them) race and give
 *     wrong results.  Serialise them, or use lr_linear with your own workspace.
 * It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
#define LR_NOALLOC_SCRATCH_BYTES (1u << 20)
LR_API lr_status_t lr_linear_noalloc(const lr_factor_desc_t* desc, const void* x, int batch, void* y,
                                     lr_stream_t stream);

/*
 * Dense linear, the uncompressed baseline of a factorised projection:
 * y = x W for a weight stored output-major as W_store [d_out, d_in] (row k =
 * output channel k, the layout of a framework's linear weight), bf16 or int8
 * with one scale per output channel (y_k = (x . W_store[k]) * scale[k]).  The
 * pages compare their factorised kernels against uncompressed execution
 * (LASER results: decode speed-up over the uncompressed model; SAES-SVD:
 * inference speed-up of the compressed model); this call is that reference
 * on the same hardware.  Streams every weight byte once per 8 batch rows;
 * no workspace.
 *   W      [d_out, d_in] bf16 (scale NULL) or int8 (scale [d_out], LR_F16/LR_F32)
 *   x      bf16 [batch, d_in] -> y bf16 [batch, d_out]
 * Limits: d_in a multiple of 16 with d_in * element size <= 32 KiB.
 */
LR_API lr_status_t lr_dense_linear(const void* W, lr_dtype_t w_dtype, const void* scale, lr_dtype_t scale_dtype,
                                   int d_in, int d_out, const void* x, int batch, void* y, lr_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Hybrid SwiGLU FFN                                                        */
/* ------------------------------------------------------------------------ */

/*
 * LASER "Hybrid SVD-Quantization for FFNs": the first n_lr hidden channels are
 * low-rank through one latent of width `rank` shared by gate and up; the other
 * n_dense = inter - n_lr channels are dense; every matrix is int8 RTN with one
 * scale per output channel; an orthogonal rotation between the factors is
 * folded offline (A' = A R, B' = R^T B), so the kernels never see it.
 *
 *   A      [rank, hidden]        int8, s_A [rank]        latent-major A'
 *   B      [rank, 2*n_lr]        int8, s_B [2*n_lr]      latent-major B'; columns
 *                                                        gate_0, up_0, gate_1, up_1, ...
 *   D      [2*n_dense, hidden]   int8, s_D [2*n_dense]   dense gate/up, output-major,
 *                                                        rows gate_0, up_0, gate_1, ...
 *   W_down [inter, hidden]       int8, s_down [hidden]   input-major down projection,
 *                                                        rows in [S; D] channel order
 *   scale_dtype  LR_F16 or LR_F32 for all scales.
 * Computes, per token (LASER "System Implementation": fused input projection,
 * latent activation, SwiGLU and dequantisation):
 *   z = x A';  [g_S, u_S] = z B';  [g_D, u_D] = x D';
 *   h = [silu(g_S) u_S, silu(g_D) u_D];  y = h W_down;  silu(t) = t / (1 + e^-t).
 */
typedef struct lr_ffn_desc {
  int hidden;
  int inter;
  int n_lr;
  int rank;
  lr_dtype_t scale_dtype;
  const int8_t* A;
  const void* s_A;
  const int8_t* B;
  const void* s_B;
  const int8_t* D;
  const void* s_D;
  const int8_t* W_down;
  const void* s_down;
} lr_ffn_desc_t;

/* x bf16 [batch, hidden] -> y bf16 [batch, hidden], any batch >= 1.
 * Limits: hidden a multiple of 16 and <= 32768; n_lr a multiple of 8 and
 * <= 16384.  Errors as lr_linear. */
LR_API lr_status_t lr_swiglu_ffn(const lr_ffn_desc_t* desc, const void* x, int batch, void* y, void* ws,
                          size_t ws_bytes, lr_stream_t stream);

LR_API lr_status_t lr_swiglu_ffn_workspace_size(const lr_ffn_desc_t* desc, int batch, size_t* bytes);

/* ------------------------------------------------------------------------ */
/* Per-head latent K/V decode attention                                     */
/* ------------------------------------------------------------------------ */

/*
 * WSVD "Fine-Grained Per-Head SVD": the key projection of head h is factored
 * W_Kh = A_Kh B_Kh at rank r and the cache keeps the per-head latent C_K,h
 * (likewise for values); WSVD "Quantization-Aware Training (QAT) en Fused
 * Kernel": K and V are reconstructed inside the flash-decoding pipeline and
 * never written to global memory.
 *
 *   B_K, B_V  [heads, rank, head_dim] bf16: key t of head h is
 *             K_t = C_K[b,h,t,:] B_K[h], value V_t = C_V[b,h,t,:] B_V[h]
 *   scale     softmax scale (1/sqrt(head_dim) for standard attention)
 *   mode      LR_KV_ABSORBED: scores s_t = C_K[t] (B_K q) * scale, latent
 *             values accumulated and reconstructed once per split; exact
 *             only without a rotary embedding (rope_base must be 0);
 *             LR_KV_RECONSTRUCT: keys reconstructed on chip, 128 cached
 *             positions at a time on the tensor cores, and rotated before the
 *             score: with rope_base > 0, K_t is rotated to position t and q to
 *             position seq_lens[b] - 1 (LLaMA convention: theta_i =
 *             rope_base^(-2i/head_dim), dimension i turns with i + head_dim/2
 *             by pos * theta_i; the pages' models are LLaMA-family, the pages do
 *             not write the embedding out); values carry no rotation.  bf16
 *             caches only (lr_latent_kv_decode); split_tokens 0 or 256;
 *             batch * heads * max_ctx < 2^31 - 256.  Scores use the query and
 *             B_K folded into one bf16 operand per tile (error well inside the
 *             1e-2 normwise bar).
 *   split_tokens  tokens per split-K chunk (multiple of 64), 0 = library choice
 *   rope_base     0: no rotary embedding; > 0: its base (e.g. 10000)
 * Supported: rank 32, head_dim 128.
 */
#define LR_KV_ABSORBED 0
#define LR_KV_RECONSTRUCT 1
typedef struct lr_latent_kv_desc {
  int batch;
  int heads;
  int head_dim;
  int rank;
  int max_ctx;
  float scale;
  const void* B_K;
  const void* B_V;
  int mode;
  int split_tokens;
  lr_dtype_t cache_scale_dtype;  /* lr_latent_kv_decode_q8 only: LR_F16 or LR_F32 */
  float rope_base;               /* LR_KV_RECONSTRUCT only; 0 = no rotary embedding */
} lr_latent_kv_desc_t;

/*
 * q bf16 [batch, heads, head_dim]; C_K, C_V bf16 [batch, heads, max_ctx, rank];
 * seq_lens int32 [batch] (device) with 0 <= seq_lens[b] <= max_ctx (values are
 * clamped into that range; a length of 0 yields a zero output row);
 * out bf16 [batch, heads, head_dim].  The single query of each sequence attends
 * to cached positions 0 .. seq_lens[b]-1.
 */
LR_API lr_status_t lr_latent_kv_decode(const lr_latent_kv_desc_t* desc, const void* q, const void* C_K,
                                const void* C_V, const int* seq_lens, void* out, void* ws,
                                size_t ws_bytes, lr_stream_t stream);

LR_API lr_status_t lr_latent_kv_workspace_size(const lr_latent_kv_desc_t* desc, size_t* bytes);

/*
 * The same decode over int8 latent caches (LASER results: under W8A8 the KV
 * cache is kept in 8 bits), half the cache bytes of bf16:
 *   C_K, C_V  int8 [batch, heads, max_ctx, rank] codes
 *   s_K, s_V  [batch, heads, max_ctx] one scale per cached position
 *             (desc->cache_scale_dtype: LR_F16 or LR_F32)
 * C[t, j] = code[t, j] * s[t]; the key scale multiplies the token's score,
 * the value scale its softmax weight.  Everything else as lr_latent_kv_decode
 * (same workspace size).
 */
LR_API lr_status_t lr_latent_kv_decode_q8(const lr_latent_kv_desc_t* desc, const void* q, const int8_t* C_K,
                                          const void* s_K, const int8_t* C_V, const void* s_V, const int* seq_lens,
                                          void* out, void* ws, size_t ws_bytes, lr_stream_t stream);

/*
 * The latent producer of the per-head caches (WSVD "Fine-Grained Per-Head
 * SVD": the cache keeps the latent x A_Kh of each head instead of its key, and
 * x A_Vh instead of its value): one GEMV over all heads' first factors at
 * once, whose outputs are written straight into the caches at each
 * sequence's new position.
 *   A_KV  bf16 [2 * heads * rank, hidden], latent-major: row h * rank + j is
 *         column j of A_Kh, row (heads + h) * rank + j column j of A_Vh
 *   x     bf16 [batch, hidden], the new token of each sequence
 *   pos   int32 [batch] (device): the position written for sequence b
 *         (normally seq_lens[b] before it is incremented); a position outside
 *         [0, max_ctx) writes nothing for that sequence
 *   C_K, C_V  bf16 [batch, heads, max_ctx, rank], updated in place at
 *         [b, :, pos[b], :]; nothing else is written
 *   ws    lr_latent_kv_append_workspace_size bytes, zero on entry and left
 *         zero: the product then runs on the tensor cores (tcgen05, the stacked
 *         factors as the M operand, the tokens as N, split over the reduction
 *         into an fp32 accumulator) and a scatter writes the bf16 latents; NULL
 *         (or heads * rank not a multiple of 4) keeps the CUDA-core GEMV, which
 *         writes the caches from its epilogue and needs no workspace
 * Only desc->batch, heads, rank and max_ctx are read.  Limits: hidden a
 * multiple of 16 with hidden * 2 <= 32 KiB.
 */
LR_API lr_status_t lr_latent_kv_append(const lr_latent_kv_desc_t* desc, const void* A_KV, int hidden, const void* x,
                                       const int* pos, void* C_K, void* C_V, void* ws, size_t ws_bytes,
                                       lr_stream_t stream);

LR_API lr_status_t lr_latent_kv_append_workspace_size(const lr_latent_kv_desc_t* desc, int hidden, size_t* bytes);

/*
 * Standard single-query flash decoding over full K/V caches: the uncompressed
 * baseline of the latent-KV path (WSVD "Resultaten" and LASER results report
 * speed-ups over FlashDecoding).  out[b,h] = softmax((K q) * scale) V over the
 * first seq_lens[b] positions, split over the context and merged with
 * log-sum-exp rescaling.
 *   q    bf16 [batch, heads, head_dim];  K, V bf16 [batch, heads, max_ctx, head_dim]
 *   seq_lens int32 [batch] (device), clamped to [0, max_ctx]; 0 gives a zero row
 *   out  bf16 [batch, heads, head_dim]
 *   split_tokens  positions per split (multiple of 64, at most 256), 0 = library choice
 * Supported: head_dim 128.  ws: lr_flash_decode_workspace_size bytes (fp32
 * partials; no zero-fill needed).
 */
typedef struct lr_flash_desc {
  int batch;
  int heads;
  int head_dim;
  int max_ctx;
  float scale;
  int split_tokens;
} lr_flash_desc_t;

LR_API lr_status_t lr_flash_decode(const lr_flash_desc_t* desc, const void* q, const void* K, const void* V,
                                   const int* seq_lens, void* out, void* ws, size_t ws_bytes, lr_stream_t stream);

LR_API lr_status_t lr_flash_decode_workspace_size(const lr_flash_desc_t* desc, size_t* bytes);

/* ------------------------------------------------------------------------ */
/* W8A8 helpers                                                             */
/* ------------------------------------------------------------------------ */

/*
 * Per-token symmetric int8 quantisation (LASER results, W8A8 setting):
 * s[t] = fp32(max_i |x[t,i]| / 127) (1 when the row is all zero),
 * x_q[t,i] = clamp(rint(x[t,i] / s[t]), -127, 127), division in IEEE fp32,
 * rint ties to even.  x bf16 [rows, cols] -> x_q int8 [rows, cols], s f32 [rows].
 */
LR_API lr_status_t lr_quantize_per_token(const void* x, int rows, int cols, int8_t* x_q, float* s,
                                  lr_stream_t stream);

/*
 * The tensor-core product behind the W8A8 path, exposed on its own so that
 * its integer results can be checked exactly: C = A B with int8 operands and
 * int32 accumulation (tcgen05 kind::i8), nothing else.
 *   A      [M, K] int8, row-major
 *   B      b_layout 0: [N, K] int8 row-major (the layout of the first factor,
 *          latent-major A_q [r, d_in]); b_layout 1: [K, N] int8 row-major
 *          (the layout of the second factor B_q [r, d_out])
 *   C      [M, N] int32, row-major
 * Limits: K and N multiples of 16; M, N, K >= 1.  No workspace.
 * |C| must stay below 2^31 (K * 127^2 < 2^31 holds for K < 133144).
 */
LR_API lr_status_t lr_gemm_s8s32(const int8_t* A, const int8_t* B, int b_layout, int M, int N, int K, int32_t* C,
                                 lr_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Utilities                                                                */
/* ------------------------------------------------------------------------ */

/* Zero-fill a workspace (cudaMemsetAsync on `stream`). */
LR_API lr_status_t lr_workspace_init(void* ws, size_t ws_bytes, lr_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the library's device error word on
 * the current device.  *err = 0 when no kernel gave up a bounded wait since the
 * last check; otherwise the first code recorded:
 *   1  a wait for the kernel's own asynchronous copies (an mbarrier) gave up
 *      after 2 s: the memory system did not deliver; treat the CUDA context as
 *      unusable;
 *   2  a tensor-memory allocation could not be obtained;
 *   3  a wait for the other CTAs of a persistent grid gave up (see
 *      lr_set_wait_timeout_us): the outputs of that call are wrong and its
 *      workspace may hold partial sums; zero it with lr_workspace_init before
 *      reusing it (the lr_linear_noalloc scratch is re-zeroed by the library).
 * Returns LR_ERR_DEVICE_TIMEOUT when *err != 0, LR_ERR_CUDA if synchronisation
 * failed.
 */
LR_API lr_status_t lr_check_device_error(lr_stream_t stream, int* err);

/*
 * Bound of every wait of a persistent kernel on its other CTAs (the grid-wide
 * barriers of lr_linear_chain and lr_swiglu_ffn), in microseconds, for
 * launches issued after this call; 0 restores the default of one second.  The CTAs of one launch
 * are all resident (checked before every launch), so these waits end within
 * microseconds unless other work occupies the device; a wait that gives up
 * records code 3 in the device error word and the kernel carries on without
 * hanging.  Process-wide.
 */
LR_API lr_status_t lr_set_wait_timeout_us(unsigned int us);

/*
 * Smallest batch at which lr_linear, lr_linear_grouped, lr_linear_chain (bf16
 * or int8 factors, weight-only) and lr_swiglu_ffn switch from the CUDA-core
 * decode kernels to the tensor-core path; 0 restores the defaults, measured on
 * B200: 4 for the linears (the CUDA-core kernels stream the weights once per
 * 2 to 8 tokens, the tensor cores once per 32) and 1 for the FFN (its
 * CUDA-core kernels are bound by int8-to-float conversion).
 * Process-wide, for calls issued after this one; the workspace sizes reported
 * afterwards follow the setting.  A tuning knob: both paths compute the same
 * products (see lr_linear and lr_swiglu_ffn for their precision).
 */
LR_API lr_status_t lr_set_tensor_core_min_batch(int linear, int ffn);

/* Static string for a status code. */
LR_API const char* lr_status_string(lr_status_t status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
LR_API int lr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LR_DECODE_H */
