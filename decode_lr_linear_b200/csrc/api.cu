// C ABI of the low-rank decode library: argument validation, workspace sizing
// and dispatch to the sm_100a kernels.  Nothing here computes on the host.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace lr {

// The library's device error word: set by kernels whose bounded waits give up.
__device__ int g_device_error = 0;

// Looked up on every call (cheap): the address belongs to the module loaded in
// the current context, which a device reset replaces.
int* device_error_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
  return reinterpret_cast<int*>(p);
}

namespace {
std::atomic<unsigned long long> g_grid_wait_ns{kGridWaitDefaultNs};
}  // namespace

unsigned long long grid_wait_ns() { return g_grid_wait_ns.load(std::memory_order_relaxed); }

cudaError_t check_resident(const void* fn, int threads, size_t smem, int grid, int sm_count) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void*, size_t>, int>> cache;
  int per_sm = -1;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (auto& e : cache)
      if (e.first.first == fn && e.first.second == smem) per_sm = e.second;
  }
  if (per_sm < 0) {
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    cache.push_back({{fn, smem}, per_sm});
  }
  return per_sm * sm_count >= grid ? cudaSuccess : cudaErrorCooperativeLaunchTooLarge;
}

}  // namespace lr

namespace {

using namespace lr;

constexpr int kMaxDevices = 64;

int sm_count_current() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline lr_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return LR_OK;
  // a persistent grid that cannot be resident at once: a configuration limit
  if (e == cudaErrorCooperativeLaunchTooLarge) return LR_ERR_UNSUPPORTED;
  return LR_ERR_CUDA;
}


// Shape/pointer checks common to every factor descriptor.
lr_status_t check_factor(const lr_factor_desc_t* d) {
  if (!d || !d->A || !d->B) return LR_ERR_INVALID_ARG;
  if (d->d_in <= 0 || d->d_out <= 0 || d->rank <= 0) return LR_ERR_INVALID_ARG;
  if (d->active_rank < 0 || d->active_rank > d->rank) return LR_ERR_INVALID_ARG;
  if (d->w_dtype != LR_F32 && d->w_dtype != LR_BF16 && d->w_dtype != LR_I8) return LR_ERR_UNSUPPORTED;
  if (d->w_dtype == LR_I8) {
    if (!d->scale_A || !d->scale_B) return LR_ERR_INVALID_ARG;
    if (d->scale_dtype != LR_F16 && d->scale_dtype != LR_F32) return LR_ERR_UNSUPPORTED;
    if (!al16(d->scale_A) || !al16(d->scale_B)) return LR_ERR_MISALIGNED;
  }
  if ((d->d_in % 8) != 0 || (d->d_out % 8) != 0) return LR_ERR_UNSUPPORTED;
  if (!al16(d->A) || !al16(d->B)) return LR_ERR_MISALIGNED;
  return LR_OK;
}

inline int active(const lr_factor_desc_t* d) { return d->active_rank ? d->active_rank : d->rank; }

// Limits of the streaming decode kernels: rows are moved by bulk copies, so a
// row must be 16-byte aligned and fit one 32 KiB shared-memory stage.
lr_status_t check_rank1_limits(const lr_factor_desc_t* d) {
  const size_t es = d->w_dtype == LR_F32 ? 4 : (d->w_dtype == LR_BF16 ? 2 : 1);
  if ((size_t(d->d_in) * es) % 16 != 0 || (size_t(d->d_out) * es) % 16 != 0) return LR_ERR_UNSUPPORTED;
  if (size_t(d->d_in) * es > 32768 || size_t(d->d_out) * es > 32768) return LR_ERR_UNSUPPORTED;
  return LR_OK;
}

// One step of a chain as the host sees it.
struct HostStep {
  const lr_factor_desc_t* d;
  int n;
  int input_step;
  int input_proj;
  void* const* y;
};

// Floats of step s's accumulators for one batch chunk (8-float aligned).
size_t chain_step_floats(const HostStep& h, int batch) {
  const int chunk = std::min(batch, kMaxDecodeChunk);
  size_t t = 0;
  for (int p = 0; p < h.n; ++p) t += size_t(chunk) * h.d[p].d_out;
  return round_up(t, 8);
}

// ---- batched decode on the tensor cores (bf16 or int8 factors) ----
// Tokens per pass of the weights, and the accumulator columns of one pass.
constexpr int kTcMaxPass = 32;
// Smallest batch that takes the tensor-core path (lr_set_tensor_core_min_batch).
// Measured on B200 (7B shapes): from batch 4 the tensor-core path streams the
// factorised linears faster (stack 0.43 against 0.32 of HBM); the int8 FFN is
// faster there at every batch (batch 1: 41 against 47.5 us; batch 8: 46 against
// 217 us), its CUDA-core kernels being bound by int8-to-float conversion.
constexpr int kTcDefaultMinBatchLinear = 4;
constexpr int kTcDefaultMinBatchFfn = 1;
std::atomic<int> g_tc_min_linear{kTcDefaultMinBatchLinear};
std::atomic<int> g_tc_min_ffn{kTcDefaultMinBatchFfn};
bool use_tc_path(const HostStep* steps, int batch) {
  return batch >= g_tc_min_linear.load(std::memory_order_relaxed) &&
         (steps[0].d[0].w_dtype == LR_BF16 || steps[0].d[0].w_dtype == LR_I8);
}
bool use_tc_ffn(int batch) { return batch >= g_tc_min_ffn.load(std::memory_order_relaxed); }
int tc_cols(int batch) { return int(round_up(size_t(std::min(batch, kTcMaxPass)), 8)); }

// Workspace of the tensor-core path: z accumulator [sum of a step's active ranks, cols]
// and two y accumulator sets [sum of a step's d_out, cols], fp32, zero on entry and exit.
// Row length of projection p's latent accumulator (token-major, 8-float aligned rows).
inline size_t tc_zld(const lr_factor_desc_t& d) { return round_up(size_t(active(&d)), 8); }

void tc_sizes(const HostStep* steps, int n_steps, size_t* zmax, size_t* ymax) {
  *zmax = 0;
  *ymax = 0;
  for (int s = 0; s < n_steps; ++s) {
    size_t z = 0, y = 0;
    for (int p = 0; p < steps[s].n; ++p) {
      z += tc_zld(steps[s].d[p]);
      y += size_t(steps[s].d[p].d_out);
    }
    *zmax = std::max(*zmax, z);
    *ymax = std::max(*ymax, y);
  }
}
size_t tc_ws_bytes(const HostStep* steps, int n_steps, int batch) {
  size_t zm, ym;
  tc_sizes(steps, n_steps, &zm, &ym);
  return kTicketBytes + (2 * zm + 2 * ym) * size_t(tc_cols(batch)) * 4;
}

size_t chain_ws_bytes(const HostStep* steps, int n_steps, int batch, bool allow_tc = true) {
  size_t b = chain_counter_bytes(n_steps);
  for (int s = 0; s < n_steps; ++s) b += chain_step_floats(steps[s], batch) * 4;
  if (allow_tc && use_tc_path(steps, batch)) b = std::max(b, tc_ws_bytes(steps, n_steps, batch));
  return b;
}

size_t rank1_ws_bytes(const lr_factor_desc_t* descs, int n, int batch, bool allow_tc = true) {
  HostStep h{descs, n, -1, 0, nullptr};
  return chain_ws_bytes(&h, 1, batch, allow_tc);
}

lr_status_t check_chain(const HostStep* steps, int n_steps) {
  if (n_steps < 1 || n_steps > LR_MAX_CHAIN) return LR_ERR_INVALID_ARG;
  const lr_factor_desc_t& d0 = steps[0].d[0];
  int x_width = -1;
  for (int s = 0; s < n_steps; ++s) {
    const HostStep& h = steps[s];
    if (h.n < 1 || h.n > LR_MAX_GROUP || !h.d || !h.y) return LR_ERR_INVALID_ARG;
    for (int p = 0; p < h.n; ++p) {
      lr_status_t st = check_factor(&h.d[p]);
      if (st != LR_OK) return st;
      st = check_rank1_limits(&h.d[p]);
      if (st != LR_OK) return st;
      if (h.d[p].d_in != h.d[0].d_in || h.d[p].w_dtype != d0.w_dtype) return LR_ERR_INVALID_ARG;
      if (d0.w_dtype == LR_I8 && h.d[p].scale_dtype != d0.scale_dtype) return LR_ERR_INVALID_ARG;
      if (!h.y[p]) return LR_ERR_INVALID_ARG;
      if (!al16(h.y[p])) return LR_ERR_MISALIGNED;
    }
    if (h.input_step < 0) {
      if (x_width >= 0 && x_width != h.d[0].d_in) return LR_ERR_INVALID_ARG;
      x_width = h.d[0].d_in;
    } else {
      if (h.input_step >= s) return LR_ERR_INVALID_ARG;
      const HostStep& src = steps[h.input_step];
      if (h.input_proj < 0 || h.input_proj >= src.n) return LR_ERR_INVALID_ARG;
      if (src.d[h.input_proj].d_out != h.d[0].d_in) return LR_ERR_INVALID_ARG;
    }
  }
  return LR_OK;
}

// Tensor maps of weight matrices, cached by (address, shape, layout): weights keep
// their addresses across calls, and encoding a map costs host time on every launch.
bool weight_map(CUtensorMap* out, const void* W, int rows, int cols, int mn_major, bool i8) {
  struct Key {
    const void* W;
    int rows, cols, mn, i8;
    bool operator==(const Key& o) const {
      return W == o.W && rows == o.rows && cols == o.cols && mn == o.mn && i8 == o.i8;
    }
  };
  static std::mutex mu;
  static std::vector<std::pair<Key, CUtensorMap>> cache;
  const Key k{W, rows, cols, mn_major, i8 ? 1 : 0};
  std::lock_guard<std::mutex> lock(mu);
  for (auto& e : cache)
    if (e.first == k) {
      *out = e.second;
      return true;
    }
  if (!tc_make_weight_map(out, W, rows, cols, mn_major, i8)) return false;
  if (cache.size() >= 4096) cache.clear();
  cache.push_back({k, *out});
  return true;
}

// One product launch over the segments already filled in (maps, seg[].M/K/act/out):
// split the reduction so that the launch has about two units per SM.
cudaError_t tc_product(TcMaps& maps, TcGemvParams& g, int sms, bool i8, cudaStream_t stream) {
  const int kbe = i8 ? 128 : 64;  // reduction elements per k-block
  int tiles = 0;
  for (int i = 0; i < g.nseg; ++i) {
    g.seg[i].m_tiles = (g.seg[i].M + 127) / 128;
    tiles += g.seg[i].m_tiles;
  }
  int ks = std::max(1, (2 * sms + tiles / 2) / std::max(1, tiles));
  int unit = 0;
  for (int i = 0; i < g.nseg; ++i) {
    TcSeg& sg = g.seg[i];
    int kc = tc_gemv_kc(sg.K, ks, i8);
    kc = std::max(kc, std::min(4 * kbe, int(round_up(size_t(sg.K), kbe))));  // at least 4 k-blocks per unit
    while (!tc_gemv_fits(kc, g.N, i8) && kc > kbe) kc -= kbe;
    sg.kc = kc;
    sg.k_splits = (sg.K + kc - 1) / kc;   // no empty unit
    sg.unit0 = unit;
    unit += sg.m_tiles * sg.k_splits;
  }
  int cols = 32;
  while (cols < g.N + 16) cols *= 2;
  g.tmem_cols = cols;
  return launch_tc_gemv(maps, g, i8, stream);
}

// The chain on the tensor cores, per pass of up to kTcMaxPass tokens and per step s:
//   product 1: z_p += x A_p into latent set s % 2; its units first finalize step
//              s-1 (bf16 outputs from y set (s-1) % 2) and clear y set s % 2 and
//              latent set (s-1) % 2, neither of which it reads
//   product 2: y_p += z_p B_p into y set s % 2 (fp32 z as bf16 high and low
//              parts, or int8 high and low codes for int8 factors)
// and after the last step one finalize launch.  All accumulators are token-major
// fp32; the input is the chain input, the previous step's y set (fp32), or an
// older step's stored bf16 output.
lr_status_t run_chain_tc(const HostStep* steps, int n_steps, const void* x, int batch, void* ws, cudaStream_t stream) {
  size_t zmax, ymax;
  tc_sizes(steps, n_steps, &zmax, &ymax);
  const int cols = tc_cols(batch);
  float* acc0 = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kTicketBytes);
  float* zacc[2] = {acc0, acc0 + zmax * cols};
  float* yacc[2] = {acc0 + 2 * zmax * cols, acc0 + (2 * zmax + ymax) * cols};
  int* err = device_error_word();
  const int sms = sm_count_current();
  const bool i8 = steps[0].d[0].w_dtype == LR_I8;
  const int scale_f16 = steps[0].d[0].scale_dtype == LR_F16 ? 1 : 0;
  int x_width = 0;
  for (int s = 0; s < n_steps; ++s)
    if (steps[s].input_step < 0) x_width = steps[s].d[0].d_in;
  // finalize of step t of this pass: its bf16 outputs from y set t % 2
  auto set_targets = [&](TcFinalizeParams& f, int t, int b0, int nb) {
    const HostStep& h = steps[t];
    f.nt = h.n;
    f.nb = nb;
    size_t yoff = 0;
    for (int p = 0; p < h.n; ++p) {
      f.t[p].acc = yacc[t & 1] + yoff * cols;
      f.t[p].y = reinterpret_cast<char*>(h.y[p]) + size_t(b0) * h.d[p].d_out * 2;
      f.t[p].M = h.d[p].d_out;
      yoff += size_t(h.d[p].d_out);
    }
  };
  for (int b0 = 0; b0 < batch; b0 += kTcMaxPass) {
    const int nb = std::min(kTcMaxPass, batch - b0);
    const int nh = int(round_up(size_t(nb), 8));
    for (int s = 0; s < n_steps; ++s) {
      const HostStep& h = steps[s];
      float* z = zacc[s & 1];
      // ---- the step's input ----
      const void* act;
      int act_kind, act_ld;
      if (h.input_step < 0) {
        act = reinterpret_cast<const char*>(x) + size_t(b0) * x_width * 2;
        act_kind = 0;
        act_ld = x_width;
      } else if (h.input_step == s - 1) {
        size_t off = 0;
        for (int q = 0; q < h.input_proj; ++q) off += size_t(steps[s - 1].d[q].d_out);
        act = yacc[(s - 1) & 1] + off * cols;
        act_kind = 1;
        act_ld = steps[s - 1].d[h.input_proj].d_out;
      } else {
        const HostStep& src = steps[h.input_step];
        act = reinterpret_cast<const char*>(src.y[h.input_proj]) + size_t(b0) * src.d[h.input_proj].d_out * 2;
        act_kind = 0;
        act_ld = src.d[h.input_proj].d_out;
      }
      cudaError_t e;
      // ---- product 1: z_p = x A_p ----
      TcMaps maps;
      TcGemvParams g;
      std::memset(&maps, 0, sizeof(maps));
      std::memset(&g, 0, sizeof(g));
      g.nseg = h.n;
      g.nb = nb;
      g.err = err;
      g.hilo = (i8 || act_kind == 1) ? 1 : 0;
      g.N = g.hilo ? std::max(16, 2 * nh) : int(round_up(size_t(nb), 16));
      if (s > 0) {
        set_targets(g.pre, s - 1, b0, nb);
        g.pre.zero[0] = yacc[s & 1];                 // step s-2's set, finalized by the previous launch
        g.pre.zero_floats[0] = ymax * cols;
        g.pre.zero[1] = zacc[(s - 1) & 1];           // consumed by step s-1's second product
        g.pre.zero_floats[1] = zmax * cols;
        g.pre.nz = 2;
      }
      size_t zoff = 0;
      for (int p = 0; p < h.n; ++p) {
        const lr_factor_desc_t& d = h.d[p];
        if (!weight_map(&maps.m[p], d.A, active(&d), d.d_in, 0, i8)) return LR_ERR_CUDA;
        TcSeg& sg = g.seg[p];
        sg.row_scale = i8 ? d.scale_A : nullptr;
        sg.row_scale_f16 = scale_f16;
        sg.M = active(&d);
        sg.K = d.d_in;
        sg.a_mn_major = 0;
        sg.act = act;
        sg.act_kind = act_kind;
        sg.act_ld = act_ld;
        sg.out = z + zoff * cols;
        sg.out_ld = int(tc_zld(d));
        zoff += tc_zld(d);
      }
      e = tc_product(maps, g, sms, i8, stream);
      if (e != cudaSuccess) return from_cuda(e);
      // ---- product 2: y_p = z_p B_p ----
      std::memset(&maps, 0, sizeof(maps));
      std::memset(&g.pre, 0, sizeof(g.pre));
      g.hilo = 1;
      g.N = std::max(16, 2 * nh);
      zoff = 0;
      size_t yoff = 0;
      for (int p = 0; p < h.n; ++p) {
        const lr_factor_desc_t& d = h.d[p];
        if (!weight_map(&maps.m[p], d.B, active(&d), d.d_out, 1, i8)) return LR_ERR_CUDA;
        TcSeg& sg = g.seg[p];
        sg.row_scale = i8 ? d.scale_B : nullptr;
        sg.row_scale_f16 = scale_f16;
        sg.M = d.d_out;
        sg.K = active(&d);
        sg.a_mn_major = 1;
        sg.act = z + zoff * cols;
        sg.act_kind = 1;
        sg.act_ld = int(tc_zld(d));
        sg.out = yacc[s & 1] + yoff * cols;
        sg.out_ld = d.d_out;
        zoff += tc_zld(d);
        yoff += size_t(d.d_out);
      }
      e = tc_product(maps, g, sms, i8, stream);
      if (e != cudaSuccess) return from_cuda(e);
    }
    // the last step: outputs (clearing its y set), its latent set, the other y set
    const int last = n_steps - 1;
    TcFinalizeParams f;
    std::memset(&f, 0, sizeof(f));
    set_targets(f, last, b0, nb);
    f.zero_targets = 1;
    f.zero[0] = zacc[last & 1];
    f.zero_floats[0] = zmax * cols;
    f.zero[1] = yacc[(last + 1) & 1];
    f.zero_floats[1] = ymax * cols;
    f.nz = 2;
    cudaError_t e = launch_tc_finalize(f, sms, stream);
    if (e != cudaSuccess) return from_cuda(e);
  }
  return LR_OK;
}

lr_status_t run_chain(const HostStep* steps, int n_steps, const void* x, int batch, void* ws, size_t ws_bytes,
                      cudaStream_t stream, bool allow_tc = true) {
  lr_status_t st = check_chain(steps, n_steps);
  if (st != LR_OK) return st;
  if (!x || batch < 1) return LR_ERR_INVALID_ARG;
  if (!al16(x)) return LR_ERR_MISALIGNED;
  if (!ws || ws_bytes < chain_ws_bytes(steps, n_steps, batch, allow_tc)) return LR_ERR_WORKSPACE;
  if (!al16(ws)) return LR_ERR_MISALIGNED;
  if (allow_tc && use_tc_path(steps, batch)) return run_chain_tc(steps, n_steps, x, batch, ws, stream);
  const lr_dtype_t wt = steps[0].d[0].w_dtype;
  const size_t es = (wt == LR_F32) ? 4 : 2;  // activation / output element size
  static ChainParams P;                      // large (kernel parameters); filled under a lock
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  std::memset(&P, 0, sizeof(P));
  P.n_steps = n_steps;
  P.scale_f16 = steps[0].d[0].scale_dtype == LR_F16 ? 1 : 0;
  P.bar = reinterpret_cast<unsigned int*>(ws);
  P.acc = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + chain_counter_bytes(n_steps));
  P.err = device_error_word();
  P.wait_ns = grid_wait_ns();
  int x_width = 0;
  size_t acc_off = 0;
  for (int s = 0; s < n_steps; ++s) {
    ChainStep& c = P.step[s];
    c.acc_off = int(acc_off);
    acc_off += chain_step_floats(steps[s], batch);
    c.n = steps[s].n;
    c.d_in = steps[s].d[0].d_in;
    c.input_step = steps[s].input_step < 0 ? -1 : steps[s].input_step;
    c.input_proj = steps[s].input_proj;
    if (c.input_step < 0) x_width = c.d_in;
    int rows = 0;
    for (int p = 0; p < c.n; ++p) {
      const lr_factor_desc_t& d = steps[s].d[p];
      c.p[p].A = d.A;
      c.p[p].B = d.B;
      c.p[p].sA = wt == LR_I8 ? d.scale_A : nullptr;
      c.p[p].sB = wt == LR_I8 ? d.scale_B : nullptr;
      c.p[p].d_out = d.d_out;
      c.p[p].rows = active(&d);
      rows += c.p[p].rows;
    }
    c.total_rows = rows;
  }
  const int sms = sm_count_current();
  for (int b0 = 0; b0 < batch; b0 += kMaxDecodeChunk) {
    P.nb = std::min(kMaxDecodeChunk, batch - b0);
    P.x = reinterpret_cast<const char*>(x) + size_t(b0) * x_width * es;
    for (int s = 0; s < n_steps; ++s)
      for (int p = 0; p < P.step[s].n; ++p)
        P.step[s].p[p].y = reinterpret_cast<char*>(steps[s].y[p]) + size_t(b0) * steps[s].d[p].d_out * es;
    st = from_cuda(launch_chain(P, wt, sms, stream));
    if (st != LR_OK) return st;
  }
  return LR_OK;
}

lr_status_t run_rank1(const lr_factor_desc_t* descs, int n, const void* x, int batch, void* const* ys, void* ws,
                      size_t ws_bytes, cudaStream_t stream, bool allow_tc = true) {
  HostStep h{descs, n, -1, 0, ys};
  return run_chain(&h, 1, x, batch, ws, ws_bytes, stream, allow_tc);
}

// ---------------------------------------------------------------------------
// Scratch for lr_linear_noalloc: a fixed-size device array that belongs to the
// library, so that callers who cannot allocate device memory still have the
// split-reduction accumulators and arrival counter that lr_linear needs.  Host
// code never uses the symbol itself as a pointer: its device address is looked
// up on every call with the device current.  The array is zero-filled on the
// first call in a CUDA context (the looked-up address is new) and again after
// lr_check_device_error has reported a kernel that gave up a wait (such a
// kernel may leave partial sums behind); the kernels leave it zeroed otherwise.
// ---------------------------------------------------------------------------
__device__ __align__(256) unsigned char g_noalloc_scratch[LR_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};  // address zero-filled last, per device

// Device address of the scratch on the current device, zero-filled on `s`
// first when it is new or was marked dirty.
lr_status_t noalloc_scratch(cudaStream_t s, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LR_ERR_UNSUPPORTED;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] != p) {
    if (cudaMemsetAsync(p, 0, LR_NOALLOC_SCRATCH_BYTES, s) != cudaSuccess) return LR_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = p;
  return LR_OK;
}

void noalloc_mark_dirty() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  g_noalloc_ptr[dev] = nullptr;
}

}  // namespace

extern "C" {

lr_status_t lr_set_tensor_core_min_batch(int linear, int ffn) {
  if (linear < 0 || ffn < 0) return LR_ERR_INVALID_ARG;
  g_tc_min_linear.store(linear ? linear : kTcDefaultMinBatchLinear, std::memory_order_relaxed);
  g_tc_min_ffn.store(ffn ? ffn : kTcDefaultMinBatchFfn, std::memory_order_relaxed);
  return LR_OK;
}

lr_status_t lr_set_wait_timeout_us(unsigned int us) {
  g_grid_wait_ns.store(us ? (unsigned long long)us * 1000ull : kGridWaitDefaultNs, std::memory_order_relaxed);
  return LR_OK;
}

lr_status_t lr_linear_noalloc(const lr_factor_desc_t* desc, const void* x, int batch, void* y,
                              lr_stream_t stream) {
  lr_status_t st = check_factor(desc);
  if (st != LR_OK) return st;
  if (!x || !y || batch < 1) return LR_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y)) return LR_ERR_MISALIGNED;
  st = check_rank1_limits(desc);
  if (st != LR_OK) return st;
  // the CUDA-core path only: its scratch need is what the fixed array is sized for
  if (rank1_ws_bytes(desc, 1, batch, false) > size_t(LR_NOALLOC_SCRATCH_BYTES)) return LR_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  st = noalloc_scratch(s, &ws);
  if (st != LR_OK) return st;
  void* ys[1] = {y};
  return run_rank1(desc, 1, x, batch, ys, ws, LR_NOALLOC_SCRATCH_BYTES, s, false);
}

lr_status_t lr_linear_workspace_size(const lr_factor_desc_t* desc, int batch, int w8a8, size_t* bytes) {
  if (!bytes) return LR_ERR_INVALID_ARG;
  lr_status_t st = check_factor(desc);
  if (st != LR_OK) return st;
  if (batch < 1) return LR_ERR_INVALID_ARG;
  if (w8a8) {
    if (desc->w_dtype != LR_I8) return LR_ERR_UNSUPPORTED;
    *bytes = w8a8_workspace_bytes(batch, active(desc));
  } else {
    *bytes = rank1_ws_bytes(desc, 1, batch);
  }
  return LR_OK;
}

lr_status_t lr_linear(const lr_factor_desc_t* desc, const void* x, const float* x_scale, int batch, void* y,
                      void* ws, size_t ws_bytes, lr_stream_t stream) {
  lr_status_t st = check_factor(desc);
  if (st != LR_OK) return st;
  if (!x || !y || batch < 1) return LR_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y)) return LR_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (x_scale) {
    if (desc->w_dtype != LR_I8 || desc->scale_dtype != LR_F32) return LR_ERR_UNSUPPORTED;
    if (!al16(x_scale)) return LR_ERR_MISALIGNED;
    if ((desc->d_in % 16) != 0 || (desc->d_out % 16) != 0) return LR_ERR_UNSUPPORTED;
    if (!ws) return LR_ERR_WORKSPACE;
    const int r = active(desc);
    if (ws_bytes < w8a8_workspace_bytes(batch, r)) return LR_ERR_WORKSPACE;
    if (!al16(ws)) return LR_ERR_MISALIGNED;
    W8A8Params P;
    std::memset(&P, 0, sizeof(P));
    P.T = batch; P.d_in = desc->d_in; P.d_out = desc->d_out; P.rank = r;
    P.xq = reinterpret_cast<const int8_t*>(x); P.sx = x_scale;
    P.Aq = reinterpret_cast<const int8_t*>(desc->A); P.sA = reinterpret_cast<const float*>(desc->scale_A);
    P.Bq = reinterpret_cast<const int8_t*>(desc->B); P.sB = reinterpret_cast<const float*>(desc->scale_B);
    P.y = y;
    char* w = reinterpret_cast<char*>(ws);
    P.rank_pad = int(round_up(size_t(r), 128));
    P.acc = reinterpret_cast<int32_t*>(w);
    w += round_up(size_t(batch) * P.rank_pad * 4, 256);
    P.zq = reinterpret_cast<int8_t*>(w);
    w += round_up(size_t(round_up(batch, 128)) * P.rank_pad, 256);
    P.sz = reinterpret_cast<float*>(w);
    P.err = device_error_word();
    return from_cuda(launch_w8a8(P, sm_count_current(), s));
  }
  void* ys[1] = {y};
  return run_rank1(desc, 1, x, batch, ys, ws, ws_bytes, s);
}

lr_status_t lr_linear_grouped_workspace_size(const lr_factor_desc_t* descs, int n, int batch, size_t* bytes) {
  if (!bytes || !descs || n < 1 || n > LR_MAX_GROUP || batch < 1) return LR_ERR_INVALID_ARG;
  for (int p = 0; p < n; ++p) {
    lr_status_t st = check_factor(&descs[p]);
    if (st != LR_OK) return st;
  }
  *bytes = rank1_ws_bytes(descs, n, batch);
  return LR_OK;
}

lr_status_t lr_linear_grouped(const lr_factor_desc_t* descs, int n, const void* x, int batch, void* const* ys,
                              void* ws, size_t ws_bytes, lr_stream_t stream) {
  if (!descs || n < 1 || n > LR_MAX_GROUP || !x || !ys || batch < 1) return LR_ERR_INVALID_ARG;
  for (int p = 0; p < n; ++p) {
    lr_status_t st = check_factor(&descs[p]);
    if (st != LR_OK) return st;
    if (!ys[p]) return LR_ERR_INVALID_ARG;
    if (!al16(ys[p])) return LR_ERR_MISALIGNED;
    if (descs[p].d_in != descs[0].d_in || descs[p].w_dtype != descs[0].w_dtype) return LR_ERR_INVALID_ARG;
    if (descs[0].w_dtype == LR_I8 && descs[p].scale_dtype != descs[0].scale_dtype) return LR_ERR_INVALID_ARG;
  }
  if (!al16(x)) return LR_ERR_MISALIGNED;
  return run_rank1(descs, n, x, batch, ys, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

lr_status_t lr_linear_chain_workspace_size(const lr_chain_step_t* steps, int n_steps, int batch, size_t* bytes) {
  if (!bytes || !steps || n_steps < 1 || n_steps > LR_MAX_CHAIN || batch < 1) return LR_ERR_INVALID_ARG;
  HostStep h[LR_MAX_CHAIN];
  for (int s = 0; s < n_steps; ++s) h[s] = HostStep{steps[s].proj, steps[s].n, steps[s].input_step, steps[s].input_proj, steps[s].y};
  lr_status_t st = check_chain(h, n_steps);
  if (st != LR_OK) return st;
  *bytes = chain_ws_bytes(h, n_steps, batch);
  return LR_OK;
}

lr_status_t lr_rank_allocate(const double* alpha, int n, double r_budget, const lr_rank_vec_t* cap,
                             int* ranks_out) {
  if (!alpha || n < 1 || !cap || !cap->ranks || cap->n != n || !ranks_out) return LR_ERR_INVALID_ARG;
  if (!(r_budget >= 0.0) || !std::isfinite(r_budget)) return LR_ERR_INVALID_ARG;
  double S = 0.0;
  for (int p = 0; p < n; ++p) {
    if (!(alpha[p] > 0.0) || !std::isfinite(alpha[p]) || cap->ranks[p] < 1) return LR_ERR_INVALID_ARG;
    S += alpha[p];
  }
  for (int p = 0; p < n; ++p) {
    const double r = std::nearbyint((alpha[p] / S) * r_budget);  // default rounding: to nearest, ties to even
    ranks_out[p] = int(std::min(std::max(r, 1.0), double(cap->ranks[p])));
  }
  return LR_OK;
}

lr_status_t lr_linear_chain_ranked(const lr_chain_step_t* steps, int n_steps, const lr_rank_vec_t* active,
                                   const void* x, int batch, void* ws, size_t ws_bytes, lr_stream_t stream) {
  if (!steps || n_steps < 1 || n_steps > LR_MAX_CHAIN || !active || !active->ranks) return LR_ERR_INVALID_ARG;
  int total = 0;
  for (int s = 0; s < n_steps; ++s) {
    if (steps[s].n < 1 || steps[s].n > LR_MAX_GROUP) return LR_ERR_INVALID_ARG;
    total += steps[s].n;
  }
  if (active->n != total) return LR_ERR_INVALID_ARG;
  static lr_factor_desc_t descs[LR_MAX_CHAIN][LR_MAX_GROUP];  // the steps' descriptors with the vector's ranks
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  HostStep h[LR_MAX_CHAIN];
  int k = 0;
  for (int s = 0; s < n_steps; ++s) {
    for (int p = 0; p < steps[s].n; ++p, ++k) {
      descs[s][p] = steps[s].proj[p];
      const int r = active->ranks[k];
      if (r < 0 || r > descs[s][p].rank) return LR_ERR_INVALID_ARG;
      descs[s][p].active_rank = r == descs[s][p].rank ? 0 : r;
    }
    h[s] = HostStep{descs[s], steps[s].n, steps[s].input_step, steps[s].input_proj, steps[s].y};
  }
  return run_chain(h, n_steps, x, batch, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

lr_status_t lr_linear_chain(const lr_chain_step_t* steps, int n_steps, const void* x, int batch, void* ws,
                            size_t ws_bytes, lr_stream_t stream) {
  if (!steps || n_steps < 1 || n_steps > LR_MAX_CHAIN) return LR_ERR_INVALID_ARG;
  HostStep h[LR_MAX_CHAIN];
  for (int s = 0; s < n_steps; ++s) h[s] = HostStep{steps[s].proj, steps[s].n, steps[s].input_step, steps[s].input_proj, steps[s].y};
  return run_chain(h, n_steps, x, batch, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

// --------------------------------------------------------------------------

static lr_status_t check_ffn(const lr_ffn_desc_t* d) {
  if (!d) return LR_ERR_INVALID_ARG;
  if (d->hidden <= 0 || d->inter <= 0 || d->n_lr < 0 || d->n_lr > d->inter) return LR_ERR_INVALID_ARG;
  if (d->n_lr > 0 && (d->rank <= 0 || !d->A || !d->s_A || !d->B || !d->s_B)) return LR_ERR_INVALID_ARG;
  if (d->inter > d->n_lr && (!d->D || !d->s_D)) return LR_ERR_INVALID_ARG;
  if (!d->W_down || !d->s_down) return LR_ERR_INVALID_ARG;
  if (d->scale_dtype != LR_F16 && d->scale_dtype != LR_F32) return LR_ERR_UNSUPPORTED;
  if ((d->hidden % 16) != 0 || (d->n_lr % 8) != 0) return LR_ERR_UNSUPPORTED;
  if (d->hidden > 32768 || 2 * d->n_lr > 32768) return LR_ERR_UNSUPPORTED;
  const void* ptrs[] = {d->A, d->s_A, d->B, d->s_B, d->D, d->s_D, d->W_down, d->s_down};
  for (const void* p : ptrs)
    if (p && !al16(p)) return LR_ERR_MISALIGNED;
  return LR_OK;
}

// On the tensor-core path the FFN keeps token-major fp32 accumulators: z [rank],
// gu [2 n_lr], dd [2 n_dense], h [inter], y [hidden] per token (rows 8-float
// aligned) for cols tokens, zero on entry and exit.
static size_t ffn_tc_floats_per_token(const lr_ffn_desc_t* d) {
  return round_up(size_t(d->n_lr > 0 ? d->rank : 0), 8) + 2 * size_t(d->inter) + round_up(size_t(d->inter), 8) +
         size_t(d->hidden);
}

// Up to this many tokens in a pass the down projection evaluates the SwiGLU
// while it stages h (each of its row tiles repeats it for its slice); above
// it a SwiGLU kernel writes h once.
constexpr int kFusedSwigluMaxTokens = 4;

static size_t ffn_ws_bytes(const lr_ffn_desc_t* d, int batch) {
  const int chunk = std::min(batch, kMaxDecodeChunk);
  const int n_dense = d->inter - d->n_lr;
  size_t b = kTicketBytes + round_up(size_t(chunk) * 2 * d->n_lr * 4, 256) + round_up(size_t(chunk) * n_dense * 4, 256) +
             round_up(size_t(chunk) * d->hidden * 4, 256);
  if (use_tc_ffn(batch)) b = std::max(b, kTicketBytes + ffn_tc_floats_per_token(d) * size_t(tc_cols(batch)) * 4);
  return b;
}

// The hybrid FFN on the tensor cores (int8 weights, kind::i8), per pass of up
// to kTcMaxPass tokens (every product scales its int8 activation codes per
// token over each unit's slice of the reduction):
//   product 1: z += A' x (low-rank latent) and dd += D x (dense gate/up), scaled per row
//   product 2: gu += B'^T z (low-rank gate/up), scaled per column of B'
//   up to kFusedSwigluMaxTokens tokens:
//     product 3: y += W_down^T h with h = silu(g) u of both branches, evaluated
//                while the product stages its activations; it first zeroes z
//     finalize:  y (bf16), clearing the y accumulator; zeroes gu and dd
//   more tokens:
//     SwiGLU:    h = silu(g) u (clears gu, dd; zeroes z)
//     product 3: y += W_down^T h
//     finalize:  y (bf16), clearing the y accumulator; zeroes h
static lr_status_t run_ffn_tc(const lr_ffn_desc_t* d, const void* x, int batch, void* y, void* ws,
                              cudaStream_t stream) {
  const int cols = tc_cols(batch);
  const int n_dense = d->inter - d->n_lr;
  const int rz = d->n_lr > 0 ? int(round_up(size_t(d->rank), 8)) : 0;
  float* zacc = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kTicketBytes);
  float* gu = zacc + size_t(rz) * cols;
  float* dd = gu + size_t(2 * d->n_lr) * cols;
  const int hld = int(round_up(size_t(d->inter), 8));
  float* h = dd + size_t(2 * n_dense) * cols;
  float* yacc = h + size_t(hld) * cols;
  int* err = device_error_word();
  const int sms = sm_count_current();
  const int f16 = d->scale_dtype == LR_F16 ? 1 : 0;
  for (int b0 = 0; b0 < batch; b0 += kTcMaxPass) {
    const int nb = std::min(kTcMaxPass, batch - b0);
    const int nh = int(round_up(size_t(nb), 8));
    const int N = std::max(16, 2 * nh);
    const void* xb = reinterpret_cast<const char*>(x) + size_t(b0) * d->hidden * 2;
    auto seg = [&](TcGemvParams& g, TcMaps& maps, int i, const void* W, int rows, int cols_w, int mn, int M, int K,
                   const void* act, int act_kind, int act_ld, float* out, int out_ld, const void* rs) -> bool {
      if (!weight_map(&maps.m[i], W, rows, cols_w, mn, true)) return false;
      TcSeg& sg = g.seg[i];
      sg.M = M;
      sg.K = K;
      sg.a_mn_major = mn;
      sg.act = act;
      sg.act_kind = act_kind;
      sg.act_ld = act_ld;
      sg.out = out;
      sg.out_ld = out_ld;
      sg.row_scale = rs;
      sg.row_scale_f16 = f16;
      g.nseg = i + 1;
      return true;
    };
    TcMaps maps;
    TcGemvParams g;
    std::memset(&maps, 0, sizeof(maps));
    std::memset(&g, 0, sizeof(g));
    g.nb = nb;
    g.N = N;
    g.hilo = 1;
    g.err = err;
    int i = 0;
    if (d->n_lr > 0 &&
        !seg(g, maps, i++, d->A, d->rank, d->hidden, 0, d->rank, d->hidden, xb, 0, d->hidden, zacc, rz, d->s_A))
      return LR_ERR_CUDA;
    if (n_dense > 0 && !seg(g, maps, i++, d->D, 2 * n_dense, d->hidden, 0, 2 * n_dense, d->hidden, xb, 0,
                            d->hidden, dd, 2 * n_dense, d->s_D))
      return LR_ERR_CUDA;
    cudaError_t e = tc_product(maps, g, sms, true, stream);
    if (e != cudaSuccess) return from_cuda(e);
    if (d->n_lr > 0) {
      std::memset(&maps, 0, sizeof(maps));
      if (!seg(g, maps, 0, d->B, d->rank, 2 * d->n_lr, 1, 2 * d->n_lr, d->rank, zacc, 1, rz, gu, 2 * d->n_lr, d->s_B))
        return LR_ERR_CUDA;
      g.nseg = 1;
      e = tc_product(maps, g, sms, true, stream);
      if (e != cudaSuccess) return from_cuda(e);
    }
    const bool fused = nb <= kFusedSwigluMaxTokens;
    std::memset(&maps, 0, sizeof(maps));
    if (fused) {
      if (!seg(g, maps, 0, d->W_down, d->inter, d->hidden, 1, d->hidden, d->inter, gu, 2, 2 * d->n_lr, yacc,
               d->hidden, d->s_down))
        return LR_ERR_CUDA;
      g.seg[0].act2 = dd;
      g.seg[0].act2_ld = 2 * n_dense;
      g.seg[0].n_lr = d->n_lr;
      if (rz > 0) {   // the latent, read by product 2 only
        g.pre.zero[0] = zacc;
        g.pre.zero_floats[0] = size_t(rz) * cols;
        g.pre.nz = 1;
      }
    } else {
      TcSwigluParams sw;
      std::memset(&sw, 0, sizeof(sw));
      sw.gu = gu;
      sw.dd = dd;
      sw.h = h;
      sw.h_ld = hld;
      sw.n_lr = d->n_lr;
      sw.n_dense = n_dense;
      sw.nb = nb;
      sw.zero = rz ? zacc : nullptr;
      sw.zero_row = rz;
      e = launch_tc_swiglu(sw, stream);
      if (e != cudaSuccess) return from_cuda(e);
      if (!seg(g, maps, 0, d->W_down, d->inter, d->hidden, 1, d->hidden, d->inter, h, 1, hld, yacc, d->hidden,
               d->s_down))
        return LR_ERR_CUDA;
    }
    g.nseg = 1;
    e = tc_product(maps, g, sms, true, stream);
    if (e != cudaSuccess) return from_cuda(e);
    TcFinalizeParams f;
    std::memset(&f, 0, sizeof(f));
    f.nt = 1;
    f.nb = nb;
    f.zero_targets = 1;
    f.t[0].acc = yacc;
    f.t[0].y = reinterpret_cast<char*>(y) + size_t(b0) * d->hidden * 2;
    f.t[0].M = d->hidden;
    if (fused) {
      f.zero[0] = gu;   // the gate/up accumulators of both branches, read by product 3
      f.zero_floats[0] = size_t(2 * d->inter) * cols;
    } else {
      f.zero[0] = h;    // read by product 3
      f.zero_floats[0] = size_t(hld) * cols;
    }
    f.nz = 1;
    e = launch_tc_finalize(f, sms, stream);
    if (e != cudaSuccess) return from_cuda(e);
  }
  return LR_OK;
}

lr_status_t lr_dense_linear(const void* W, lr_dtype_t w_dtype, const void* scale, lr_dtype_t scale_dtype, int d_in,
                            int d_out, const void* x, int batch, void* y, lr_stream_t stream) {
  if (!W || !x || !y || d_in <= 0 || d_out <= 0 || batch < 1) return LR_ERR_INVALID_ARG;
  if (w_dtype != LR_BF16 && w_dtype != LR_I8) return LR_ERR_UNSUPPORTED;
  if (w_dtype == LR_I8 && !scale) return LR_ERR_INVALID_ARG;
  if (scale && scale_dtype != LR_F16 && scale_dtype != LR_F32) return LR_ERR_UNSUPPORTED;
  const size_t es = w_dtype == LR_BF16 ? 2 : 1;
  if ((d_in % 16) != 0 || size_t(d_in) * es > 32768) return LR_ERR_UNSUPPORTED;
  if (!al16(W) || !al16(x) || !al16(y) || (scale && !al16(scale))) return LR_ERR_MISALIGNED;
  FfnParams P;
  std::memset(&P, 0, sizeof(P));
  P.hidden = d_in;
  P.n_dense = d_out;
  P.nb = batch;
  P.D = reinterpret_cast<const int8_t*>(W);
  P.sD = scale;
  P.scale_f16 = scale_dtype == LR_F16 ? 1 : 0;
  P.x = x;
  P.y = y;
  P.err = device_error_word();
  return from_cuda(launch_dense(P, w_dtype, sm_count_current(), reinterpret_cast<cudaStream_t>(stream)));
}

lr_status_t lr_swiglu_ffn_workspace_size(const lr_ffn_desc_t* desc, int batch, size_t* bytes) {
  if (!bytes || batch < 1) return LR_ERR_INVALID_ARG;
  lr_status_t st = check_ffn(desc);
  if (st != LR_OK) return st;
  *bytes = ffn_ws_bytes(desc, batch);
  return LR_OK;
}

lr_status_t lr_swiglu_ffn(const lr_ffn_desc_t* d, const void* x, int batch, void* y, void* ws, size_t ws_bytes,
                          lr_stream_t stream) {
  lr_status_t st = check_ffn(d);
  if (st != LR_OK) return st;
  if (!x || !y || batch < 1) return LR_ERR_INVALID_ARG;
  if (!al16(x) || !al16(y)) return LR_ERR_MISALIGNED;
  if (!ws || ws_bytes < ffn_ws_bytes(d, batch)) return LR_ERR_WORKSPACE;
  if (!al16(ws)) return LR_ERR_MISALIGNED;
  if (use_tc_ffn(batch)) return run_ffn_tc(d, x, batch, y, ws, reinterpret_cast<cudaStream_t>(stream));
  const int chunk = std::min(batch, kMaxDecodeChunk);
  FfnParams P;
  std::memset(&P, 0, sizeof(P));
  P.hidden = d->hidden; P.inter = d->inter; P.n_lr = d->n_lr; P.n_dense = d->inter - d->n_lr; P.rank = d->rank;
  P.scale_f16 = d->scale_dtype == LR_F16 ? 1 : 0;
  P.A = d->A; P.sA = d->s_A; P.B = d->B; P.sB = d->s_B; P.D = d->D; P.sD = d->s_D; P.Wd = d->W_down; P.sd = d->s_down;
  char* w = reinterpret_cast<char*>(ws);
  P.ticket = reinterpret_cast<unsigned int*>(w);
  w += kTicketBytes;
  P.gu_acc = reinterpret_cast<float*>(w);
  w += round_up(size_t(chunk) * 2 * d->n_lr * 4, 256);
  P.h_dense = reinterpret_cast<float*>(w);
  w += round_up(size_t(chunk) * P.n_dense * 4, 256);
  P.y_acc = reinterpret_cast<float*>(w);
  P.wait_ns = grid_wait_ns();
  P.err = device_error_word();
  const int sms = sm_count_current();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int b0 = 0; b0 < batch; b0 += kMaxDecodeChunk) {
    P.nb = std::min(kMaxDecodeChunk, batch - b0);
    P.x = reinterpret_cast<const char*>(x) + size_t(b0) * d->hidden * 2;
    P.y = reinterpret_cast<char*>(y) + size_t(b0) * d->hidden * 2;
    st = from_cuda(launch_ffn(P, sms, s));
    if (st != LR_OK) return st;
  }
  return LR_OK;
}

// --------------------------------------------------------------------------

static lr_status_t check_kv(const lr_latent_kv_desc_t* d, int* split) {
  if (!d || !d->B_K || !d->B_V) return LR_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->heads <= 0 || d->max_ctx <= 0 || d->rank <= 0 || d->head_dim <= 0) return LR_ERR_INVALID_ARG;
  if (d->rank != 32 || d->head_dim != 128) return LR_ERR_UNSUPPORTED;
  if (d->mode != LR_KV_ABSORBED && d->mode != LR_KV_RECONSTRUCT) return LR_ERR_UNSUPPORTED;
  if (!(d->rope_base >= 0.0f) || std::isinf(d->rope_base)) return LR_ERR_INVALID_ARG;
  // a rotation of the keys makes the absorbed score inexact
  if (d->mode == LR_KV_ABSORBED && d->rope_base != 0.0f) return LR_ERR_UNSUPPORTED;
  if (d->split_tokens < 0 || (d->split_tokens % 64) != 0 || d->split_tokens > 1024) return LR_ERR_INVALID_ARG;
  if (d->heads > 65535 || d->batch > 65535) return LR_ERR_UNSUPPORTED;
  if (!al16(d->B_K) || !al16(d->B_V)) return LR_ERR_MISALIGNED;
  int t = d->split_tokens;
  if (d->mode == LR_KV_RECONSTRUCT) {
    // two 128-position tensor-core tiles per work item; tiled-copy row coordinates are 32-bit
    if (t != 0 && t != latent_kv_rope_split()) return LR_ERR_UNSUPPORTED;
    if (double(d->batch) * d->heads * d->max_ctx + 256.0 >= 2147483648.0) return LR_ERR_UNSUPPORTED;
    t = latent_kv_rope_split();
  }
  if (t == 0) t = 256;  // measured best at ctx 4K-32K (8 x 32 heads): 32 KiB of cache per CTA, 6 CTAs per SM
  *split = t;
  return LR_OK;
}

// int8 caches: twice the positions per split keep 32 KiB of cache per CTA.
static int kv_split_q8(const lr_latent_kv_desc_t* d, int t) { return d->split_tokens ? t : 2 * t; }

static size_t kv_partial_bytes(const lr_latent_kv_desc_t* d, int t) {
  const size_t ns = (size_t(d->max_ctx) + t - 1) / t;
  return round_up(size_t(d->batch) * d->heads * ns * (d->rank + 2) * 4, 256);
}

lr_status_t lr_latent_kv_workspace_size(const lr_latent_kv_desc_t* d, size_t* bytes) {
  int t = 0;
  if (!bytes) return LR_ERR_INVALID_ARG;
  lr_status_t st = check_kv(d, &t);
  if (st != LR_OK) return st;
  *bytes = kv_partial_bytes(d, t) + size_t(d->batch) * d->heads * d->rank * 4;
  return LR_OK;
}

static lr_status_t run_latent_kv(const lr_latent_kv_desc_t* d, const void* q, const void* C_K, const void* s_K,
                                 const void* C_V, const void* s_V, bool q8, const int* seq_lens, void* out, void* ws,
                                 size_t ws_bytes, lr_stream_t stream) {
  int t = 0;
  lr_status_t st = check_kv(d, &t);
  if (st != LR_OK) return st;
  if (q8) t = kv_split_q8(d, t);  // fewer splits: the workspace sized for t suffices
  if (!q || !C_K || !C_V || !seq_lens || !out) return LR_ERR_INVALID_ARG;
  if (!al16(q) || !al16(C_K) || !al16(C_V) || !al16(seq_lens) || !al16(out)) return LR_ERR_MISALIGNED;
  if (q8) {
    if (d->mode != LR_KV_ABSORBED) return LR_ERR_UNSUPPORTED;
    if (!s_K || !s_V) return LR_ERR_INVALID_ARG;
    if (d->cache_scale_dtype != LR_F16 && d->cache_scale_dtype != LR_F32) return LR_ERR_UNSUPPORTED;
  }
  size_t need = 0;
  lr_latent_kv_workspace_size(d, &need);
  if (!ws || ws_bytes < need) return LR_ERR_WORKSPACE;
  if (!al16(ws)) return LR_ERR_MISALIGNED;
  LatentKvParams P;
  std::memset(&P, 0, sizeof(P));
  P.batch = d->batch; P.heads = d->heads; P.head_dim = d->head_dim; P.rank = d->rank; P.max_ctx = d->max_ctx;
  P.split_tokens = t; P.n_splits = (d->max_ctx + t - 1) / t; P.scale = d->scale;
  P.q = q; P.CK = C_K; P.CV = C_V; P.BK = d->B_K; P.BV = d->B_V; P.seq_lens = seq_lens; P.out = out;
  P.partial = reinterpret_cast<float*>(ws);
  P.qt = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kv_partial_bytes(d, t));
  P.mode = d->mode;
  P.cache_q8 = q8 ? 1 : 0;
  P.cache_scale_f16 = d->cache_scale_dtype == LR_F16 ? 1 : 0;
  P.sK = s_K; P.sV = s_V;
  P.err = device_error_word();
  if (d->mode == LR_KV_RECONSTRUCT) {
    KvRopeParams R;
    std::memset(&R, 0, sizeof(R));
    R.p = P;
    for (int i = 0; i < d->head_dim / 2; ++i) {
      R.theta_d[i] = d->rope_base > 0.0f ? std::pow(double(d->rope_base), -2.0 * i / d->head_dim) : 0.0;
      R.theta_f[i] = float(R.theta_d[i]);
    }
    return from_cuda(launch_latent_kv_rope(R, sm_count_current(), reinterpret_cast<cudaStream_t>(stream)));
  }
  return from_cuda(launch_latent_kv(P, reinterpret_cast<cudaStream_t>(stream)));
}

static lr_status_t check_append(const lr_latent_kv_desc_t* d, const void* A_KV, int hidden) {
  if (!d || !A_KV) return LR_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->heads <= 0 || d->rank <= 0 || d->max_ctx <= 0 || hidden <= 0) return LR_ERR_INVALID_ARG;
  if ((hidden % 16) != 0 || size_t(hidden) * 2 > 32768) return LR_ERR_UNSUPPORTED;
  if (double(2) * d->heads * d->rank > 2147483647.0) return LR_ERR_UNSUPPORTED;
  return LR_OK;
}

// The tensor-core path needs 8-float aligned accumulator rows (2 H r a multiple of 8).
static bool append_tc(const lr_latent_kv_desc_t* d) { return (size_t(d->heads) * d->rank) % 4 == 0; }

lr_status_t lr_latent_kv_append_workspace_size(const lr_latent_kv_desc_t* d, int hidden, size_t* bytes) {
  if (!bytes) return LR_ERR_INVALID_ARG;
  lr_status_t st = check_append(d, reinterpret_cast<const void*>(16), hidden);
  if (st != LR_OK) return st;
  *bytes = append_tc(d) ? kTicketBytes + size_t(2) * d->heads * d->rank * size_t(tc_cols(d->batch)) * 4 : 0;
  return LR_OK;
}

lr_status_t lr_latent_kv_append(const lr_latent_kv_desc_t* d, const void* A_KV, int hidden, const void* x,
                                const int* pos, void* C_K, void* C_V, void* ws, size_t ws_bytes,
                                lr_stream_t stream) {
  lr_status_t st = check_append(d, A_KV, hidden);
  if (st != LR_OK) return st;
  if (!x || !pos || !C_K || !C_V) return LR_ERR_INVALID_ARG;
  if (!al16(A_KV) || !al16(x) || !al16(pos) || !al16(C_K) || !al16(C_V)) return LR_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int width = 2 * d->heads * d->rank;
  if (ws && append_tc(d)) {
    // tensor cores: latents = x A_KV^T into a token-major fp32 accumulator, then scattered
    size_t need = 0;
    lr_latent_kv_append_workspace_size(d, hidden, &need);
    if (ws_bytes < need) return LR_ERR_WORKSPACE;
    if (!al16(ws)) return LR_ERR_MISALIGNED;
    float* acc = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kTicketBytes);
    const int sms = sm_count_current();
    const size_t per_seq = size_t(d->heads) * d->max_ctx * d->rank * 2;  // bytes of one sequence's cache
    for (int b0 = 0; b0 < d->batch; b0 += kTcMaxPass) {
      const int nb = std::min(kTcMaxPass, d->batch - b0);
      TcMaps maps;
      TcGemvParams g;
      std::memset(&maps, 0, sizeof(maps));
      std::memset(&g, 0, sizeof(g));
      if (!weight_map(&maps.m[0], A_KV, width, hidden, 0, false)) return LR_ERR_CUDA;
      g.nseg = 1;
      g.nb = nb;
      g.N = int(round_up(size_t(nb), 16));
      g.hilo = 0;
      g.err = device_error_word();
      TcSeg& sg = g.seg[0];
      sg.M = width;
      sg.K = hidden;
      sg.act = reinterpret_cast<const char*>(x) + size_t(b0) * hidden * 2;
      sg.act_kind = 0;
      sg.act_ld = hidden;
      sg.out = acc;
      sg.out_ld = width;
      cudaError_t e = tc_product(maps, g, sms, false, s);
      if (e != cudaSuccess) return from_cuda(e);
      TcScatterParams sp;
      sp.acc = acc;
      sp.cache_k = reinterpret_cast<char*>(C_K) + size_t(b0) * per_seq;
      sp.cache_v = reinterpret_cast<char*>(C_V) + size_t(b0) * per_seq;
      sp.pos = pos + b0;
      sp.nb = nb;
      sp.heads = d->heads;
      sp.rank = d->rank;
      sp.ctx = d->max_ctx;
      e = launch_tc_cache_scatter(sp, s);
      if (e != cudaSuccess) return from_cuda(e);
    }
    return LR_OK;
  }
  FfnParams P;
  std::memset(&P, 0, sizeof(P));
  P.hidden = hidden;
  P.n_dense = width;
  P.nb = d->batch;
  P.D = reinterpret_cast<const int8_t*>(A_KV);
  P.x = x;
  P.cache_k = C_K;
  P.cache_v = C_V;
  P.cache_pos = pos;
  P.cache_heads = d->heads;
  P.cache_rank = d->rank;
  P.cache_ctx = d->max_ctx;
  P.err = device_error_word();
  return from_cuda(launch_dense(P, LR_BF16, sm_count_current(), s));
}

lr_status_t lr_latent_kv_decode(const lr_latent_kv_desc_t* d, const void* q, const void* C_K, const void* C_V,
                                const int* seq_lens, void* out, void* ws, size_t ws_bytes, lr_stream_t stream) {
  return run_latent_kv(d, q, C_K, nullptr, C_V, nullptr, false, seq_lens, out, ws, ws_bytes, stream);
}

lr_status_t lr_latent_kv_decode_q8(const lr_latent_kv_desc_t* d, const void* q, const int8_t* C_K, const void* s_K,
                                   const int8_t* C_V, const void* s_V, const int* seq_lens, void* out, void* ws,
                                   size_t ws_bytes, lr_stream_t stream) {
  return run_latent_kv(d, q, C_K, s_K, C_V, s_V, true, seq_lens, out, ws, ws_bytes, stream);
}

// --------------------------------------------------------------------------

static lr_status_t check_flash(const lr_flash_desc_t* d, int* split) {
  if (!d) return LR_ERR_INVALID_ARG;
  if (d->batch <= 0 || d->heads <= 0 || d->max_ctx <= 0 || d->head_dim <= 0) return LR_ERR_INVALID_ARG;
  if (d->head_dim != 128) return LR_ERR_UNSUPPORTED;
  if (d->split_tokens < 0 || (d->split_tokens % 64) != 0 || d->split_tokens > 256) return LR_ERR_INVALID_ARG;
  if (d->heads > 65535 || d->batch > 65535) return LR_ERR_UNSUPPORTED;
  *split = d->split_tokens ? d->split_tokens : 128;
  return LR_OK;
}

lr_status_t lr_flash_decode_workspace_size(const lr_flash_desc_t* d, size_t* bytes) {
  int t = 0;
  if (!bytes) return LR_ERR_INVALID_ARG;
  lr_status_t st = check_flash(d, &t);
  if (st != LR_OK) return st;
  const size_t ns = (size_t(d->max_ctx) + t - 1) / t;
  *bytes = size_t(d->batch) * d->heads * ns * flash_partial_floats() * 4;
  return LR_OK;
}

lr_status_t lr_flash_decode(const lr_flash_desc_t* d, const void* q, const void* K, const void* V,
                            const int* seq_lens, void* out, void* ws, size_t ws_bytes, lr_stream_t stream) {
  int t = 0;
  lr_status_t st = check_flash(d, &t);
  if (st != LR_OK) return st;
  if (!q || !K || !V || !seq_lens || !out) return LR_ERR_INVALID_ARG;
  if (!al16(q) || !al16(K) || !al16(V) || !al16(seq_lens) || !al16(out)) return LR_ERR_MISALIGNED;
  size_t need = 0;
  lr_flash_decode_workspace_size(d, &need);
  if (!ws || ws_bytes < need) return LR_ERR_WORKSPACE;
  if (!al16(ws)) return LR_ERR_MISALIGNED;
  FlashParams P;
  std::memset(&P, 0, sizeof(P));
  P.batch = d->batch; P.heads = d->heads; P.max_ctx = d->max_ctx;
  P.split_tokens = t; P.n_splits = (d->max_ctx + t - 1) / t; P.scale = d->scale;
  P.q = q; P.K = K; P.V = V; P.seq_lens = seq_lens; P.out = out;
  P.partial = reinterpret_cast<float*>(ws);
  P.err = device_error_word();
  return from_cuda(launch_flash(P, reinterpret_cast<cudaStream_t>(stream)));
}

lr_status_t lr_quantize_per_token(const void* x, int rows, int cols, int8_t* x_q, float* s, lr_stream_t stream) {
  if (!x || !x_q || !s || rows < 1 || cols < 1) return LR_ERR_INVALID_ARG;
  if ((cols % 16) != 0 || cols > 49152) return LR_ERR_UNSUPPORTED;
  if (!al16(x) || !al16(x_q) || !al16(s)) return LR_ERR_MISALIGNED;
  return from_cuda(launch_quantize_per_token(x, rows, cols, x_q, s, reinterpret_cast<cudaStream_t>(stream)));
}

lr_status_t lr_gemm_s8s32(const int8_t* A, const int8_t* B, int b_layout, int M, int N, int K, int32_t* C,
                          lr_stream_t stream) {
  if (!A || !B || !C || M < 1 || N < 1 || K < 1) return LR_ERR_INVALID_ARG;
  if (b_layout != 0 && b_layout != 1) return LR_ERR_INVALID_ARG;
  if ((K % 16) != 0 || (N % 16) != 0 || K >= 133144) return LR_ERR_UNSUPPORTED;
  if (!al16(A) || !al16(B) || !al16(C)) return LR_ERR_MISALIGNED;
  return from_cuda(launch_gemm_s8s32(A, B, b_layout, M, N, K, C, device_error_word(), sm_count_current(),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

lr_status_t lr_workspace_init(void* ws, size_t ws_bytes, lr_stream_t stream) {
  if (!ws) return LR_ERR_INVALID_ARG;
  if (!al16(ws)) return LR_ERR_MISALIGNED;
  return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

lr_status_t lr_check_device_error(lr_stream_t stream, int* err) {
  if (!err) return LR_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return LR_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, lr::g_device_error, sizeof(int)) != cudaSuccess) return LR_ERR_CUDA;
  *err = v;
  if (v != 0) {
    noalloc_mark_dirty();
    const int zero = 0;
    if (cudaMemcpyToSymbol(lr::g_device_error, &zero, sizeof(int)) != cudaSuccess) return LR_ERR_CUDA;
    return LR_ERR_DEVICE_TIMEOUT;
  }
  return LR_OK;
}

const char* lr_status_string(lr_status_t s) {
  switch (s) {
    case LR_OK: return "ok";
    case LR_ERR_INVALID_ARG: return "invalid argument";
    case LR_ERR_UNSUPPORTED: return "unsupported dtype or shape";
    case LR_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case LR_ERR_WORKSPACE: return "workspace missing or too small";
    case LR_ERR_CUDA: return "CUDA error";
    case LR_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

int lr_version(void) { return 100; }

}  // extern "C"
