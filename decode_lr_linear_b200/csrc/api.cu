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

// Floats of one accumulator set: the largest step's outputs for one batch chunk.
size_t chain_acc_set(const HostStep* steps, int n_steps, int batch) {
  const int chunk = std::min(batch, kMaxDecodeChunk);
  size_t m = 0;
  for (int s = 0; s < n_steps; ++s) {
    size_t t = 0;
    for (int p = 0; p < steps[s].n; ++p) t += size_t(chunk) * steps[s].d[p].d_out;
    m = std::max(m, t);
  }
  return round_up(m, 64);
}

size_t chain_ws_bytes(const HostStep* steps, int n_steps, int batch) {
  return kTicketBytes + 3 * chain_acc_set(steps, n_steps, batch) * 4;
}

size_t rank1_ws_bytes(const lr_factor_desc_t* descs, int n, int batch) {
  HostStep h{descs, n, -1, 0, nullptr};
  return chain_ws_bytes(&h, 1, batch);
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

lr_status_t run_chain(const HostStep* steps, int n_steps, const void* x, int batch, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
  lr_status_t st = check_chain(steps, n_steps);
  if (st != LR_OK) return st;
  if (!x || batch < 1) return LR_ERR_INVALID_ARG;
  if (!al16(x)) return LR_ERR_MISALIGNED;
  if (!ws || ws_bytes < chain_ws_bytes(steps, n_steps, batch)) return LR_ERR_WORKSPACE;
  if (!al16(ws)) return LR_ERR_MISALIGNED;
  const lr_dtype_t wt = steps[0].d[0].w_dtype;
  const size_t es = (wt == LR_F32) ? 4 : 2;  // activation / output element size
  static ChainParams P;                      // large (kernel parameters); filled under a lock
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  std::memset(&P, 0, sizeof(P));
  P.n_steps = n_steps;
  P.scale_f16 = steps[0].d[0].scale_dtype == LR_F16 ? 1 : 0;
  P.bar = reinterpret_cast<unsigned int*>(ws);
  P.acc = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kTicketBytes);
  P.acc_set = int(chain_acc_set(steps, n_steps, batch));
  P.err = device_error_word();
  P.wait_ns = grid_wait_ns();
  int x_width = 0;
  for (int s = 0; s < n_steps; ++s) {
    ChainStep& c = P.step[s];
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
                      size_t ws_bytes, cudaStream_t stream) {
  HostStep h{descs, n, -1, 0, ys};
  return run_chain(&h, 1, x, batch, ws, ws_bytes, stream);
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
  if (rank1_ws_bytes(desc, 1, batch) > size_t(LR_NOALLOC_SCRATCH_BYTES)) return LR_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  st = noalloc_scratch(s, &ws);
  if (st != LR_OK) return st;
  void* ys[1] = {y};
  return run_rank1(desc, 1, x, batch, ys, ws, LR_NOALLOC_SCRATCH_BYTES, s);
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
    P.z = reinterpret_cast<float*>(w);
    w += round_up(size_t(batch) * r * 4, 256);
    P.zq = reinterpret_cast<int8_t*>(w);
    w += round_up(size_t(round_up(batch, 128)) * P.rank_pad, 256);
    P.sz = reinterpret_cast<float*>(w);
    w += round_up(size_t(round_up(batch, 128)) * 4, 256);
    P.amax = reinterpret_cast<unsigned int*>(w);
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

static size_t ffn_ws_bytes(const lr_ffn_desc_t* d, int batch) {
  const int chunk = std::min(batch, kMaxDecodeChunk);
  const int n_dense = d->inter - d->n_lr;
  return kTicketBytes + round_up(size_t(chunk) * 2 * d->n_lr * 4, 256) + round_up(size_t(chunk) * n_dense * 4, 256) +
         round_up(size_t(chunk) * d->hidden * 4, 256);
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
  if (d->mode != LR_KV_ABSORBED) return LR_ERR_UNSUPPORTED;
  if (d->split_tokens < 0 || (d->split_tokens % 64) != 0 || d->split_tokens > 1024) return LR_ERR_INVALID_ARG;
  if (d->heads > 65535 || d->batch > 65535) return LR_ERR_UNSUPPORTED;
  if (!al16(d->B_K) || !al16(d->B_V)) return LR_ERR_MISALIGNED;
  int t = d->split_tokens;
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
  return from_cuda(launch_latent_kv(P, reinterpret_cast<cudaStream_t>(stream)));
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
  return from_cuda(launch_gemm_s8s32(A, B, b_layout, M, N, K, C, device_error_word(),
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
