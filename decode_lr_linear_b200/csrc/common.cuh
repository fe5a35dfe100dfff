// Device helpers shared by the sm_100a kernels of the low-rank decode library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#define LR_DEV __device__ __forceinline__
#define LR_HD_INLINE __host__ __device__ __forceinline__

namespace lr {

// Codes stored in the library's device error word (read by lr_check_device_error).
// Kernels receive the word's device address in their parameters.
enum DeviceErrorCode : int {
  kErrNone = 0,
  kErrMbarTimeout = 1,   // an mbarrier wait gave up
  kErrTmemTimeout = 2,   // a TMEM allocation could not be obtained
  kErrGridBarrier = 3,   // a grid-wide barrier wait gave up
};

LR_DEV void set_device_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Bounds of the waits, in nanoseconds of the GPU's global timer.  A wait for
// this CTA's own asynchronous copies (an mbarrier) only ends early if the
// memory system has failed; a wait for other CTAs (grid barriers, arrival
// counters) ends early when a CTA of the grid was not resident or a limit
// shorter than the barrier latency was set on purpose.
constexpr uint64_t kMbarTimeoutNs = 2000000000ull;      // 2 s
constexpr uint64_t kGridWaitDefaultNs = 1000000000ull;  // 1 s (lr_set_wait_timeout_us)
constexpr uint64_t kDegradedMbarNs = 1000000ull;        // per stage, after a first mbarrier timeout (1 ms)

LR_DEV uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (PDL).
// wait: block until the preceding grid in the stream has completed and its
// memory is visible; launch_dependents: allow the next grid to be scheduled.
// ---------------------------------------------------------------------------
LR_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
LR_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ---------------------------------------------------------------------------
// Global loads / stores / reductions.
// ---------------------------------------------------------------------------
// Streaming read of data no kernel writes during the call (weights, caches):
// non-coherent path, no L1 allocation.
LR_DEV uint4 ld_stream16(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
LR_DEV uint2 ld_stream8(const void* p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
// Coherent L2 read (data written by other CTAs of the same grid).
LR_DEV float4 ld_cg_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p) : "memory");
  return v;
}
LR_DEV uint4 ld_cg_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p) : "memory");
  return v;
}
LR_DEV unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
LR_DEV void st_cg_f4(float* p, float4 v) {
  asm volatile("st.global.cg.v4.f32 [%0], {%1,%2,%3,%4};" :: "l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w) : "memory");
}
LR_DEV void red_add_f4(float* p, float a, float b, float c, float d) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1,%2,%3,%4};" :: "l"(p), "f"(a), "f"(b),
               "f"(c), "f"(d) : "memory");
}
LR_DEV void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------
// Element conversion: a lane chunk is always 8 consecutive elements.
// ---------------------------------------------------------------------------
LR_DEV void bf16x8_to_f32(const uint4 v, float* f) {
  f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
  f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
  f[4] = __uint_as_float(v.z << 16); f[5] = __uint_as_float(v.z & 0xffff0000u);
  f[6] = __uint_as_float(v.w << 16); f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// int8 -> fp32 exactly: place (q + 128) in the mantissa of 2^23 and subtract.
LR_DEV float i8_biased_to_f32(uint32_t biased_word, int byte) {
  const uint32_t m = __byte_perm(biased_word, 0x4B000000u, 0x7440u + byte);
  return __uint_as_float(m) - 8388736.0f;  // 2^23 + 128
}
LR_DEV void i8x8_to_f32(const uint2 v, float* f) {
  const uint32_t a = v.x ^ 0x80808080u, b = v.y ^ 0x80808080u;
#pragma unroll
  for (int k = 0; k < 4; ++k) { f[k] = i8_biased_to_f32(a, k); f[4 + k] = i8_biased_to_f32(b, k); }
}

template <typename T> struct Chunk;  // 8-element chunk loader for weight type T

template <> struct Chunk<float> {
  static constexpr int kBytes = 32;
  LR_DEV static void load(const float* p, float* f) {
    const uint4 a = ld_stream16(p), b = ld_stream16(p + 4);
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
    f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
  }
};
template <> struct Chunk<__nv_bfloat16> {
  static constexpr int kBytes = 16;
  LR_DEV static void load(const __nv_bfloat16* p, float* f) { bf16x8_to_f32(ld_stream16(p), f); }
};
template <> struct Chunk<int8_t> {
  static constexpr int kBytes = 8;
  LR_DEV static void load(const int8_t* p, float* f) { i8x8_to_f32(ld_stream8(p), f); }
};

// Activation chunk (coherent: activations may come from the previous kernel).
LR_DEV void load_act8(const float* p, float* f) {
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
LR_DEV void load_act8(const __nv_bfloat16* p, float* f) {
  bf16x8_to_f32(*reinterpret_cast<const uint4*>(p), f);
}

LR_DEV float load_scale(const void* s, int i, bool f16) {
  return f16 ? __half2float(reinterpret_cast<const __half*>(s)[i]) : reinterpret_cast<const float*>(s)[i];
}

LR_DEV void store_out(float* y, float v) { *y = v; }
LR_DEV void store_out(__nv_bfloat16* y, float v) { *y = __float2bfloat16_rn(v); }

LR_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
LR_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device) (host
// side); later calls that need no more than what is set do not touch the driver,
// so launches issued during stream capture make no attribute calls.
inline cudaError_t ensure_smem_fn(const void* fn, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> done;
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({fn, dev});
  if (it != done.end() && it->second >= int(bytes)) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e == cudaSuccess) done[{fn, dev}] = int(bytes);
  return e;
}
template <typename Kern>
inline cudaError_t ensure_smem(Kern kern, size_t bytes) {
  return ensure_smem_fn(reinterpret_cast<const void*>(kern), bytes);
}

LR_DEV float silu(float t) { return t / (1.0f + __expf(-t)); }

// ---------------------------------------------------------------------------
// mbarrier + bulk copy (TMA, non-tensor form) with bounded waits.
// ---------------------------------------------------------------------------
LR_DEV uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

LR_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
LR_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
LR_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

LR_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
LR_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
LR_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait: gives up after kMbarTimeoutNs (checked every 64 polls; each
// try_wait itself suspends for a while), records the failure in the device
// error word and returns false.
LR_DEV bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0 && global_ns() - t0 > kMbarTimeoutNs) break;
  }
  set_device_error(err, kErrMbarTimeout);
  return false;
}

// Bounded wait until *word >= target (acquire, gpu scope): gives up after
// limit_ns, records kErrGridBarrier and returns false.
LR_DEV bool wait_counter_geq(const unsigned int* word, unsigned int target, uint64_t limit_ns, int* err) {
  if (ld_acquire_u32(word) >= target) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (ld_acquire_u32(word) >= target) return true;
    if (global_ns() - t0 > limit_ns) break;  // one timer read per poll: cheap next to the acquire load
  }
  set_device_error(err, kErrGridBarrier);
  return false;
}

// 1-D bulk copy global -> shared completing on an mbarrier (16-byte aligned
// addresses, size a multiple of 16).
LR_DEV void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(smem_u32(smem_dst)), "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

}  // namespace lr
