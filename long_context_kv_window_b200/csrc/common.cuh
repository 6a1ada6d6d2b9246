// common.cuh -- shared host/device helpers of libkvc (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <string>

#include "kvc.h"

namespace kvc {

// ---------------------------------------------------------------- host side
// Thread-local reason of the last failing call (kvc_last_error).
void set_error(const std::string& msg);
void clear_error();
kvc_status fail(kvc_status s, const std::string& msg);
kvc_status cuda_fail(cudaError_t e, const char* what);

// Count of kernels launched by this library (kvc_launch_count).
extern std::atomic<int64_t> g_launches;
inline void count_launch(int64_t n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Number of SMs of the current device (cached per device).
int num_sms();

// Unique id (cuCtxGetId) of the CUDA context current on the calling thread,
// 0 if there is none yet or the driver cannot tell.  A device reset ends the
// context and the next runtime call creates one with a new id, so state the
// library sets up once per device (function attributes, the address of a
// static device array) is keyed on it.
uint64_t current_context_id();

// Runs setup() unless it already succeeded on the current device in the
// current context (one cache per kind of set-up).
struct ContextCache {
  std::mutex mu;
  uint64_t ids[64] = {};
};
template <class F>
kvc_status once_per_context(ContextCache& c, F&& setup) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(c.mu);
  const bool slot = dev >= 0 && dev < 64;
  const uint64_t id = current_context_id();
  if (slot && id != 0 && c.ids[dev] == id) return KVC_OK;
  const kvc_status s = setup();
  if (s != KVC_OK) return s;
  if (slot) c.ids[dev] = current_context_id();
  return KVC_OK;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr size_t kWsAlign = 256;
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over the caller's workspace.
struct WsCursor {
  char* base;
  size_t cap;
  size_t off = 0;
  bool ok = true;
  template <class T>
  T* take(size_t count) {
    size_t bytes = round_up(count * sizeof(T), kWsAlign);
    if (off + bytes > cap) {
      ok = false;
      return nullptr;
    }
    T* p = reinterpret_cast<T*>(base + off);
    off += bytes;
    return p;
  }
};

#define KVC_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t _e = (expr);                                 \
    if (_e != cudaSuccess) return ::kvc::cuda_fail(_e, #expr); \
  } while (0)

#define KVC_CHECK_ARG(cond, msg) \
  do {                           \
    if (!(cond)) return ::kvc::fail(KVC_ERR_INVALID_ARG, msg); \
  } while (0)

// ------------------------------------------------ programmatic dependent launch
// Every kernel of the library is launched with programmatic stream
// serialization: its CTAs may start once every CTA of the previous kernel in
// the stream has called pdl_trigger() (or exited), i.e. while that kernel
// still runs.  A kernel calls pdl_wait() -- which returns once the previous
// kernel has completed and its memory is visible -- before it touches global
// memory that an earlier kernel of the stream writes or reads, and calls
// pdl_trigger() (if at all) only after its own pdl_wait(): then whatever a
// kernel reads before its pdl_wait() (inputs of the library call) was
// complete before the previous kernel passed its own wait, and a kernel is
// never started while the kernel two places before it still runs.  Only
// kernels whose grid is resident at once and whose dependents cannot hold
// the SMs their own unscheduled CTAs would need trigger early (scoring pass 1,
// the bias combine, the statistics); the others let their dependents launch
// at completion.
struct Launch {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  Launch(dim3 grid, dim3 block, size_t smem, cudaStream_t st) : cfg{}, attr{} {
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  Launch(const Launch&) = delete;
  Launch& operator=(const Launch&) = delete;
  // thread-block clusters of x CTAs along the grid's x axis
  void cluster_x(unsigned x) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  template <class... K, class... A>
  cudaError_t run(void (*kernel)(K...), A&&... args) const {
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<A&&>(args)...);
  }
};

// -------------------------------------------------------------- device side
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_dev_err(int32_t* err, int32_t bit) {
  if (err) atomicOr(err, bit);
}

// Sequence b of a (possibly ragged) batch: [start, start + len).
// cu == nullptr means a single sequence of length `n`.
struct SeqSpan {
  int64_t start;
  int64_t len;
};
__device__ __forceinline__ SeqSpan seq_span(const int32_t* cu, int b, int64_t n) {
  if (cu == nullptr) return {0, n};
  int64_t s = cu[b], e = cu[b + 1];
  return {s, e - s};
}

}  // namespace kvc
