// Shared definitions of the GPTQ sm_100a library: context, status flag, launch helpers.
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdio.h>
#include <string>
#include <utility>
#include <vector>

#include "../../include/gptq.h"

namespace gptq {

// Device-side status word layout (first bytes of the context's workspace).
struct DeviceStatus {
  int code;        // first error code raised by a kernel (0 = none)
  int where;       // kernel-specific detail (e.g. failing pivot index)
  double dsum;     // scratch: reductions that need a deterministic fp64 result
  float lam;       // damping λ in use
  float pad;
};

// Bounded waits.  A pipeline wait (for the next stage, buffer or partial) gives up after the
// context's budget, records GPTQ_ERR_TIMEOUT and makes its CTA unwind.  While unwinding, a CTA
// waits for the copies and tensor-core operations it issued itself, with the fixed drain
// budget: those complete on their own, and no CTA may free TMEM or exit before they have.
constexpr long long kDefaultWaitCycles = 4000000000LL;
constexpr long long kDrainCycles = 4000000000LL;

// One timed launch: CUDA events recorded on the launching stream around the kernel.
struct TimedLaunch {
  int stage;
  cudaEvent_t start, stop;
};

struct Ctx {
  cudaStream_t stream = nullptr;
  int device = 0;
  int num_sms = 148;
  char* ws = nullptr;          // workspace base (device)
  size_t ws_bytes = 0;
  bool owns_ws = false;
  DeviceStatus* status = nullptr;  // lives at the start of ws
  std::string last_error;
  long long timeout_cycles = kDefaultWaitCycles;  // pipeline waits (gptq_set_wait_budget)
  unsigned long long launches = 0;          // kernels this context has launched
  cudaStream_t side = nullptr;              // second stream of the factorization recursion
  cudaEvent_t ev[2 * 64] = {};              // its per-level events
  // per-stage timing (gptq_timing_enable): the stage every launch is counted under, the launches
  // recorded since the last read, and a pool of reusable events
  int stage = GPTQ_STAGE_OTHER;
  bool timing = false;
  std::vector<TimedLaunch> timed;
  std::vector<cudaEvent_t> event_pool;
  size_t pool_used = 0;
};

// Sets the stage that launches are counted under for the lifetime of the scope.
struct StageScope {
  Ctx* c;
  int saved;
  StageScope(Ctx* ctx, int stage) : c(ctx), saved(ctx->stage) { c->stage = stage; }
  ~StageScope() { c->stage = saved; }
};

inline cudaError_t pooled_event(Ctx* c, cudaEvent_t* e) {
  if (c->pool_used == c->event_pool.size()) {
    cudaEvent_t n;
    cudaError_t r = cudaEventCreate(&n);
    if (r != cudaSuccess) return r;
    c->event_pool.push_back(n);
  }
  *e = c->event_pool[c->pool_used++];
  return cudaSuccess;
}

constexpr size_t kStatusBytes = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carves aligned sub-buffers out of the context workspace (after the status block).
struct Carver {
  char* base;
  size_t cap, off;
  Carver(Ctx* c) : base(c->ws), cap(c->ws_bytes), off(kStatusBytes) {}
  template <class T> T* take(size_t count) {
    off = align_up(off, 256);
    T* p = reinterpret_cast<T*>(base + off);
    off += count * sizeof(T);
    return p;
  }
  bool ok() const { return off <= cap; }
};

__device__ __forceinline__ void raise_error(DeviceStatus* st, int code, int where) {
  if (atomicCAS(&st->code, 0, code) == 0) st->where = where;
}

// ---- programmatic dependent launch
// Every kernel is launched with programmatic stream serialization, so it may start while the
// previous kernel of its stream is still running.  Before its first access to memory that the
// previous kernel writes (or reads, for memory this kernel writes) it calls pdl_wait(), which
// returns once that kernel has completed and its writes are visible, and only after that
// pdl_release(), which lets the next kernel start its own set-up.  A kernel that has not waited
// yet may therefore read data written two or more kernels back, never data of the kernel right
// before it.  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(Ctx* c, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                              size_t smem, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c->stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  ++c->launches;
  if (!c->timing) return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  // timed launch: the events serialize this kernel with its neighbours on the stream
  TimedLaunch t{c->stage, nullptr, nullptr};
  cudaError_t r = pooled_event(c, &t.start);
  if (r == cudaSuccess) r = pooled_event(c, &t.stop);
  if (r == cudaSuccess) r = cudaEventRecord(t.start, c->stream);
  if (r == cudaSuccess) r = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (r == cudaSuccess) r = cudaEventRecord(t.stop, c->stream);
  if (r == cudaSuccess) c->timed.push_back(t);
  return r;
}

template <class T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

}  // namespace gptq

#define GPTQ_SET_ERR(ctx, code, ...)                                            \
  do {                                                                          \
    char _b[512];                                                               \
    snprintf(_b, sizeof(_b), __VA_ARGS__);                                      \
    if (ctx) (ctx)->last_error = _b;                                            \
    return (code);                                                              \
  } while (0)

#define GPTQ_CUDA_CHECK(ctx, expr)                                              \
  do {                                                                          \
    cudaError_t _e = (expr);                                                    \
    if (_e != cudaSuccess)                                                      \
      GPTQ_SET_ERR(ctx, GPTQ_ERR_CUDA, "%s: %s (%s:%d)", #expr,                 \
                   cudaGetErrorString(_e), __FILE__, __LINE__);                 \
  } while (0)

// Launches a kernel on the context's stream (programmatic dependent launch, counted).
#define GPTQ_LAUNCH(ctx, ...) GPTQ_CUDA_CHECK(ctx, ::gptq::launch_pdl(ctx, __VA_ARGS__))
