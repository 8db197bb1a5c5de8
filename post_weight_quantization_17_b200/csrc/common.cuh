// Shared definitions of the GPTQ sm_100a library: context, status flag, launch helpers.
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stdio.h>
#include <string>

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

struct Ctx {
  cudaStream_t stream = nullptr;
  int device = 0;
  int num_sms = 148;
  char* ws = nullptr;          // workspace base (device)
  size_t ws_bytes = 0;
  bool owns_ws = false;
  DeviceStatus* status = nullptr;  // lives at the start of ws
  std::string last_error;
  long long timeout_cycles = 4000000000LL;  // bounded waits in the pipelined kernels
  unsigned long long launches = 0;          // kernels this context has launched
  cudaStream_t side = nullptr;              // second stream of the factorization recursion
  cudaEvent_t ev[2 * 64] = {};              // its per-level events
};

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

#define GPTQ_LAUNCH_CHECK(ctx)                                                  \
  do {                                                                          \
    (ctx)->launches++;                                                          \
    GPTQ_CUDA_CHECK(ctx, cudaGetLastError());                                   \
  } while (0)
