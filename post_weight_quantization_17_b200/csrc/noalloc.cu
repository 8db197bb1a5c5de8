// gptq_quantize_layer_noalloc: gptq_quantize_layer for callers that cannot allocate device
// memory (for example code running inside another allocator's hooks, or a host process whose
// memory budget is fixed before it loads this library).  Its scratch is one file-scope device
// array of GPTQ_NOALLOC_SCRATCH_BYTES that every GPU loading the library keeps until exit; the
// caller still provides all inputs and outputs.
#include "kernels.h"

struct gptq_ctx {
  gptq::Ctx c;
};

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GPTQ_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device, looked up on every call (the
// lookup allocates nothing): an address cached across calls would go stale if the device's
// primary context were torn down and created again.  In host code `g_noalloc_scratch` names a
// host-side stand-in, not device memory, so kernels are given the address this returns.  The
// first lookup on a device loads the library's module there, which is when the array is
// reserved.
int scratch_for_current_device(void** addr, int* device, int* num_sms) {
  if (cudaGetDevice(device) != cudaSuccess) return GPTQ_ERR_CUDA;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GPTQ_ERR_CUDA;
  if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, *device) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  *addr = p;
  return GPTQ_OK;
}

}  // namespace

extern "C" int gptq_quantize_layer_noalloc(void* cuda_stream, const void* W, int w_dtype,
                                           int64_t m, int64_t d, const float* R,
                                           const int32_t* perm, const uint8_t* dead, int bits,
                                           int group, int block, int grid_given, float* scales,
                                           int32_t* zeros, uint8_t* codes, float* W_hat,
                                           float* col_loss) {
  void* scratch = nullptr;
  int device = 0, num_sms = 0;
  int rc = scratch_for_current_device(&scratch, &device, &num_sms);
  if (rc) return rc;
  // the scratch address belongs to the current device, so the stream must belong to it too
  // (the legacy default stream, NULL, always does)
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(cuda_stream);
  if (stream) {
    int sdev = -1;
    if (cudaStreamGetDevice(stream, &sdev) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (sdev != device) return GPTQ_ERR_ARG;
  }
  gptq_ctx tmp;
  tmp.c.stream = stream;
  tmp.c.device = device;
  tmp.c.num_sms = num_sms;
  tmp.c.ws = reinterpret_cast<char*>(scratch);
  tmp.c.ws_bytes = GPTQ_NOALLOC_SCRATCH_BYTES;
  tmp.c.owns_ws = false;
  tmp.c.status = reinterpret_cast<gptq::DeviceStatus*>(scratch);
  // the status word must start at zero; the rest of the scratch is written before it is read
  if (cudaMemsetAsync(scratch, 0, gptq::kStatusBytes, stream) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  rc = gptq_quantize_layer(&tmp, W, w_dtype, m, d, R, perm, dead, bits, group, block, grid_given,
                           scales, zeros, codes, W_hat, col_loss);
  // ARG and NOMEM are found before any kernel is enqueued; NOMEM means the layer needs more
  // than the fixed scratch, which is an argument error of this entry point
  if (rc == GPTQ_ERR_NOMEM) return GPTQ_ERR_ARG;
  if (rc == GPTQ_ERR_ARG) return rc;
  if (rc) {
    // a launch failed after earlier kernels were enqueued: let those finish before returning,
    // so that the caller may reuse its buffers
    cudaStreamSynchronize(stream);
    return rc;
  }
  return gptq_sync_status(&tmp);
}
