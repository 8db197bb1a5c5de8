// gptq_quantize_layer_noalloc: gptq_quantize_layer for callers that cannot allocate device
// memory (for example code running inside another allocator's hooks, or a host process whose
// memory budget is fixed before it loads this library).  Its scratch is one file-scope device
// array of GPTQ_NOALLOC_SCRATCH_BYTES that every GPU loading the library keeps until exit; the
// caller still provides all inputs and outputs.
#include <mutex>

#include "kernels.h"

struct gptq_ctx {
  gptq::Ctx c;
};

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GPTQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.  In
// host code `g_noalloc_scratch` names a host-side stand-in, not device memory, so kernels are
// given the address cudaGetSymbolAddress returns.
int scratch_for_current_device(void** addr, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GPTQ_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_num_sms[dev] = sms;
  }
  *addr = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
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
  int num_sms = 0;
  int rc = scratch_for_current_device(&scratch, &num_sms);
  if (rc) return rc;
  gptq_ctx tmp;
  tmp.c.stream = reinterpret_cast<cudaStream_t>(cuda_stream);
  cudaGetDevice(&tmp.c.device);
  tmp.c.num_sms = num_sms;
  tmp.c.ws = reinterpret_cast<char*>(scratch);
  tmp.c.ws_bytes = GPTQ_NOALLOC_SCRATCH_BYTES;
  tmp.c.owns_ws = false;
  tmp.c.status = reinterpret_cast<gptq::DeviceStatus*>(scratch);
  // the status word must start at zero; the rest of the scratch is written before it is read
  if (cudaMemsetAsync(scratch, 0, gptq::kStatusBytes, tmp.c.stream) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  rc = gptq_quantize_layer(&tmp, W, w_dtype, m, d, R, perm, dead, bits, group, block, grid_given,
                           scales, zeros, codes, W_hat, col_loss);
  if (rc == GPTQ_ERR_NOMEM) return GPTQ_ERR_ARG;  // layer needs more than the fixed scratch
  if (rc) return rc;
  return gptq_sync_status(&tmp);
}
