// a1: Hessian statistic S += Xc^T Xc over one token chunk ([T] eq.(9); accumulated in batches,
// [T] §9.4).  This translation unit holds the CUDA-core path (fp32 inputs, and any input when
// the tensor-core path does not apply); only tiles touching the lower triangle are computed.
#include "kernels.h"
#include "gemm_simt.cuh"

namespace gptq {

int syrk_tc(Ctx* c, const void* X, int dtype, long long n, int d, float* S, bool overwrite);

int syrk_simt(Ctx* c, const void* X, int dtype, long long n, int d, float* S, bool overwrite) {
  GemmArgs g{d, d, (int)n, X, 1, d, X, d, 1, S, d, 1.f, overwrite ? 0.f : 1.f, kCLower};
  if (dtype == GPTQ_BF16) return gemm_simt<__nv_bfloat16, __nv_bfloat16>(c, g);
  if (dtype == GPTQ_F16) return gemm_simt<__half, __half>(c, g);
  return gemm_simt<float, float>(c, g);
}

int syrk_accumulate(Ctx* c, const void* X, int dtype, long long n, int d, float* S,
                    bool overwrite) {
  return syrk_simt(c, X, dtype, n, d, S, overwrite);
}

}  // namespace gptq
