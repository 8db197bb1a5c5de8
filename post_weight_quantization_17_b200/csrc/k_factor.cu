// a3: damped inverse Hessian in upper-Cholesky form.
//
// [T] §9.1 eq.(37)-(40): GPTQ needs the upper factor R with R^T R = H_λ^{-1}.  Route used
// here: H_λ = U U^T with U upper ("reverse" Cholesky, eliminating from the last index), then
// R = U^{-1}.  R is upper with a positive diagonal and R^T R = U^{-T} U^{-1} = (U U^T)^{-1},
// so by uniqueness of the Cholesky factor it is the same R as the pages' route (Cholesky of
// H_λ, its inverse, then the upper Cholesky factor of that inverse), at half the work.
//
// Both factors are computed together by recursion on a 2x2 block split
//   H_λ = [[A, B], [B^T, C]],  U = [[U11, U12], [0, U22]],  R = [[R11, R12], [0, R22]]:
//   C = U22 U22^T            -> (U22, R22) by recursion, only R22 kept
//   U12 = B R22^T            (from B = U12 U22^T)
//   A - U12 U12^T = U11 U11^T -> (U11, R11) by recursion
//   R12 = -R11 U12 R22
// All off-diagonal work is GEMM (fp32, CUDA cores); blocks of <= 128 are factored and
// inverted inside one CTA.  A non-positive or non-finite pivot raises GPTQ_ERR_NOT_PD /
// GPTQ_ERR_NONFINITE in the device status word (the host retries with more damping).
#include "kernels.h"
#include "gemm_simt.cuh"

namespace gptq {

constexpr int FB = 128;
constexpr int FB_THREADS = 256;                        // 16 x 16 threads, 8 x 8 elements each
constexpr int FB_SMEM = FB * (FB + 1) * 4;

template <int N>
__device__ __forceinline__ float pick(const float (&v)[N], int k) {
  float r = v[0];
#pragma unroll
  for (int t = 1; t < N; ++t) r = (k == t) ? v[t] : r;
  return r;
}

// Factor + invert the diagonal block M[s:s+n, s:s+n] (upper triangle read), n <= FB.
// Writes R = U^{-1} into the upper triangle and zeros below it.  Thread (ty, tx) holds rows
// 8 ty .. 8 ty + 7 and columns 8 tx .. 8 tx + 7 of the symmetric block in registers.
__global__ void __launch_bounds__(FB_THREADS) k_factor_base(float* __restrict__ M, long long ld,
                                                             int s, int n, DeviceStatus* st) {
  extern __shared__ float fsm[];
  float(*U)[FB + 1] = reinterpret_cast<float(*)[FB + 1]>(fsm);
  __shared__ float ucol[FB];
  __shared__ float s_piv;
  __shared__ int bad;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  if (tid == 0) bad = 0;
  float a[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = 8 * ty + r, k = 8 * tx + c;
      float v = 0.f;
      if (i < n && k < n) v = M[(long long)(s + min(i, k)) * ld + s + max(i, k)];
      a[r][c] = v;
    }
  // reverse Cholesky H = U U^T, eliminating from the last index; U's column j goes to U[:, j]
  for (int j = n - 1; j >= 0; --j) {
    const int jb = j >> 3, jr = j & 7;
    if (ty == jb && tx == jb) {
      float dg[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) dg[t] = a[t][t];
      s_piv = pick(dg, jr);
    }
    __syncthreads();
    float piv = s_piv;
    const bool good = (piv > 0.f) && isfinite(piv);
    if (!good) {
      if (tid == 0 && bad == 0) bad = isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE;
      piv = 1.f;
    }
    const float dj = sqrtf(piv);
    if (tx == jb) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = 8 * ty + r;
        if (i < j) {
          const float v = pick(a[r], jr) / dj;
          ucol[i] = v;
          U[i][j] = v;
        }
      }
    }
    if (tid == 0) U[j][j] = dj;
    __syncthreads();
    if (8 * ty < j && 8 * tx < j) {
      float ur[8], uc[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        ur[r] = ucol[8 * ty + r];
        uc[r] = ucol[8 * tx + r];
      }
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (8 * ty + r < j && 8 * tx + c < j) a[r][c] = fmaf(-ur[r], uc[c], a[r][c]);
    }
  }
  __syncthreads();
  // R = U^{-1} (upper), in place in U, row by row from the bottom:
  // R[i][c] = -(sum_{l=i+1..c} U[i][l] R[l][c]) / U[i][i].  2 threads per column c.
  const int c = tid >> 1, part = tid & 1;
  for (int i = n - 1; i >= 0; --i) {
    const float uii = U[i][i];
    float acc0 = 0.f, acc1 = 0.f;
    if (c > i && c < n) {
      int l = i + 1 + part;
      for (; l + 2 <= c; l += 4) {
        acc0 = fmaf(U[i][l], U[l][c], acc0);
        acc1 = fmaf(U[i][l + 2], U[l + 2][c], acc1);
      }
      if (l <= c) acc0 = fmaf(U[i][l], U[l][c], acc0);
    }
    float acc = acc0 + acc1;
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    __syncthreads();
    if (part == 0 && c < n && c >= i) U[i][c] = (c == i) ? 1.f / uii : -acc / uii;
    __syncthreads();
  }
  for (int e = tid; e < n * n; e += FB_THREADS) {
    const int i = e / n, k = e - i * n;
    M[(long long)(s + i) * ld + s + k] = (k >= i) ? U[i][k] : 0.f;
  }
  if (tid == 0 && bad) raise_error(st, bad, s);
}

__global__ void k_copy2d(const float* __restrict__ src, long long lds, float* __restrict__ dst,
                         long long ldd, int rows, int cols) {
  long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  long long total = (long long)rows * cols;
  for (; e < total; e += (long long)gridDim.x * blockDim.x) {
    int r = (int)(e / cols), k = (int)(e % cols);
    dst[(long long)r * ldd + k] = src ? src[(long long)r * lds + k] : 0.f;
  }
}

static int copy2d(Ctx* c, const float* src, long long lds, float* dst, long long ldd, int rows,
                  int cols) {
  long long total = (long long)rows * cols;
  if (total <= 0) return GPTQ_OK;
  int blocks = (int)std::min<long long>((total + 255) / 256, (long long)c->num_sms * 16);
  k_copy2d<<<blocks, 256, 0, c->stream>>>(src, lds, dst, ldd, rows, cols);
  GPTQ_LAUNCH_CHECK(c);
  return GPTQ_OK;
}

size_t factor_tmp_floats(int d) {
  size_t h = (size_t)d / 2 + FB;
  return h * h;
}

static int rec(Ctx* c, float* M, long long ld, int s, int e, float* tmp) {
  const int n = e - s;
  if (n <= FB) {
    k_factor_base<<<1, FB_THREADS, FB_SMEM, c->stream>>>(M, ld, s, n, c->status);
    GPTQ_LAUNCH_CHECK(c);
    return GPTQ_OK;
  }
  int n1 = ((n / 2 + FB - 1) / FB) * FB;
  if (n1 >= n) n1 = n - FB;
  const int mid = s + n1, n2 = e - mid;
  int rc = rec(c, M, ld, mid, e, tmp);
  if (rc) return rc;
  float* Bblk = M + (long long)s * ld + mid;       // rows s..mid, cols mid..e
  float* R22 = M + (long long)mid * ld + mid;
  float* Ablk = M + (long long)s * ld + s;
  // U12 = B R22^T  (opB(k,j) = R22[j][k], zero for k < j)
  GemmArgs g{n1, n2, n2, Bblk, ld, 1, R22, 1, ld, tmp, n2, 1.f, 0.f, kBLower};
  if ((rc = gemm_simt(c, g))) return rc;
  if ((rc = copy2d(c, tmp, n2, Bblk, ld, n1, n2))) return rc;
  // A' = A - U12 U12^T  (upper tiles only)
  GemmArgs g2{n1, n1, n2, tmp, n2, 1, tmp, 1, n2, Ablk, ld, -1.f, 1.f, kCUpper};
  if ((rc = gemm_simt(c, g2))) return rc;
  if ((rc = rec(c, M, ld, s, mid, tmp))) return rc;
  // T2 = U12 R22  (R22(k,j) = 0 for k > j)
  GemmArgs g3{n1, n2, n2, Bblk, ld, 1, R22, ld, 1, tmp, n2, 1.f, 0.f, kBUpper};
  if ((rc = gemm_simt(c, g3))) return rc;
  // R12 = -R11 T2  (R11(i,k) = 0 for k < i)
  GemmArgs g4{n1, n2, n1, Ablk, ld, 1, tmp, n2, 1, Bblk, ld, -1.f, 0.f, kAUpper};
  if ((rc = gemm_simt(c, g4))) return rc;
  // strict lower block of this level
  return copy2d(c, nullptr, 0, M + (long long)mid * ld + s, ld, n2, n1);
}

int factor_inverse(Ctx* c, float* M, int d, float* tmp) {
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_factor_base,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, FB_SMEM));
  return rec(c, M, d, 0, d, tmp);
}

}  // namespace gptq
