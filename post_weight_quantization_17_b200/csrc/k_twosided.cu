// Two-sided GPTQ rounding (GPTQ-2D), "GPTQ-2D：把一个"四次方"难题压回"三次方"的故事": round X [m, n]
// to integers Z for the metric ||A (Z - X) B||^2 given R_A, R_B upper triangular with
// R_A^T R_A = (A^T A)^{-1} and R_B^T R_B = (B B^T)^{-1}.
//
// The buffered row / column push of the page (its Algorithm 3), over anti-diagonal wavefronts
// (its Theorem 1: the cells of one anti-diagonal do not depend on one another).  Rounding (i, j):
//   z = rint(y), η = (y - z) / (R_A[i, i] R_B[j, j]);
//   (a) C[p, j] += η R_A[i, p]           for p >= i   (fold into the buffer, down the column)
//   (b) Y[p, j] -= η R_A[i, p] R_B[j, j] for p >  i   (push down the column)
//   (c) Y[i, q] -= C[i, j] R_B[j, q]     for q >  j   (push the buffer along the row)
// The cells of one anti-diagonal own distinct columns for (a), (b) and distinct rows for (c), so
// a diagonal is two launches: k_twosided_col (round, (a), (b)), then k_twosided_row ((c)); the
// second reads C[i, j] only after every contribution to it (rows <= i of column j) has landed.
// One CTA per cell; Y and C are fp32 [m, n] row-major in the workspace.
#include "kernels.h"

#include <algorithm>

namespace gptq {

constexpr int TS_THREADS = 256;

__global__ void k_twosided_init(const float* __restrict__ X, long long mn, float* __restrict__ Y,
                                float* __restrict__ C) {
  pdl_wait();
  pdl_release();
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= mn) return;
  Y[e] = X[e];
  C[e] = 0.f;
}

// Cells (i, s - i) for i = i0 + blockIdx.x.
__global__ void __launch_bounds__(TS_THREADS)
    k_twosided_col(int m, int n, int s, int i0, const float* __restrict__ RA,
                   const float* __restrict__ RB, float* __restrict__ Y, float* __restrict__ C,
                   float* __restrict__ Z, float* __restrict__ eta) {
  pdl_wait();
  pdl_release();
  const int i = i0 + blockIdx.x, j = s - i;
  __shared__ float e_sh;
  if (threadIdx.x == 0) {
    const float y = Y[(long long)i * n + j];
    const float z = rintf(y);
    const float e = __fdiv_rn(y - z, __fmul_rn(RA[(long long)i * m + i], RB[(long long)j * n + j]));
    Z[(long long)i * n + j] = z;
    eta[(long long)i * n + j] = e;
    e_sh = e;
  }
  __syncthreads();
  const float e = e_sh;
  const float eb = e * RB[(long long)j * n + j];
  const float* ra = RA + (long long)i * m;
  for (int p = i + threadIdx.x; p < m; p += TS_THREADS) {
    const float r = ra[p];
    C[(long long)p * n + j] = fmaf(e, r, C[(long long)p * n + j]);
    if (p > i) Y[(long long)p * n + j] = fmaf(-eb, r, Y[(long long)p * n + j]);
  }
}

__global__ void __launch_bounds__(TS_THREADS)
    k_twosided_row(int m, int n, int s, int i0, const float* __restrict__ RB,
                   float* __restrict__ Y, const float* __restrict__ C) {
  pdl_wait();
  pdl_release();
  const int i = i0 + blockIdx.x, j = s - i;
  const float c = C[(long long)i * n + j];
  const float* rb = RB + (long long)j * n;
  float* yrow = Y + (long long)i * n;
  for (int q = j + 1 + threadIdx.x; q < n; q += TS_THREADS) yrow[q] = fmaf(-c, rb[q], yrow[q]);
}

int twosided_round(Ctx* c, const float* X, int m, int n, const float* RA, const float* RB,
                   float* Z, float* eta, float* Y, float* C) {
  const long long mn = (long long)m * n;
  GPTQ_LAUNCH(c, k_twosided_init, (int)((mn + 255) / 256), 256, 0, X, mn, Y, C);
  for (int s = 0; s < m + n - 1; ++s) {
    const int i0 = std::max(0, s - n + 1), i1 = std::min(s, m - 1);
    const int cells = i1 - i0 + 1;
    GPTQ_LAUNCH(c, k_twosided_col, cells, TS_THREADS, 0, m, n, s, i0, RA, RB, Y, C, Z, eta);
    GPTQ_LAUNCH(c, k_twosided_row, cells, TS_THREADS, 0, m, n, s, i0, RB, Y, (const float*)C);
  }
  return GPTQ_OK;
}

}  // namespace gptq
