// Two-sided GPTQ rounding (GPTQ-2D), "GPTQ-2D：把一个"四次方"难题压回"三次方"的故事": round X [m, n]
// to integers Z for the metric ||A (Z - X) B||^2 given R_A, R_B upper triangular with
// R_A^T R_A = (A^T A)^{-1} and R_B^T R_B = (B B^T)^{-1}.
//
// The page's buffered row / column push (its Algorithm 3) on cells, rounding (i, j) as
//   z = rint(y), η = (y - z) / (R_A[i, i] R_B[j, j]);
//   (a) C[p, j] += η R_A[i, p]           for p >= i   (fold into the buffer, down the column)
//   (b) Y[p, j] -= η R_A[i, p] R_B[j, j] for p >  i   (push down the column)
//   (c) Y[i, q] -= C[i, j] R_B[j, q]     for q >  j   (push the buffer along the row)
// organised as a wavefront of 64 x 64 tiles (the page's lazy idea, on tiles).  Tiles of one
// tile-anti-diagonal are independent (its Theorem 1 on tiles) and run as one CTA each
// (k_twosided_tile): the tile's Y, C and the diagonal blocks of R_A and R_B in shared memory, the
// cells in anti-diagonal order inside the tile with (a)-(c) restricted to the tile.  After a
// tile-diagonal, every finished tile (I, J) sends the rest of its effect with GEMMs:
//   U = R_A[I, rows below]^T η_IJ:  C[below, J] += U  and  Y[below, J] -= U diag(R_B)   (a), (b)
//   Y[I, columns right] -= C[I, J] R_B[J, columns right]                              (c)
// (the second from η_IJ diag(R_B), which the tile kernel writes beside η).  All launches share one
// stream, so the column updates of one tile-diagonal land before its row updates.
#include "kernels.h"
#include "gemm_simt.cuh"

#include <algorithm>

namespace gptq {

constexpr int TS_TILE = 64;
constexpr int TS_LD = TS_TILE + 1;  // odd stride: column walks hit distinct banks
constexpr int TS_THREADS = 256;
constexpr int TS_SMEM = 4 * TS_TILE * TS_LD * 4;

__global__ void k_twosided_init(const float* __restrict__ X, long long mn, float* __restrict__ Y,
                                float* __restrict__ C) {
  pdl_wait();
  pdl_release();
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= mn) return;
  Y[e] = X[e];
  C[e] = 0.f;
}

// RAT = R_A^T (m x m), so that the column GEMMs read their A operand K-contiguous.
__global__ void k_twosided_transpose(const float* __restrict__ R, int k, float* __restrict__ RT) {
  pdl_wait();
  pdl_release();
  __shared__ float t[32][33];
  const int x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int y = y0 + r, x = x0 + threadIdx.x;
    t[r][threadIdx.x] = (y < k && x < k) ? R[(long long)y * k + x] : 0.f;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int y = x0 + r, x = y0 + threadIdx.x;
    if (y < k && x < k) RT[(long long)y * k + x] = t[threadIdx.x][r];
  }
}

// Tile (I, J) = (I0 + blockIdx.x, t - I) of tile-anti-diagonal t.
__global__ void __launch_bounds__(TS_THREADS)
    k_twosided_tile(int m, int n, int t, int I0, const float* __restrict__ RA,
                    const float* __restrict__ RB, float* __restrict__ Y, float* __restrict__ C,
                    float* __restrict__ Z, float* __restrict__ eta, float* __restrict__ etas) {
  pdl_wait();
  pdl_release();
  extern __shared__ float tsm[];
  float(*Ys)[TS_LD] = reinterpret_cast<float(*)[TS_LD]>(tsm);
  float(*Cs)[TS_LD] = reinterpret_cast<float(*)[TS_LD]>(tsm + TS_TILE * TS_LD);
  float(*RAs)[TS_LD] = reinterpret_cast<float(*)[TS_LD]>(tsm + 2 * TS_TILE * TS_LD);
  float(*RBs)[TS_LD] = reinterpret_cast<float(*)[TS_LD]>(tsm + 3 * TS_TILE * TS_LD);
  const int I = I0 + blockIdx.x, J = t - I;
  const int r0 = I * TS_TILE, c0 = J * TS_TILE;
  const int R = min(TS_TILE, m - r0), Cn = min(TS_TILE, n - c0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < TS_TILE * TS_TILE; e += TS_THREADS) {
    const int a = e / TS_TILE, b = e % TS_TILE;
    const bool in = a < R && b < Cn;
    Ys[a][b] = in ? Y[(long long)(r0 + a) * n + c0 + b] : 0.f;
    Cs[a][b] = in ? C[(long long)(r0 + a) * n + c0 + b] : 0.f;
    RAs[a][b] = (a < R && b < R) ? RA[(long long)(r0 + a) * m + r0 + b] : 0.f;
    RBs[a][b] = (a < Cn && b < Cn) ? RB[(long long)(c0 + a) * n + c0 + b] : 0.f;
  }
  __syncthreads();
  for (int s = 0; s < R + Cn - 1; ++s) {
    const int a_lo = max(0, s - Cn + 1), a_hi = min(s, R - 1);
    // round, fold and push down: one warp per cell; the cells own distinct columns
    for (int a = a_lo + warp; a <= a_hi; a += TS_THREADS / 32) {
      const int b = s - a;
      const float y = Ys[a][b];
      const float z = rintf(y);
      const float rbb = RBs[b][b];
      const float e = __fdiv_rn(y - z, __fmul_rn(RAs[a][a], rbb));
      const float eb = e * rbb;
      if (lane == 0) {
        const long long g = (long long)(r0 + a) * n + c0 + b;
        Z[g] = z;
        eta[g] = e;
        etas[g] = eb;
      }
      for (int a2 = a + lane; a2 < R; a2 += 32) {
        const float r = RAs[a][a2];
        Cs[a2][b] = fmaf(e, r, Cs[a2][b]);
        if (a2 > a) Ys[a2][b] = fmaf(-eb, r, Ys[a2][b]);
      }
    }
    __syncthreads();
    // push the buffer along the rows: the cells own distinct rows
    for (int a = a_lo + warp; a <= a_hi; a += TS_THREADS / 32) {
      const int b = s - a;
      const float cv = Cs[a][b];
      for (int b2 = b + 1 + lane; b2 < Cn; b2 += 32) Ys[a][b2] = fmaf(-cv, RBs[b][b2], Ys[a][b2]);
    }
    __syncthreads();
  }
  for (int e = tid; e < TS_TILE * TS_TILE; e += TS_THREADS) {
    const int a = e / TS_TILE, b = e % TS_TILE;
    if (a < R && b < Cn) C[(long long)(r0 + a) * n + c0 + b] = Cs[a][b];
  }
}

int twosided_round(Ctx* c, const float* X, int m, int n, const float* RA, const float* RB,
                   float* Z, float* eta, float* Y, float* C, float* etas, float* RAT) {
  const long long mn = (long long)m * n;
  GPTQ_LAUNCH(c, k_twosided_init, (int)((mn + 255) / 256), 256, 0, X, mn, Y, C);
  GPTQ_LAUNCH(c, k_twosided_transpose, dim3((m + 31) / 32, (m + 31) / 32), dim3(32, 8), 0, RA, m,
              RAT);
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_twosided_tile,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, TS_SMEM));
  const int TI = (m + TS_TILE - 1) / TS_TILE, TJ = (n + TS_TILE - 1) / TS_TILE;
  for (int t = 0; t < TI + TJ - 1; ++t) {
    const int I0 = std::max(0, t - TJ + 1), I1 = std::min(t, TI - 1);
    GPTQ_LAUNCH(c, k_twosided_tile, I1 - I0 + 1, TS_THREADS, TS_SMEM, m, n, t, I0, RA, RB, Y, C,
                Z, eta, etas);
    int rc;
    for (int I = I0; I <= I1; ++I) {  // (a) and (b) for the rows below each finished tile
      const int J = t - I;
      const int r0 = I * TS_TILE, r1 = std::min(m, r0 + TS_TILE);
      const int c0 = J * TS_TILE, c1 = std::min(n, c0 + TS_TILE);
      if (r1 >= m) continue;
      GemmArgs g{};
      g.M = m - r1; g.N = c1 - c0; g.K = r1 - r0;
      g.A = RAT + (long long)r1 * m + r0; g.sai = m; g.sak = 1;
      g.B = eta + (long long)r0 * n + c0; g.sbk = n; g.sbj = 1;
      g.C = C + (long long)r1 * n + c0; g.ldc = n;
      g.alpha = 1.f; g.beta = 1.f; g.flags = 0;
      if ((rc = gemm_f32(c, g))) return rc;
      g.B = etas + (long long)r0 * n + c0;
      g.C = Y + (long long)r1 * n + c0;
      g.alpha = -1.f;
      if ((rc = gemm_f32(c, g))) return rc;
    }
    for (int I = I0; I <= I1; ++I) {  // (c) for the columns right of each finished tile
      const int J = t - I;
      const int r0 = I * TS_TILE, r1 = std::min(m, r0 + TS_TILE);
      const int c0 = J * TS_TILE, c1 = std::min(n, c0 + TS_TILE);
      if (c1 >= n) continue;
      GemmArgs g{};
      g.M = r1 - r0; g.N = n - c1; g.K = c1 - c0;
      g.A = C + (long long)r0 * n + c0; g.sai = n; g.sak = 1;
      g.B = RB + (long long)c0 * n + c1; g.sbk = n; g.sbj = 1;
      g.C = Y + (long long)r0 * n + c1; g.ldc = n;
      g.alpha = -1.f; g.beta = 1.f; g.flags = 0;
      if ((rc = gemm_f32(c, g))) return rc;
    }
  }
  return GPTQ_OK;
}

}  // namespace gptq
