// CUDA-core fp32 GEMM with general strides, used where the arithmetic must stay fp32-exact
// per product (factorization recursion, fp32 Hessian, first trailing update):
//   C[i, j] = alpha * sum_k opA(i, k) opB(k, j) + beta * C[i, j]
//   opA(i, k) = A[i * sai + k * sak], opB(k, j) = B[k * sbk + j * sbj]
// Tiles of 128 x 128 x 8, 256 threads, 8 x 8 outputs per thread, register prefetch of the
// next k-slab.  Structure flags skip work that is known to be zero:
//   kAUpper: opA(i,k) = 0 for k < i      kALower: opA(i,k) = 0 for k > i
//   kBUpper: opB(k,j) = 0 for k > j      kBLower: opB(k,j) = 0 for k < j
//   kCUpper: only tiles touching i <= j are computed   kCLower: only tiles touching i >= j
#pragma once
#include "common.cuh"

namespace gptq {

enum : int {
  kAUpper = 1, kALower = 2, kBUpper = 4, kBLower = 8, kCUpper = 16, kCLower = 32
};

struct GemmArgs {
  int M, N, K;
  const void* A; long long sai, sak;
  const void* B; long long sbk, sbj;
  float* C; long long ldc;
  float alpha, beta;
  int flags;
};

constexpr int GBM = 128, GBN = 128, GBK = 8, GTHREADS = 256;

template <class TA, class TB>
__global__ void __launch_bounds__(GTHREADS) k_gemm_simt(GemmArgs g) {
  __shared__ __align__(16) float As[2][GBK][GBM + 4];
  __shared__ __align__(16) float Bs[2][GBK][GBN + 4];
  const int tid = threadIdx.x;
  const int i0 = blockIdx.y * GBM, j0 = blockIdx.x * GBN;
  if ((g.flags & kCUpper) && i0 > j0 + GBN - 1) return;
  if ((g.flags & kCLower) && j0 > i0 + GBM - 1) return;
  int kbeg = 0, kend = g.K;
  if (g.flags & kAUpper) kbeg = max(kbeg, i0);
  if (g.flags & kBLower) kbeg = max(kbeg, j0);
  if (g.flags & kALower) kend = min(kend, i0 + GBM);
  if (g.flags & kBUpper) kend = min(kend, j0 + GBN);
  kbeg = kbeg / GBK * GBK;

  const TA* A = reinterpret_cast<const TA*>(g.A);
  const TB* B = reinterpret_cast<const TB*>(g.B);
  // loader mapping: 1024 elements per operand slab, 4 per thread; consecutive threads walk the
  // unit-stride dimension so that global reads coalesce.
  const bool a_kcontig = (g.sak == 1);
  const bool b_ncontig = (g.sbj == 1);
  float ra[4], rb[4];
  auto load_slab = [&](int k0) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int e = tid + r * GTHREADS;
      int ii, kk;
      if (a_kcontig) { ii = e >> 3; kk = e & 7; } else { kk = e >> 7; ii = e & 127; }
      int gi = i0 + ii, gk = k0 + kk;
      ra[r] = (gi < g.M && gk < kend && gk >= kbeg) ? to_f32<TA>(A[(long long)gi * g.sai + (long long)gk * g.sak]) : 0.f;
      int jj, kb;
      if (b_ncontig) { kb = e >> 7; jj = e & 127; } else { jj = e >> 3; kb = e & 7; }
      int gj = j0 + jj, gkb = k0 + kb;
      rb[r] = (gj < g.N && gkb < kend && gkb >= kbeg) ? to_f32<TB>(B[(long long)gkb * g.sbk + (long long)gj * g.sbj]) : 0.f;
    }
  };
  auto store_slab = [&](int buf) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int e = tid + r * GTHREADS;
      int ii, kk;
      if (a_kcontig) { ii = e >> 3; kk = e & 7; } else { kk = e >> 7; ii = e & 127; }
      As[buf][kk][ii] = ra[r];
      int jj, kb;
      if (b_ncontig) { kb = e >> 7; jj = e & 127; } else { jj = e >> 3; kb = e & 7; }
      Bs[buf][kb][jj] = rb[r];
    }
  };

  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

  if (kbeg < kend) {
    load_slab(kbeg);
    store_slab(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = kbeg; k0 < kend; k0 += GBK) {
      const bool more = k0 + GBK < kend;
      if (more) load_slab(k0 + GBK);
#pragma unroll
      for (int kk = 0; kk < GBK; ++kk) {
        float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
        float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
        float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
        float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
        float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
      }
      if (more) {
        store_slab(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    int gi = i0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + a - 4);
    if (gi >= g.M) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      int gj = j0 + (b < 4 ? tx * 4 + b : 64 + tx * 4 + b - 4);
      if (gj >= g.N) continue;
      float* c = g.C + (long long)gi * g.ldc + gj;
      float v = g.alpha * acc[a][b];
      *c = (g.beta == 0.f) ? v : fmaf(g.beta, *c, v);
    }
  }
}

template <class TA = float, class TB = float>
inline int gemm_simt(Ctx* c, const GemmArgs& g) {
  if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
  dim3 grid((g.N + GBN - 1) / GBN, (g.M + GBM - 1) / GBM);
  k_gemm_simt<TA, TB><<<grid, GTHREADS, 0, c->stream>>>(g);
  GPTQ_LAUNCH_CHECK(c);
  return GPTQ_OK;
}

}  // namespace gptq
