// CUDA-core fp32 GEMM with general strides, used where the arithmetic must stay fp32-exact
// per product (factorization recursion, fp32 Hessian, first trailing update):
//   C[i, j] = alpha * sum_k opA(i, k) opB(k, j) + beta * C[i, j]
//   opA(i, k) = A[i * sai + k * sak], opB(k, j) = B[k * sbk + j * sbj]
// Tiles of 128 x 128 (8 x 8 outputs per thread) or 64 x 64 (4 x 4), k-slabs of 8, 256 threads,
// register prefetch of the next k-slab.  Structure flags skip work that is known to be zero:
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
  int partial_k;  // tensor path: k-elements per TMEM partial (multiple of 32; 0: 128)
};

constexpr int GBK = 8, GTHREADS = 256;

// BM x BN tile, 16 x 16 threads, each computing (BM/16) x (BN/16) outputs split into groups of
// 4 rows / 4 columns spaced BM/2 (BN/2) apart, so that the shared-memory reads are float4s.
template <class TA, class TB, int BM, int BN>
__global__ void __launch_bounds__(GTHREADS) k_gemm_simt(GemmArgs g) {
  pdl_wait();
  pdl_release();
  constexpr int TM = BM / 16, TN = BN / 16;          // 8 or 4
  constexpr int LA = BM * GBK / GTHREADS, LB = BN * GBK / GTHREADS;
  __shared__ __align__(16) float As[2][GBK][BM + 4];
  __shared__ __align__(16) float Bs[2][GBK][BN + 4];
  const int tid = threadIdx.x;
  const int i0 = blockIdx.y * BM, j0 = blockIdx.x * BN;
  if ((g.flags & kCUpper) && i0 > j0 + BN - 1) return;
  if ((g.flags & kCLower) && j0 > i0 + BM - 1) return;
  int kbeg = 0, kend = g.K;
  if (g.flags & kAUpper) kbeg = max(kbeg, i0);
  if (g.flags & kBLower) kbeg = max(kbeg, j0);
  if (g.flags & kALower) kend = min(kend, i0 + BM);
  if (g.flags & kBUpper) kend = min(kend, j0 + BN);
  kbeg = kbeg / GBK * GBK;

  const TA* A = reinterpret_cast<const TA*>(g.A);
  const TB* B = reinterpret_cast<const TB*>(g.B);
  // loader mapping: consecutive threads walk the unit-stride dimension so reads coalesce
  const bool a_kcontig = (g.sak == 1);
  const bool b_ncontig = (g.sbj == 1);
  float ra[LA], rb[LB];
  auto a_idx = [&](int e, int& ii, int& kk) {
    if (a_kcontig) { ii = e / GBK; kk = e % GBK; } else { kk = e / BM; ii = e % BM; }
  };
  auto b_idx = [&](int e, int& jj, int& kb) {
    if (b_ncontig) { kb = e / BN; jj = e % BN; } else { jj = e / GBK; kb = e % GBK; }
  };
  auto load_slab = [&](int k0) {
#pragma unroll
    for (int r = 0; r < LA; ++r) {
      int ii, kk;
      a_idx(tid + r * GTHREADS, ii, kk);
      const int gi = i0 + ii, gk = k0 + kk;
      ra[r] = (gi < g.M && gk < kend && gk >= kbeg)
                  ? to_f32<TA>(A[(long long)gi * g.sai + (long long)gk * g.sak]) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < LB; ++r) {
      int jj, kb;
      b_idx(tid + r * GTHREADS, jj, kb);
      const int gj = j0 + jj, gkb = k0 + kb;
      rb[r] = (gj < g.N && gkb < kend && gkb >= kbeg)
                  ? to_f32<TB>(B[(long long)gkb * g.sbk + (long long)gj * g.sbj]) : 0.f;
    }
  };
  auto store_slab = [&](int buf) {
#pragma unroll
    for (int r = 0; r < LA; ++r) {
      int ii, kk;
      a_idx(tid + r * GTHREADS, ii, kk);
      As[buf][kk][ii] = ra[r];
    }
#pragma unroll
    for (int r = 0; r < LB; ++r) {
      int jj, kb;
      b_idx(tid + r * GTHREADS, jj, kb);
      Bs[buf][kb][jj] = rb[r];
    }
  };

  const int tx = tid & 15, ty = tid >> 4;
  float acc[TM][TN];
#pragma unroll
  for (int a = 0; a < TM; ++a)
#pragma unroll
    for (int b = 0; b < TN; ++b) acc[a][b] = 0.f;

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
        float av[TM], bv[TN];
#pragma unroll
        for (int h = 0; h < TM / 4; ++h) {
          const float4 x = *reinterpret_cast<const float4*>(&As[buf][kk][h * (BM / 2) + ty * 4]);
          av[4 * h] = x.x; av[4 * h + 1] = x.y; av[4 * h + 2] = x.z; av[4 * h + 3] = x.w;
        }
#pragma unroll
        for (int h = 0; h < TN / 4; ++h) {
          const float4 x = *reinterpret_cast<const float4*>(&Bs[buf][kk][h * (BN / 2) + tx * 4]);
          bv[4 * h] = x.x; bv[4 * h + 1] = x.y; bv[4 * h + 2] = x.z; bv[4 * h + 3] = x.w;
        }
#pragma unroll
        for (int a = 0; a < TM; ++a)
#pragma unroll
          for (int b = 0; b < TN; ++b) acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
      }
      if (more) {
        store_slab(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }
#pragma unroll
  for (int a = 0; a < TM; ++a) {
    const int gi = i0 + (a / 4) * (BM / 2) + ty * 4 + (a % 4);
    if (gi >= g.M) continue;
#pragma unroll
    for (int b = 0; b < TN; ++b) {
      const int gj = j0 + (b / 4) * (BN / 2) + tx * 4 + (b % 4);
      if (gj >= g.N) continue;
      float* c = g.C + (long long)gi * g.ldc + gj;
      const float v = g.alpha * acc[a][b];
      *c = (g.beta == 0.f) ? v : fmaf(g.beta, *c, v);
    }
  }
}

// Picks 128 x 128 tiles when they fill the GPU, else 64 x 64 tiles.
template <class TA = float, class TB = float>
inline int gemm_simt(Ctx* c, const GemmArgs& g) {
  if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
  const long long big = (long long)((g.N + 127) / 128) * ((g.M + 127) / 128);
  if (big >= 2LL * c->num_sms) {
    dim3 grid((g.N + 127) / 128, (g.M + 127) / 128);
    GPTQ_LAUNCH(c, k_gemm_simt<TA, TB, 128, 128>, grid, GTHREADS, 0, g);
  } else {
    dim3 grid((g.N + 63) / 64, (g.M + 63) / 64);
    GPTQ_LAUNCH(c, k_gemm_simt<TA, TB, 64, 64>, grid, GTHREADS, 0, g);
  }
  return GPTQ_OK;
}

// Small GEMMs (the factorization's two lowest recursion levels: up to 256 on a side) are
// latency bound, so they take 32 x 32 tiles (2 x 2 outputs per thread, 32-deep k-slabs,
// register prefetch of the next slab): many CTAs, no tensor-core setup, fp32 products.  From
// 512 on a side, and for tall products such as the trailing update, the tensor path is as fast
// or faster.
constexpr int SBM = 32, SBK = 32;
constexpr int kSmallGemmSide = 256;

template <class TA, class TB>
__global__ void __launch_bounds__(GTHREADS) k_gemm_small(GemmArgs g) {
  pdl_wait();
  pdl_release();
  constexpr int LA = SBM * SBK / GTHREADS;  // 4 elements of each operand per thread and slab
  __shared__ __align__(16) float As[2][SBK][SBM + 4];  // As[k][i]
  __shared__ __align__(16) float Bs[2][SBK][SBM + 4];  // Bs[k][j]
  const int tid = threadIdx.x;
  const int i0 = blockIdx.y * SBM, j0 = blockIdx.x * SBM;
  if ((g.flags & kCUpper) && i0 > j0 + SBM - 1) return;
  if ((g.flags & kCLower) && j0 > i0 + SBM - 1) return;
  int kbeg = 0, kend = g.K;
  if (g.flags & kAUpper) kbeg = max(kbeg, i0);
  if (g.flags & kBLower) kbeg = max(kbeg, j0);
  if (g.flags & kALower) kend = min(kend, i0 + SBM);
  if (g.flags & kBUpper) kend = min(kend, j0 + SBM);

  const TA* A = reinterpret_cast<const TA*>(g.A);
  const TB* B = reinterpret_cast<const TB*>(g.B);
  const bool a_kcontig = (g.sak == 1);
  const bool b_ncontig = (g.sbj == 1);
  float ra[LA], rb[LA];
  // consecutive threads walk each operand's unit-stride dimension
  auto a_idx = [&](int e, int& ii, int& kk) {
    if (a_kcontig) { ii = e / SBK; kk = e % SBK; } else { kk = e / SBM; ii = e % SBM; }
  };
  auto b_idx = [&](int e, int& jj, int& kb) {
    if (b_ncontig) { kb = e / SBM; jj = e % SBM; } else { jj = e / SBK; kb = e % SBK; }
  };
  auto load_slab = [&](int k0) {
#pragma unroll
    for (int r = 0; r < LA; ++r) {
      int ii, kk, jj, kb;
      a_idx(tid + r * GTHREADS, ii, kk);
      const int gi = i0 + ii, gk = k0 + kk;
      ra[r] = (gi < g.M && gk < kend && gk >= kbeg)
                  ? to_f32<TA>(A[(long long)gi * g.sai + (long long)gk * g.sak]) : 0.f;
      b_idx(tid + r * GTHREADS, jj, kb);
      const int gj = j0 + jj, gkb = k0 + kb;
      rb[r] = (gj < g.N && gkb < kend && gkb >= kbeg)
                  ? to_f32<TB>(B[(long long)gkb * g.sbk + (long long)gj * g.sbj]) : 0.f;
    }
  };
  auto store_slab = [&](int buf) {
#pragma unroll
    for (int r = 0; r < LA; ++r) {
      int ii, kk, jj, kb;
      a_idx(tid + r * GTHREADS, ii, kk);
      As[buf][kk][ii] = ra[r];
      b_idx(tid + r * GTHREADS, jj, kb);
      Bs[buf][kb][jj] = rb[r];
    }
  };
  const int tx = tid & 15, ty = tid >> 4;
  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  kbeg = kbeg / SBK * SBK;
  if (kbeg < kend) {
    load_slab(kbeg);
    store_slab(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = kbeg; k0 < kend; k0 += SBK) {
      const bool more = k0 + SBK < kend;
      if (more) load_slab(k0 + SBK);
#pragma unroll
      for (int kk = 0; kk < SBK; ++kk) {
        const float2 a2 = *reinterpret_cast<const float2*>(&As[buf][kk][2 * ty]);
        const float2 b2 = *reinterpret_cast<const float2*>(&Bs[buf][kk][2 * tx]);
        acc[0][0] = fmaf(a2.x, b2.x, acc[0][0]);
        acc[0][1] = fmaf(a2.x, b2.y, acc[0][1]);
        acc[1][0] = fmaf(a2.y, b2.x, acc[1][0]);
        acc[1][1] = fmaf(a2.y, b2.y, acc[1][1]);
      }
      if (more) {
        store_slab(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int gi = i0 + 2 * ty + a;
    if (gi >= g.M) continue;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int gj = j0 + 2 * tx + b;
      if (gj >= g.N) continue;
      float* c = g.C + (long long)gi * g.ldc + gj;
      const float v = g.alpha * acc[a][b];
      *c = (g.beta == 0.f) ? v : fmaf(g.beta, *c, v);
    }
  }
}

template <class TA = float, class TB = float>
inline int gemm_small(Ctx* c, const GemmArgs& g) {
  if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
  dim3 grid((g.N + SBM - 1) / SBM, (g.M + SBM - 1) / SBM);
  GPTQ_LAUNCH(c, k_gemm_small<TA, TB>, grid, GTHREADS, 0, g);
  return GPTQ_OK;
}

// fp32-accurate GEMM: small ones on CUDA cores (gemm_small), else tcgen05 3xTF32 where TMA can
// take the operands, else CUDA cores (k_gemm_tc.cu).
int gemm_f32(Ctx* c, const GemmArgs& g);

}  // namespace gptq
