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
// All off-diagonal work is fp32-accurate GEMM (tcgen05 3xTF32); blocks of <= 128 are factored and
// inverted inside one CTA.  T2 = U12 R22 needs only the right subtree, so it runs on a second
// stream beside the left subtree's factorization.  A non-positive or non-finite pivot raises GPTQ_ERR_NOT_PD /
// GPTQ_ERR_NONFINITE in the device status word (the host retries with more damping).
#include "kernels.h"
#include "gemm_simt.cuh"

namespace gptq {

constexpr int FB = 128;                 // diagonal block factored inside one CTA
constexpr int FP = 32;                  // panel width (one warp factors a panel's diagonal)
constexpr int FB_THREADS = 256;
// shared memory: A (the block, then U and R), the current panel, the diagonal inverses, T
constexpr int FB_UP = 36;               // padded row of the warp-level panel buffers (16-B rows)
constexpr int FB_LDA = FB + 4;          // padded row of A: 528 bytes, so rows are 16-byte aligned
constexpr int FB_SMEM = (FB * FB_LDA + (FB - FP) * (FP + 1) + (FB / FP) * FP * (FP + 1) +
                         FP * (FB + 1) + 2 * FP * FB_UP) * 4;

// Factor + invert the diagonal block M[s:s+n, s:s+n] (upper triangle read), n <= FB.
// Writes R = U^{-1} into the upper triangle and zeros below it.
//
// Blocked reverse Cholesky over four 32-column panels, last panel first:
//   (a) one warp factors the panel's 32 x 32 diagonal block D = U_PP U_PP^T in registers
//       (lane l holds row l; pivots and columns travel by shuffles) and inverts U_PP;
//   (b) the rows above get their U panel U[0:p0, P] = A[0:p0, P] U_PP^{-T};
//   (c) the rows above are updated, A[0:p0, 0:p0] -= U[0:p0, P] U[0:p0, P]^T.
// Then R block row by block row, from the bottom: R[P, >P] = -R_PP (U[P, >P] R[>P, >P]).
// Indices >= n are padded with the identity, which factors to itself without coupling.
__global__ void __launch_bounds__(FB_THREADS) k_factor_base(float* __restrict__ M, long long ld,
                                                             int s, int n, DeviceStatus* st) {
  extern __shared__ float fsm[];
  float(*A)[FB_LDA] = reinterpret_cast<float(*)[FB_LDA]>(fsm);
  float(*Pn)[FP + 1] = reinterpret_cast<float(*)[FP + 1]>(fsm + FB * FB_LDA);
  float(*Rd)[FP][FP + 1] =
      reinterpret_cast<float(*)[FP][FP + 1]>(fsm + FB * FB_LDA + (FB - FP) * (FP + 1));
  float(*T)[FB + 1] = reinterpret_cast<float(*)[FB + 1]>(
      fsm + FB * FB_LDA + (FB - FP) * (FP + 1) + (FB / FP) * FP * (FP + 1));
  float* fsm_panel = fsm + FB * FB_LDA + (FB - FP) * (FP + 1) + (FB / FP) * FP * (FP + 1) +
                     FP * (FB + 1);
  float(*Uc)[FB_UP] = reinterpret_cast<float(*)[FB_UP]>(fsm_panel);  // Uc[j][l] = U_PP[l][j]
  float(*Ur)[FB_UP] = reinterpret_cast<float(*)[FB_UP]>(fsm_panel + FP * FB_UP);  // rows
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tx = tid & 15, ty = tid >> 4;
  if (tid == 0) bad = 0;
  // asynchronous load of the block's rows (all copies in flight; 16-byte copies when the rows
  // are 16-byte aligned), identity padding beyond n; the lower triangle is then mirrored from
  // the upper one in shared memory
  const bool vec = ((reinterpret_cast<uintptr_t>(M + (long long)s * ld + s) & 15) == 0) &&
                   (ld % 4 == 0) && (n % 4 == 0);
  if (vec) {
    for (int e = tid; e < FB * (FB / 4); e += FB_THREADS) {
      const int i = e >> 5, k4 = (e & 31) * 4;
      if (i < n && k4 < n) {
        const float* src = M + (long long)(s + i) * ld + s + k4;
        const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&A[i][k4]));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) A[i][k4 + t] = (i == k4 + t) ? 1.f : 0.f;
      }
    }
  } else {
    for (int e = tid; e < FB * FB; e += FB_THREADS) {
      const int i = e >> 7, k = e & 127;
      if (i < n && k < n) {
        const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&A[i][k]));
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst),
                     "l"(M + (long long)(s + i) * ld + s + k) : "memory");
      } else {
        A[i][k] = (i == k) ? 1.f : 0.f;
      }
    }
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  for (int e = tid; e < FB * FB; e += FB_THREADS) {
    const int i = e >> 7, k = e & 127;
    if (k < i) A[i][k] = A[k][i];
  }
  __syncthreads();

  for (int P = FB / FP - 1; P >= 0; --P) {
    const int p0 = P * FP;
    if (warp == 0) {
      float dr[FP], u[FP], r[FP];
#pragma unroll
      for (int k = 0; k < FP; ++k) dr[k] = A[p0 + lane][p0 + k];
      // (a) D = U_PP U_PP^T, eliminating from the last index.  Lane l keeps row l of D.  Column
      // jj of U_PP is written to Uc[jj][:] and read back by every lane as float4 broadcasts.
#pragma unroll
      for (int jj = FP - 1; jj >= 0; --jj) {
        float piv = __shfl_sync(0xffffffffu, dr[jj], jj);
        const bool good = (piv > 0.f) && isfinite(piv);
        if (!good) {
          if (lane == 0 && bad == 0) bad = isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE;
          piv = 1.f;
        }
        const float rs = rsqrtf(piv);
        const float uj = (lane < jj) ? dr[jj] * rs : (lane == jj ? piv * rs : 0.f);
        u[jj] = uj;
        Uc[jj][lane] = uj;
        __syncwarp();
#pragma unroll
        for (int k4 = 0; k4 < (jj + 3) / 4; ++k4) {
          const float4 c4 = *reinterpret_cast<const float4*>(&Uc[jj][4 * k4]);
          const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
          for (int t = 0; t < 4; ++t)
            if (4 * k4 + t < jj) dr[4 * k4 + t] = fmaf(-uj, cv[t], dr[4 * k4 + t]);
        }
      }
      // rows of U_PP to Ur (lane l writes row l)
#pragma unroll
      for (int k = 0; k < FP; ++k) Ur[lane][k] = u[k];
      __syncwarp();
      // U_PP^{-1}: lane c computes column c, rows from the bottom.  Rows not yet computed are
      // zero, so each dot product runs over the whole row (float4 broadcasts of U_PP's row i,
      // four partial sums).
#pragma unroll
      for (int k = 0; k < FP; ++k) r[k] = 0.f;
#pragma unroll
      for (int i = FP - 1; i >= 0; --i) {
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k4 = (i + 1) / 4; k4 < FP / 4; ++k4) {
          const float4 u4 = *reinterpret_cast<const float4*>(&Ur[i][4 * k4]);
          const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
          for (int t = 0; t < 4; ++t)
            if (4 * k4 + t > i) part[t] = fmaf(uv[t], r[4 * k4 + t], part[t]);
        }
        const float inv = 1.f / Ur[i][i];
        const float acc = (part[0] + part[1]) + (part[2] + part[3]);
        r[i] = (lane == i) ? inv : (lane > i ? -acc * inv : 0.f);
      }
#pragma unroll
      for (int i = 0; i < FP; ++i) Rd[P][i][lane] = r[i];
    }
    __syncthreads();
    if (p0 > 0) {
      // (b) U panel of the rows above: Pn[i][c] = sum_k A[i][p0 + k] Rd[c][k] (Rd upper, its
      //     lower part stored as zeros).  Thread (ty, tx): rows ty + 16 a, columns tx, tx + 16.
      const int na = p0 / 16;
      {
        float acc[6][2];
#pragma unroll
        for (int a = 0; a < 6; ++a) acc[a][0] = acc[a][1] = 0.f;
#pragma unroll 4
        for (int k = 0; k < FP; ++k) {
          const float r0 = Rd[P][tx][k], r1 = Rd[P][tx + 16][k];
#pragma unroll
          for (int a = 0; a < 6; ++a)
            if (a < na) {
              const float x = A[ty + 16 * a][p0 + k];
              acc[a][0] = fmaf(x, r0, acc[a][0]);
              acc[a][1] = fmaf(x, r1, acc[a][1]);
            }
        }
#pragma unroll
        for (int a = 0; a < 6; ++a)
          if (a < na) {
            Pn[ty + 16 * a][tx] = acc[a][0];
            Pn[ty + 16 * a][tx + 16] = acc[a][1];
          }
      }
      __syncthreads();
      for (int e = tid; e < p0 * FP; e += FB_THREADS) {
        const int i = e >> 5, c = e & 31;
        A[i][p0 + c] = Pn[i][c];
      }
      // (c) A[0:p0, 0:p0] -= Pn Pn^T; thread (ty, tx) owns rows ty + 16 a, columns tx + 16 b
      {
        float acc[6][6];
#pragma unroll
        for (int a = 0; a < 6; ++a)
#pragma unroll
          for (int b = 0; b < 6; ++b) acc[a][b] = 0.f;
#pragma unroll 4
        for (int c = 0; c < FP; ++c) {
          float xa[6], xb[6];
#pragma unroll
          for (int a = 0; a < 6; ++a) {
            xa[a] = (a < na) ? Pn[ty + 16 * a][c] : 0.f;
            xb[a] = (a < na) ? Pn[tx + 16 * a][c] : 0.f;
          }
#pragma unroll
          for (int a = 0; a < 6; ++a)
#pragma unroll
            for (int b = 0; b < 6; ++b) acc[a][b] = fmaf(xa[a], xb[b], acc[a][b]);
        }
#pragma unroll
        for (int a = 0; a < 6; ++a)
#pragma unroll
          for (int b = 0; b < 6; ++b)
            if (a < na && b < na) A[ty + 16 * a][tx + 16 * b] -= acc[a][b];
      }
      __syncthreads();
    }
  }
  // R: diagonal blocks from the panel inverses; the strict lower part is zeroed so that the
  // block products below can run over whole, uniform ranges
  for (int e = tid; e < FB * FB; e += FB_THREADS) {
    const int i = e >> 7, k = e & 127;
    const int P = i / FP;
    if (k < i) A[i][k] = 0.f;
    else if (k < (P + 1) * FP) A[i][k] = Rd[P][i - P * FP][k - P * FP];
  }
  __syncthreads();
  // block rows from the bottom: R[P, >P] = -R_PP (U[P, >P] R[>P, >P]).  Thread (ty, tx) owns
  // rows ty, ty + 16 of the block row and columns c0 + tx + 16 b.
  for (int P = FB / FP - 2; P >= 0; --P) {
    const int p0 = P * FP, c0 = p0 + FP, nb = (FB - c0) / 16;
    {
      float acc[2][6];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 6; ++b) acc[a][b] = 0.f;
#pragma unroll 4
      for (int l = c0; l < FB; ++l) {
        const float u0 = A[p0 + ty][l], u1 = A[p0 + ty + 16][l];
#pragma unroll
        for (int b = 0; b < 6; ++b)
          if (b < nb) {
            const float rr = A[l][c0 + tx + 16 * b];
            acc[0][b] = fmaf(u0, rr, acc[0][b]);
            acc[1][b] = fmaf(u1, rr, acc[1][b]);
          }
      }
#pragma unroll
      for (int b = 0; b < 6; ++b)
        if (b < nb) {
          T[ty][c0 + tx + 16 * b] = acc[0][b];
          T[ty + 16][c0 + tx + 16 * b] = acc[1][b];
        }
    }
    __syncthreads();
    {
      float acc[2][6];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 6; ++b) acc[a][b] = 0.f;
#pragma unroll 4
      for (int k = 0; k < FP; ++k) {
        const float r0 = Rd[P][ty][k], r1 = Rd[P][ty + 16][k];
#pragma unroll
        for (int b = 0; b < 6; ++b)
          if (b < nb) {
            const float tt = T[k][c0 + tx + 16 * b];
            acc[0][b] = fmaf(r0, tt, acc[0][b]);
            acc[1][b] = fmaf(r1, tt, acc[1][b]);
          }
      }
#pragma unroll
      for (int b = 0; b < 6; ++b)
        if (b < nb) {
          A[p0 + ty][c0 + tx + 16 * b] = -acc[0][b];
          A[p0 + ty + 16][c0 + tx + 16 * b] = -acc[1][b];
        }
    }
    __syncthreads();
  }
  // write R back by rows (the strict lower part of A is zero by now)
  if (vec) {
    for (int e = tid; e < FB * (FB / 4); e += FB_THREADS) {
      const int i = e >> 5, k4 = (e & 31) * 4;
      if (i < n && k4 < n)
        *reinterpret_cast<float4*>(M + (long long)(s + i) * ld + s + k4) =
            make_float4(A[i][k4], A[i][k4 + 1], A[i][k4 + 2], A[i][k4 + 3]);
    }
  } else {
    for (int e = tid; e < FB * FB; e += FB_THREADS) {
      const int i = e >> 7, k = e & 127;
      if (i < n && k < n) M[(long long)(s + i) * ld + s + k] = A[i][k];
    }
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

// Scratch: for every recursion level, U12 and T2 of that level's node ([n1 x n2] each, with
// n1 <= n/2 + FB and n2 <= n/2 at node size n).
static size_t level_floats(int n) {
  const size_t h = (size_t)n / 2 + FB;
  return h * h;
}

// Size of a node's left child: ceil(n/2) rounded up to whole blocks, so it is the larger child
// (the right one has n - larger_child(n) <= n/2 columns) and smaller than n for n > FB.
static int larger_child(int n) { return (((n + 1) / 2 + FB - 1) / FB) * FB; }

size_t factor_tmp_floats(int d) {
  size_t total = 0;
  for (int n = d; n > FB; n = larger_child(n)) total += 2 * level_floats(n);
  return total + 64;
}

struct FactorRun {
  Ctx* c;
  float* M;
  long long ld;
  float* tmp;              // level buffers, consecutive
  cudaStream_t side;       // T2 = U12 R22 runs here, beside the left subtree
  cudaEvent_t ev[2 * 64];  // per level: U12 ready, T2 ready
};

static int rec(FactorRun& f, int s, int e, int level, float* buf) {
  Ctx* c = f.c;
  const long long ld = f.ld;
  float* M = f.M;
  const int n = e - s;
  if (n <= FB) {
    k_factor_base<<<1, FB_THREADS, FB_SMEM, c->stream>>>(M, ld, s, n, c->status);
    GPTQ_LAUNCH_CHECK(c);
    return GPTQ_OK;
  }
  const int n1 = larger_child(n);  // < n for n > FB
  const int mid = s + n1, n2 = e - mid;
  float* U12 = buf;                                   // [n1 x n2]
  float* T2 = buf + level_floats(n);                  // [n1 x n2]
  float* next = buf + 2 * level_floats(n);
  int rc = rec(f, mid, e, level + 1, next);
  if (rc) return rc;
  const float* Bblk = M + (long long)s * ld + mid;    // rows s..mid, cols mid..e (H_λ)
  float* Rblk = M + (long long)s * ld + mid;          // becomes R12
  const float* R22 = M + (long long)mid * ld + mid;
  float* Ablk = M + (long long)s * ld + s;
  // U12 = B R22^T  (opB(k,j) = R22[j][k], zero for k < j)
  GemmArgs g{n1, n2, n2, Bblk, ld, 1, R22, 1, ld, U12, n2, 1.f, 0.f, kBLower};
  if ((rc = gemm_f32(c, g))) return rc;
  // A' = A - U12 U12^T  (upper tiles only)
  GemmArgs g2{n1, n1, n2, U12, n2, 1, U12, 1, n2, Ablk, ld, -1.f, 1.f, kCUpper};
  if ((rc = gemm_f32(c, g2))) return rc;
  // T2 = U12 R22 (R22(k,j) = 0 for k > j) on the side stream, beside the left subtree
  cudaEvent_t ev_u = f.ev[2 * level], ev_t = f.ev[2 * level + 1];
  GPTQ_CUDA_CHECK(c, cudaEventRecord(ev_u, c->stream));
  GPTQ_CUDA_CHECK(c, cudaStreamWaitEvent(f.side, ev_u, 0));
  {
    cudaStream_t main = c->stream;
    c->stream = f.side;
    GemmArgs g3{n1, n2, n2, U12, n2, 1, R22, ld, 1, T2, n2, 1.f, 0.f, kBUpper};
    rc = gemm_f32(c, g3);
    c->stream = main;
    if (rc) return rc;
  }
  GPTQ_CUDA_CHECK(c, cudaEventRecord(ev_t, f.side));
  if ((rc = rec(f, s, mid, level + 1, next))) return rc;
  GPTQ_CUDA_CHECK(c, cudaStreamWaitEvent(c->stream, ev_t, 0));
  // R12 = -R11 T2  (R11(i,k) = 0 for k < i)
  GemmArgs g4{n1, n2, n1, Ablk, ld, 1, T2, n2, 1, Rblk, ld, -1.f, 0.f, kAUpper};
  if ((rc = gemm_f32(c, g4))) return rc;
  // strict lower block of this level
  return copy2d(c, nullptr, 0, M + (long long)mid * ld + s, ld, n2, n1);
}

int factor_inverse(Ctx* c, float* M, int d, float* tmp) {
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_factor_base,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, FB_SMEM));
  if (!c->side) {
    GPTQ_CUDA_CHECK(c, cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking));
    for (int k = 0; k < 2 * 64; ++k)
      GPTQ_CUDA_CHECK(c, cudaEventCreateWithFlags(&c->ev[k], cudaEventDisableTiming));
  }
  FactorRun f;
  f.c = c;
  f.M = M;
  f.ld = d;
  f.tmp = tmp;
  f.side = c->side;
  for (int k = 0; k < 2 * 64; ++k) f.ev[k] = c->ev[k];
  return rec(f, 0, d, 0, tmp);
}

}  // namespace gptq
