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
// inverted inside one CTA, in registers.  T2 = U12 R22 needs only the right subtree, so it runs on a second
// stream beside the left subtree's factorization.  A non-positive or non-finite pivot raises GPTQ_ERR_NOT_PD /
// GPTQ_ERR_NONFINITE in the device status word (the host retries with more damping).
#include <algorithm>

#include "kernels.h"
#include "gemm_simt.cuh"

namespace gptq {

constexpr int FB = 128;                 // diagonal block factored inside one CTA
constexpr int FB_WARPS = FB / 8;        // warp w holds rows 8w .. 8w+7 (one pivot tile)
constexpr int FB_THREADS = 32 * FB_WARPS;
constexpr int FB_LDS = FB + 1;          // staging row stride (mirrored reads: 4-way conflicts)
constexpr int FB_SMEM = FB * FB_LDS * 4;

__device__ __forceinline__ float recip_sqrt(float p) {
  // 1/sqrt(p): hardware estimate refined by one Newton-Raphson step y <- y (3 - p y^2) / 2
  const float y = rsqrtf(p);
  return y * fmaf(-0.5f * p * y, y, 1.5f);
}

// Factor + invert the diagonal block M[s:s+n, s:s+n] (upper triangle read), n <= FB.
// Writes R = U^{-1} into the upper triangle and zeros below it.
//
// Row elimination on [H | I] from the last index: at step j the pivot row j is scaled by
// 1/sqrt(pivot) and subtracted from every row i < j so that column j of H vanishes above the
// diagonal.  The row operations form an upper-triangular E with E H lower triangular
// (= U^T), hence E = U^{-1} = R, which is what the right half holds at the end.  For a row
// i < j the live part of the left half is columns < j and that of the right half is columns
// >= j, so each row is kept as ONE 128-wide register row: column c holds H for c < j and R for
// c >= j.  When step j passes, column j switches from H (eliminated) to R (-m_i / sqrt(pivot)).
// The multiplier m_i of row i is entry i of the scaled pivot row (the trailing block stays
// exactly symmetric: both copies of an entry receive the same products).
//
// Registers: thread (warp w, lane l) holds rows 8w..8w+7, columns 4l..4l+3.  Pivots go by
// tiles of 8 (one warp's rows), last tile first:
//   phase 1  the owning warp eliminates its 8 rows among themselves (warp shuffles only) and
//            publishes the 8 scaled pivot rows to a double-buffered shared tile;
//   phase 2  every warp with rows above the tile applies them as a rank-8 update.  The 8
//            columns of the tile switch to R during the tile: their final value is
//            -sum_j m_i(j) r'_j[c] with r'_j[c] = 0 for c < j, so those entries restart from 0
//            and the published rows carry the zeros.
// The next tile's owner starts phase 1 as soon as its own phase 2 is done; warps whose rows
// are final leave the loop and write them out while the rest continue, and the barrier counts
// only the warps still working (every reader of a tile buffer takes part in the barrier that
// precedes its next overwrite).  Indices >= n are padded with the identity.
__global__ void __launch_bounds__(FB_THREADS, 1) k_factor_base(float* __restrict__ M, long long ld,
                                                                int s, int n, DeviceStatus* st) {
  pdl_wait();
  pdl_release();
  extern __shared__ __align__(16) float fsm[];
  float(*S)[FB_LDS] = reinterpret_cast<float(*)[FB_LDS]>(fsm);       // staging (load phase)
  float(*tile)[8][FB] = reinterpret_cast<float(*)[8][FB]>(fsm);       // 2 x 8 pivot rows (after)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = 8 * warp, c0 = 4 * lane;
  // coalesced load of the upper triangle's row segments into shared memory
  {
    const float* base = M + (long long)s * ld + s;
    const bool vec = ((reinterpret_cast<uintptr_t>(base) & 15) == 0) && (ld % 4 == 0);
    float4 v[FB * FB / 4 / FB_THREADS];
#pragma unroll
    for (int u = 0; u < FB * FB / 4 / FB_THREADS; ++u) {
      const int e = tid + u * FB_THREADS, i = e >> 5, k = (e & 31) * 4;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < n && k + 3 >= i && k < n) {
        const float* src = base + (long long)i * ld + k;
        if (vec && k + 4 <= n) {
          v[u] = *reinterpret_cast<const float4*>(src);
        } else {
          v[u].x = src[0];
          if (k + 1 < n) v[u].y = src[1];
          if (k + 2 < n) v[u].z = src[2];
          if (k + 3 < n) v[u].w = src[3];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < FB * FB / 4 / FB_THREADS; ++u) {
      const int e = tid + u * FB_THREADS, i = e >> 5, k = (e & 31) * 4;
      S[i][k] = v[u].x;
      S[i][k + 1] = v[u].y;
      S[i][k + 2] = v[u].z;
      S[i][k + 3] = v[u].w;
    }
  }
  __syncthreads();
  float x[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int i = i0 + a, c = c0 + t;
      x[a][t] = (i < n && c < n) ? (c >= i ? S[i][c] : S[c][i]) : (i == c ? 1.f : 0.f);
    }
  __syncthreads();  // the staging area becomes the tile buffers
  int bad = 0;
  for (int jb = FB_WARPS - 1; jb >= warp; --jb) {
    float(*tb)[FB] = tile[jb & 1];
    if (warp == jb) {
      // ---- phase 1: the tile's own rows, last first
#pragma unroll
      for (int a = 7; a >= 0; --a) {
        const int j = 8 * jb + a;
        const int jl = 2 * jb + (a >> 2);  // lane holding column j, as element a & 3
        float piv = __shfl_sync(0xffffffffu, x[a][a & 3], jl);
        if (!(piv > 0.f) || !isfinite(piv)) {
          if (bad == 0) bad = isfinite(piv) ? GPTQ_ERR_NOT_PD : GPTQ_ERR_NONFINITE;
          piv = 1.f;
        }
        const float sc = recip_sqrt(piv);
        float r[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) r[t] = x[a][t] * sc;
        if (lane == jl) r[a & 3] = sc;  // R_jj (the right half's 1, scaled)
        // row j is final: R for c >= j, zero below the diagonal
#pragma unroll
        for (int t = 0; t < 4; ++t) x[a][t] = (c0 + t < j) ? 0.f : r[t];
        // published row: tile columns below j carry 0 (see phase 2)
        const bool tcol = (lane >> 1) == jb;
        *reinterpret_cast<float4*>(&tb[a][c0]) =
            tcol ? make_float4(x[a][0], x[a][1], x[a][2], x[a][3])
                 : make_float4(r[0], r[1], r[2], r[3]);
#pragma unroll
        for (int ap = 0; ap < a; ++ap) {
          const float mm = __shfl_sync(0xffffffffu, r[ap & 3], 2 * jb + (ap >> 2));
#pragma unroll
          for (int t = 0; t < 4; ++t) x[ap][t] = fmaf(-mm, r[t], x[ap][t]);
          if (lane == jl) x[ap][a & 3] = -mm * sc;
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(32 * (jb + 1)) : "memory");
    if (warp < jb) {
      // ---- phase 2: rank-8 update of this warp's rows
      if ((lane >> 1) == jb) {
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int t = 0; t < 4; ++t) x[a][t] = 0.f;
      }
#pragma unroll
      for (int a = 7; a >= 0; --a) {
        const float4 v4 = *reinterpret_cast<const float4*>(&tb[a][c0]);
        const float4 ma = *reinterpret_cast<const float4*>(&tb[a][i0]);
        const float4 mb = *reinterpret_cast<const float4*>(&tb[a][i0 + 4]);
        const float v[4] = {v4.x, v4.y, v4.z, v4.w};
        const float m[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
        for (int ap = 0; ap < 8; ++ap)
#pragma unroll
          for (int t = 0; t < 4; ++t) x[ap][t] = fmaf(-m[ap], v[t], x[ap][t]);
      }
    }
  }
  if (bad && lane == 0) raise_error(st, bad, s);
  // write the warp's rows of R (zeros below the diagonal are already in place)
  const bool vec = ((reinterpret_cast<uintptr_t>(M + (long long)s * ld + s) & 15) == 0) &&
                   (ld % 4 == 0) && (c0 + 4 <= n);
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = i0 + a;
    if (i >= n) break;
    float* row = M + (long long)(s + i) * ld + s;
    if (vec) {
      *reinterpret_cast<float4*>(row + c0) = make_float4(x[a][0], x[a][1], x[a][2], x[a][3]);
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (c0 + t < n) row[c0 + t] = x[a][t];
    }
  }
}

// Zeros the strict lower triangle of the d x d matrix M (row stride ld).  Grid: x over
// 1024-column slices of a row (256 threads, 4 columns each), y over rows (grid-strided).
__global__ void k_zero_lower(float* __restrict__ M, long long ld, int d, int vec) {
  pdl_wait();
  pdl_release();
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  for (int r = blockIdx.y; r < d; r += gridDim.y) {
    if (c0 >= r) continue;
    float* row = M + (long long)r * ld + c0;
    if (vec && c0 + 4 <= r)
      *reinterpret_cast<float4*>(row) = make_float4(0.f, 0.f, 0.f, 0.f);
    else
      for (int u = 0; u < 4 && c0 + u < r; ++u) row[u] = 0.f;
  }
}

static int zero_lower(Ctx* c, float* M, long long ld, int d) {
  if (d <= 1) return GPTQ_OK;
  const int vec = (ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(M) & 15) == 0);
  const int gx = (d + 1023) / 1024;
  const int gy = std::min(d, std::max(1, c->num_sms * 16 / gx));
  GPTQ_LAUNCH(c, k_zero_lower, dim3(gx, gy), 256, 0, M, ld, d, vec);
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

// Nodes whose right child has at least this many columns run their four products on CTA pairs
// (k_gemm_pair) with operands split into tf32 halves beforehand; the rest on k_gemm_tc /
// k_gemm_small (below this size a grid of 256 x 256 tiles leaves most of the 74 pairs idle, and
// the single-CTA GEMM measured faster).  The pair path needs 16-byte aligned rows (ld and n2
// multiples of 4).
constexpr int kFactorPairMin = 2048;
static bool pair_node(int n2, long long ld) {
  return n2 >= kFactorPairMin && n2 % 4 == 0 && ld % 4 == 0;
}
// A pair node's buffers: the halves of B (later of R11: n1 x n1), of R22, of U12 and of T2.
static size_t pair_level_floats(int n1, int n2) {
  return 2 * (size_t)n1 * n1 + 2 * (size_t)n2 * n2 + 4 * (size_t)n1 * n2;
}

// Scratch of the recursion below a node of n columns: its own level's buffers, then (one child
// at a time) the children's.
static size_t node_floats(int n, long long ld) {
  if (n <= FB) return 0;
  const int n1 = larger_child(n), n2 = n - n1;
  const size_t own = pair_node(n2, ld) ? pair_level_floats(n1, n2) : 2 * level_floats(n);
  return own + std::max(node_floats(n1, ld), node_floats(n2, ld));
}

size_t factor_tmp_floats(int d) { return node_floats(d, d) + 64; }

struct FactorRun {
  Ctx* c;
  float* M;
  long long ld;
  float* tmp;              // level buffers, consecutive
  cudaStream_t side;       // T2 = U12 R22 runs here, beside the left subtree
  cudaEvent_t ev[2 * 64];  // per level: U12 ready, T2 ready
  int stage_base, stage_gemm, stage_copy;  // stages the launches are timed under
  bool pair;                               // large nodes on CTA pairs (k_gemm_pair)
};

static int rec(FactorRun& f, int s, int e, int level, float* buf);

// A node on CTA pairs: the same four products as below, with the operands split into tf32
// halves first (B and R22 before the right child's results are used, R11 after the left child),
// and U12 and T2 written by their products directly as halves, since they are only operands.
static int rec_pair(FactorRun& f, int s, int e, int level, float* buf) {
  Ctx* c = f.c;
  const long long ld = f.ld;
  float* M = f.M;
  const int n = e - s, n1 = larger_child(n), mid = s + n1, n2 = e - mid;
  float* Bh = buf;                                  // B's halves, later R11's (n1 x n1)
  float* Bl = Bh + (size_t)n1 * n1;
  float* R22h = Bl + (size_t)n1 * n1;
  float* R22l = R22h + (size_t)n2 * n2;
  float* U12h = R22l + (size_t)n2 * n2;
  float* U12l = U12h + (size_t)n1 * n2;
  float* T2h = U12l + (size_t)n1 * n2;
  float* T2l = T2h + (size_t)n1 * n2;
  float* next = T2l + (size_t)n1 * n2;
  int rc = rec(f, mid, e, level + 1, next);
  if (rc) return rc;
  const float* Bblk = M + (long long)s * ld + mid;   // rows s..mid, cols mid..e (H_λ)
  float* Rblk = M + (long long)s * ld + mid;         // becomes R12
  const float* R22 = M + (long long)mid * ld + mid;
  float* Ablk = M + (long long)s * ld + s;
  StageScope stage(c, f.stage_copy);
  if ((rc = split_tf32(c, Bblk, ld, n1, n2, Bh, Bl, n2))) return rc;
  if ((rc = split_tf32(c, R22, ld, n2, n2, R22h, R22l, n2, true))) return rc;
  c->stage = f.stage_gemm;
  // U12 = B R22^T: opB(k, j) = R22[j][k] (K-major), zero for k < j
  GemmPairArgs g{};
  g.M = n1; g.N = n2; g.K = n2;
  g.Ah = Bh; g.Al = Bl; g.lda = n2;
  g.Bh = R22h; g.Bl = R22l; g.ldb = n2; g.b_kmajor = true;
  g.Ch = U12h; g.Cl = U12l; g.ldc = n2; g.alpha = 1.f; g.beta = 0.f; g.flags = kBLower;
  g.partial_k = kFactorPartialK;
  if ((rc = gemm_pair(c, g))) return rc;
  // A' = A - U12 U12^T, tiles touching the upper triangle
  GemmPairArgs g2{};
  g2.M = n1; g2.N = n1; g2.K = n2;
  g2.Ah = U12h; g2.Al = U12l; g2.lda = n2;
  g2.Bh = U12h; g2.Bl = U12l; g2.ldb = n2; g2.b_kmajor = true;
  g2.C = Ablk; g2.ldc = ld; g2.alpha = -1.f; g2.beta = 1.f; g2.flags = kCUpper;
  g2.partial_k = kFactorPartialK;
  if ((rc = gemm_pair(c, g2))) return rc;
  // T2 = U12 R22 (R22(k, j) = 0 for k > j) on the side stream, beside the left subtree
  cudaEvent_t ev_u = f.ev[2 * level], ev_t = f.ev[2 * level + 1];
  GPTQ_CUDA_CHECK(c, cudaEventRecord(ev_u, c->stream));
  GPTQ_CUDA_CHECK(c, cudaStreamWaitEvent(f.side, ev_u, 0));
  {
    cudaStream_t main = c->stream;
    c->stream = f.side;
    GemmPairArgs g3{};
    g3.M = n1; g3.N = n2; g3.K = n2;
    g3.Ah = U12h; g3.Al = U12l; g3.lda = n2;
    g3.Bh = R22h; g3.Bl = R22l; g3.ldb = n2; g3.b_kmajor = false;
    g3.Ch = T2h; g3.Cl = T2l; g3.ldc = n2; g3.alpha = 1.f; g3.beta = 0.f; g3.flags = kBUpper;
    g3.partial_k = kFactorPartialK;
    rc = gemm_pair(c, g3);
    c->stream = main;
    if (rc) return rc;
  }
  GPTQ_CUDA_CHECK(c, cudaEventRecord(ev_t, f.side));
  if ((rc = rec(f, s, mid, level + 1, next))) return rc;
  GPTQ_CUDA_CHECK(c, cudaStreamWaitEvent(c->stream, ev_t, 0));
  // R12 = -R11 T2 (R11(i, k) = 0 for k < i)
  c->stage = f.stage_copy;
  if ((rc = split_tf32(c, Ablk, ld, n1, n1, Bh, Bl, n1, true))) return rc;
  c->stage = f.stage_gemm;
  GemmPairArgs g4{};
  g4.M = n1; g4.N = n2; g4.K = n1;
  g4.Ah = Bh; g4.Al = Bl; g4.lda = n1;
  g4.Bh = T2h; g4.Bl = T2l; g4.ldb = n2; g4.b_kmajor = false;
  g4.C = Rblk; g4.ldc = ld; g4.alpha = -1.f; g4.beta = 0.f; g4.flags = kAUpper;
  g4.partial_k = kFactorPartialK;
  return gemm_pair(c, g4);
}

static int rec(FactorRun& f, int s, int e, int level, float* buf) {
  Ctx* c = f.c;
  const long long ld = f.ld;
  float* M = f.M;
  const int n = e - s;
  if (n <= FB) {
    StageScope stage(c, f.stage_base);
    GPTQ_LAUNCH(c, k_factor_base, 1, FB_THREADS, FB_SMEM, M, ld, s, n, c->status);
    return GPTQ_OK;
  }
  if (f.pair && pair_node(n - larger_child(n), ld)) return rec_pair(f, s, e, level, buf);
  StageScope stage(c, f.stage_gemm);
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
  GemmArgs g{n1, n2, n2, Bblk, ld, 1, R22, 1, ld, U12, n2, 1.f, 0.f, kBLower, kFactorPartialK};
  if ((rc = gemm_f32(c, g))) return rc;
  // A' = A - U12 U12^T  (upper tiles only)
  GemmArgs g2{n1, n1, n2, U12, n2, 1, U12, 1, n2, Ablk, ld, -1.f, 1.f, kCUpper, kFactorPartialK};
  if ((rc = gemm_f32(c, g2))) return rc;
  // T2 = U12 R22 (R22(k,j) = 0 for k > j) on the side stream, beside the left subtree
  cudaEvent_t ev_u = f.ev[2 * level], ev_t = f.ev[2 * level + 1];
  GPTQ_CUDA_CHECK(c, cudaEventRecord(ev_u, c->stream));
  GPTQ_CUDA_CHECK(c, cudaStreamWaitEvent(f.side, ev_u, 0));
  {
    cudaStream_t main = c->stream;
    c->stream = f.side;
    GemmArgs g3{n1, n2, n2, U12, n2, 1, R22, ld, 1, T2, n2, 1.f, 0.f, kBUpper, kFactorPartialK};
    rc = gemm_f32(c, g3);
    c->stream = main;
    if (rc) return rc;
  }
  GPTQ_CUDA_CHECK(c, cudaEventRecord(ev_t, f.side));
  if ((rc = rec(f, s, mid, level + 1, next))) return rc;
  GPTQ_CUDA_CHECK(c, cudaStreamWaitEvent(c->stream, ev_t, 0));
  // R12 = -R11 T2  (R11(i,k) = 0 for k < i)
  GemmArgs g4{n1, n2, n1, Ablk, ld, 1, T2, n2, 1, Rblk, ld, -1.f, 0.f, kAUpper, kFactorPartialK};
  return gemm_f32(c, g4);
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
  // with per-stage timing on, T2 runs on the main stream too, so that no two timed launches
  // overlap and each launch's events measure that kernel alone
  f.side = c->timing ? c->stream : c->side;
  for (int k = 0; k < 2 * 64; ++k) f.ev[k] = c->ev[k];
  // inside the hot path the factorization has stages of its own; for two-sided rounding's
  // factors it stays under the caller's stage
  const bool own = (c->stage == GPTQ_STAGE_PREPARE);
  f.stage_base = own ? GPTQ_STAGE_FACTOR_BASE : c->stage;
  f.stage_gemm = own ? GPTQ_STAGE_FACTOR_GEMM : c->stage;
  f.stage_copy = own ? GPTQ_STAGE_FACTOR_COPY : c->stage;
  f.pair = c->num_sms >= 2 && (reinterpret_cast<uintptr_t>(M) & 15) == 0 &&
           (reinterpret_cast<uintptr_t>(tmp) & 15) == 0;
  int rc = rec(f, 0, d, 0, tmp);
  if (rc) return rc;
  // Below the diagonal M still holds H_λ and the products' by-products: no product reads there
  // (each tile's k-range starts at its own first row or column, so the only entries below the
  // diagonal that a product reads lie inside a diagonal block of <= 128, which the base kernel
  // zeroed, and the CTA-pair products read triangular operands through splits that zero them),
  // so the strict lower triangle is cleared once, here.
  StageScope stage(c, f.stage_copy);
  return zero_lower(c, M, d, d);
}

}  // namespace gptq
