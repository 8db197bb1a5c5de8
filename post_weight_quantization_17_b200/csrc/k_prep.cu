// a2: preconditioning of H in the order of [T] §10 — dead features, processing permutation
// (act-order, [T] §8.3 eq.(34)), damping ([T] eq.(12)).
#include "kernels.h"

namespace gptq {

// diag(H) = scale * diag(S); dead where it is exactly 0 (then replaced by 1).
__global__ void k_diag(const float* __restrict__ S, int d, float scale, float* __restrict__ diagv,
                       uint8_t* __restrict__ dead, DeviceStatus* st) {
  pdl_wait();
  pdl_release();
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  float h = S[(long long)j * d + j] * scale;
  if (!isfinite(h)) raise_error(st, GPTQ_ERR_NONFINITE, j);
  bool z = (h == 0.f);
  dead[j] = z ? 1 : 0;
  diagv[j] = z ? 1.f : h;
}

int prep_diag(Ctx* c, const float* S, int d, float scale, float* diagv, uint8_t* dead) {
  GPTQ_LAUNCH(c, k_diag, (d + 255) / 256, 256, 0, S, d, scale, diagv, dead, c->status);
  return GPTQ_OK;
}

// Deterministic fp64 sum of diag(H') (one CTA; the permutation does not change the mean).
__global__ void __launch_bounds__(1024) k_mean(const float* __restrict__ diagv, int d,
                                               DeviceStatus* st) {
  pdl_wait();
  pdl_release();
  __shared__ double part[32];
  double acc = 0.0;
  for (int j = threadIdx.x; j < d; j += blockDim.x) acc += (double)diagv[j];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) st->dsum = v / (double)d;
  }
}

int prep_mean(Ctx* c, const float* diagv, int d) {
  GPTQ_LAUNCH(c, k_mean, 1, 1024, 0, diagv, d, c->status);
  return GPTQ_OK;
}

// act-order: position of column j = #{l : diag_l > diag_j or (diag_l == diag_j and l < j)},
// i.e. a stable sort by descending diag(H).
__global__ void __launch_bounds__(256) k_rank(const float* __restrict__ diagv, int d,
                                              int32_t* __restrict__ perm) {
  pdl_wait();
  pdl_release();
  __shared__ float tile[1024];
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const float v = (j < d) ? diagv[j] : 0.f;
  int pos = 0;
  for (int base = 0; base < d; base += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x)
      tile[t] = (base + t < d) ? diagv[base + t] : -INFINITY;
    __syncthreads();
    const int lim = min(1024, d - base);
    for (int t = 0; t < lim; ++t) {
      float u = tile[t];
      int l = base + t;
      pos += (u > v) || (u == v && l < j);
    }
  }
  if (j < d) perm[pos] = j;
}

__global__ void k_iota(int32_t* p, int d) {
  pdl_wait();
  pdl_release();
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < d) p[j] = j;
}

int prep_perm(Ctx* c, const float* diagv, int d, int act_order, int32_t* perm) {
  if (act_order) GPTQ_LAUNCH(c, k_rank, (d + 255) / 256, 256, 0, diagv, d, perm);
  else GPTQ_LAUNCH(c, k_iota, (d + 255) / 256, 256, 0, perm, d);
  return GPTQ_OK;
}

// H'[a][b] = scale * S_sym[π_a][π_b], diagonal from diagv (dead fix-up).  S holds its lower
// triangle.  Identity permutation: block (J, I) with J <= I reads the 32 x 32 tile S[I][J] of the
// lower triangle once (coalesced, through shared memory) and writes that tile and its mirror
// (J, I) of H', to Hp and, when S2 is given, to S2 as well.  S2 may be S itself: a block reads
// only its own lower tile, before writing it or its mirror, and no other block reads either.
__global__ void k_build_identity(const float* S, int d, float scale,
                                 const float* __restrict__ diagv, float* __restrict__ Hp,
                                 float* S2) {
  pdl_wait();
  pdl_release();
  const int I = blockIdx.y, J = blockIdx.x;
  if (J > I) return;
  __shared__ float t[32][33];
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  const int r0 = I * 32, c0 = J * 32;
  for (int r = ty; r < 32; r += 8) {
    const int a = r0 + r, b = c0 + tx;
    t[r][tx] = (a < d && b < d && b <= a) ? S[(long long)a * d + b] : 0.f;
  }
  __syncthreads();
  // tile (I, J): rows r0 + r, columns c0 + tx
  for (int r = ty; r < 32; r += 8) {
    const int a = r0 + r, b = c0 + tx;
    if (a >= d || b >= d) continue;
    const float v = (a == b) ? diagv[a] : (a > b ? t[r][tx] : t[tx][r]) * scale;
    Hp[(long long)a * d + b] = v;
    if (S2) S2[(long long)a * d + b] = v;
  }
  if (I == J) return;
  // mirror (J, I): rows c0 + r, columns r0 + tx, H'[c0 + r][r0 + tx] = scale S[r0 + tx][c0 + r]
  for (int r = ty; r < 32; r += 8) {
    const int a = c0 + r, b = r0 + tx;
    if (a >= d || b >= d) continue;
    const float v = t[tx][r] * scale;
    Hp[(long long)a * d + b] = v;
    if (S2) S2[(long long)a * d + b] = v;
  }
}

__global__ void k_build_perm(const float* __restrict__ S, int d, float scale,
                             const float* __restrict__ diagv, const int32_t* __restrict__ perm,
                             float* __restrict__ Hp) {
  pdl_wait();
  pdl_release();
  const int a = blockIdx.y;
  const int pa = perm[a];
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < d; b += gridDim.x * blockDim.x) {
    int pb = perm[b];
    float v;
    if (pa == pb) v = diagv[pa];
    else {
      int hi = max(pa, pb), lo = min(pa, pb);
      v = S[(long long)hi * d + lo] * scale;
    }
    Hp[(long long)a * d + b] = v;
  }
}

int prep_build(Ctx* c, float* S, int d, float scale, const float* diagv,
               const int32_t* perm, bool identity, float* Hp, bool* wrote_S) {
  *wrote_S = false;
  if (identity) {
    dim3 grid((d + 31) / 32, (d + 31) / 32), block(32, 8);
    GPTQ_LAUNCH(c, k_build_identity, grid, block, 0, (const float*)S, d, scale, diagv, Hp, S);
    *wrote_S = true;
  } else {
    dim3 grid((d + 255) / 256 < 8 ? (d + 255) / 256 : 8, d);
    GPTQ_LAUNCH(c, k_build_perm, grid, 256, 0, S, d, scale, diagv, perm, Hp);
  }
  return GPTQ_OK;
}

__global__ void k_copy(const float* __restrict__ src, float* __restrict__ dst, size_t n,
                       bool vec) {
  pdl_wait();
  pdl_release();
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  size_t n4 = vec ? n / 4 : 0;
  for (size_t k = e; k < n4; k += stride)
    reinterpret_cast<float4*>(dst)[k] = reinterpret_cast<const float4*>(src)[k];
  for (size_t k = n4 * 4 + e; k < n; k += stride) dst[k] = src[k];
}

int prep_copy(Ctx* c, const float* src, float* dst, size_t count) {
  bool vec = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
  size_t work = vec ? count / 4 + 4 : count;
  int blocks = (int)std::min<size_t>((work + 255) / 256, (size_t)c->num_sms * 8);
  if (blocks < 1) blocks = 1;
  GPTQ_LAUNCH(c, k_copy, blocks, 256, 0, src, dst, count, vec);
  return GPTQ_OK;
}

// λ = max(percdamp * mean(diag H'), 2^-23); H_λ = H' + λ I (in place on the diagonal).
__global__ void k_damp(float* __restrict__ Hl, int d, float percdamp, DeviceStatus* st) {
  pdl_wait();
  pdl_release();
  const double mean = st->dsum;
  const double lam_d = fmax((double)percdamp * mean, 1.1920928955078125e-07);
  const float lam = (float)lam_d;
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j == 0) st->lam = lam;
  if (j < d) Hl[(long long)j * d + j] += lam;
}

int prep_damp(Ctx* c, float* Hl, int d, float percdamp) {
  GPTQ_LAUNCH(c, k_damp, (d + 255) / 256, 256, 0, Hl, d, percdamp, c->status);
  return GPTQ_OK;
}

}  // namespace gptq
