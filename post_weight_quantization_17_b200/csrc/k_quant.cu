// a4-a7: grid fit, working copy, in-block column quantization, lazy trailing update,
// per-column loss, un-permute.
//
// [W] Algorithm 1 and [T] §9.2-§9.3, §10: for each block [i, i+nb) of processing positions,
// each column j is quantized (c = clip(rint(w/Δ)+z), q = Δ(c-z), [T] eq.(36)), its scaled
// residual η = (w - q) / R_jj is kept in E, the block's remaining columns receive
// w_k -= η R_jk immediately (eq.(42)), and after the block the rest of W receives
// W[:, i+nb:] -= E R[i:i+nb, i+nb:] (eq.(46)).
#include "kernels.h"
#include "gemm_simt.cuh"
#include "tc_util.cuh"

#include <utility>

namespace gptq {

// ------------------------------------------------------------------------------------------
// a4: static grid per (row, group of original columns), [T] §1.1 and §8.3: the min-max fit
// (range extended to contain 0), or the symmetric fit around 0 (Δ = 2 max|w| / maxq,
// z = (maxq + 1) / 2; maxq = 2 is the ternary grid).  fp32 arithmetic.
template <class T>
__device__ __forceinline__ void gridfit_finish(float mn, float mx, bool bad, int maxq_i,
                                               bool symmetric, int r, float* scale,
                                               int32_t* zero, DeviceStatus* st) {
  if (bad) raise_error(st, GPTQ_ERR_NONFINITE, r);
  const float maxq = (float)maxq_i;
  float delta, z;
  if (symmetric) {
    const float M = fmaxf(-mn, mx);  // mn <= 0 <= mx
    delta = (M == 0.f) ? 1.f : __fdiv_rn(2.f * M, maxq);
    z = (float)((maxq_i + 1) / 2);
  } else {
    delta = (mx == mn) ? 1.f : __fdiv_rn(__fsub_rn(mx, mn), maxq);
    z = fminf(fmaxf(rintf(__fdiv_rn(-mn, delta)), 0.f), maxq);
  }
  *scale = delta;
  *zero = (int32_t)z;
}

// One warp per (row, 4 consecutive groups) when groups are 128 wide in 16-bit W: each lane
// loads its 4 elements of all 4 groups up front (8 bytes each) and the four reductions run
// side by side.  Otherwise one warp per (row, group).
template <class T>
__global__ void k_gridfit(const T* __restrict__ W, int m, int d, int g, int ng, int maxq,
                          bool symmetric, float* __restrict__ scales, int32_t* __restrict__ zeros,
                          DeviceStatus* st) {
  pdl_wait();
  pdl_release();
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const bool quad = (g == 128) && (d % 512 == 0) && (sizeof(T) == 2) &&
                    ((reinterpret_cast<uintptr_t>(W) & 7) == 0);
  if (quad) {
    const int nq = ng / 4;
    if (warp >= (long long)m * nq) return;
    const int r = (int)(warp / nq), k0 = 4 * (int)(warp % nq);
    const T* row = W + (long long)r * d + (long long)k0 * 128 + 4 * lane;
    uint2 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) raw[u] = *reinterpret_cast<const uint2*>(row + u * 128);
    float mn[4], mx[4];
    bool bad = false;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const T* e = reinterpret_cast<const T*>(&raw[u]);
      mn[u] = 0.f;
      mx[u] = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float v = to_f32<T>(e[t]);
        bad |= !isfinite(v);
        mn[u] = fminf(mn[u], v);
        mx[u] = fmaxf(mx[u], v);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        mn[u] = fminf(mn[u], __shfl_xor_sync(0xffffffffu, mn[u], o));
        mx[u] = fmaxf(mx[u], __shfl_xor_sync(0xffffffffu, mx[u], o));
      }
    bad = __any_sync(0xffffffffu, bad);
    if (lane < 4) {
      float a = mn[0], b = mx[0];
#pragma unroll
      for (int u = 1; u < 4; ++u)
        if (lane == u) {
          a = mn[u];
          b = mx[u];
        }
      const long long o = (long long)r * ng + k0 + lane;
      gridfit_finish<T>(a, b, bad && lane == 0, maxq, symmetric, r, scales + o, zeros + o, st);
    }
    return;
  }
  if (warp >= (long long)m * ng) return;
  const int r = (int)(warp / ng), k = (int)(warp % ng);
  const int c0 = k * g, c1 = min(d, c0 + g);
  float mn = 0.f, mx = 0.f;
  bool bad = false;
  const T* row = W + (long long)r * d;
  for (int cc = c0 + lane; cc < c1; cc += 32) {
    float v = to_f32<T>(row[cc]);
    bad |= !isfinite(v);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0)
    gridfit_finish<T>(mn, mx, bad, maxq, symmetric, r, scales + (long long)r * ng + k,
                      zeros + (long long)r * ng + k, st);
}

int grid_fit(Ctx* c, const void* W, int w_dtype, int m, int d, int maxq, bool symmetric,
             int group, float* scales, int32_t* zeros) {
  const int g = (group == -1) ? d : group;
  const int ng = (d + g - 1) / g;
  const bool quad = (g == 128) && (d % 512 == 0) && (w_dtype != GPTQ_F32) &&
                    ((reinterpret_cast<uintptr_t>(W) & 7) == 0);
  const long long warps = (long long)m * (quad ? ng / 4 : ng);
  const int blocks = (int)((warps * 32 + 255) / 256);
  if (w_dtype == GPTQ_F16)
    GPTQ_LAUNCH(c, k_gridfit<__half>, blocks, 256, 0, (const __half*)W, m, d, g, ng, maxq, symmetric, scales,
                zeros, c->status);
  else if (w_dtype == GPTQ_BF16)
    GPTQ_LAUNCH(c, k_gridfit<__nv_bfloat16>, blocks, 256, 0, (const __nv_bfloat16*)W, m, d, g, ng,
                maxq, symmetric, scales, zeros, c->status);
  else
    GPTQ_LAUNCH(c, k_gridfit<float>, blocks, 256, 0, (const float*)W, m, d, g, ng, maxq, symmetric, scales,
                zeros, c->status);
  return GPTQ_OK;
}

// grid index of each processing position (static groups: floor(π_j / g); dynamic groups:
// j / g) and the inverse permutation.
__global__ void k_gcol(const int32_t* __restrict__ perm, int d, int group, int dynamic,
                       int32_t* __restrict__ gcol, int32_t* __restrict__ inv) {
  pdl_wait();
  pdl_release();
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  int p = perm ? perm[j] : j;
  gcol[j] = (group == -1) ? 0 : (dynamic ? j : p) / group;
  if (inv) inv[p] = j;
}

int make_gcol(Ctx* c, const int32_t* perm, int d, int group, bool dynamic, int32_t* gcol,
              int32_t* inv) {
  GPTQ_LAUNCH(c, k_gcol, (d + 255) / 256, 256, 0, perm, d, group, dynamic ? 1 : 0, gcol, inv);
  return GPTQ_OK;
}

// working copy in processing order: Wk[r][j] = dead[π_j] ? 0 : W[r][π_j]  ([T] §10).
// Grid: x over groups of 4 columns, y strided over rows (no index division).
template <class T>
__global__ void k_init_work(const T* __restrict__ W, long long m, int d,
                            const int32_t* __restrict__ perm, const uint8_t* __restrict__ dead,
                            float* __restrict__ Wk) {
  pdl_wait();
  pdl_release();
  const int j0 = 4 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (j0 >= d) return;
  const bool vec = !perm && (j0 + 4 <= d) && (d % 4 == 0) && (sizeof(T) == 2) &&
                   ((reinterpret_cast<uintptr_t>(W) & 7) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Wk) & 15) == 0);
  int src[4];
  bool keep[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int j = min(j0 + t, d - 1);
    src[t] = perm ? perm[j] : j;
    keep[t] = !(dead && dead[src[t]]);
  }
  for (long long r = blockIdx.y; r < m; r += gridDim.y) {
    const T* wr = W + r * d;
    float* out = Wk + r * d + j0;
    if (vec) {
      const uint2 raw = *reinterpret_cast<const uint2*>(wr + j0);
      const T* e = reinterpret_cast<const T*>(&raw);
      *reinterpret_cast<float4*>(out) =
          make_float4(keep[0] ? to_f32<T>(e[0]) : 0.f, keep[1] ? to_f32<T>(e[1]) : 0.f,
                      keep[2] ? to_f32<T>(e[2]) : 0.f, keep[3] ? to_f32<T>(e[3]) : 0.f);
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (j0 + t < d) out[t] = keep[t] ? to_f32<T>(wr[src[t]]) : 0.f;
    }
  }
}

int init_work(Ctx* c, const void* W, int w_dtype, int m, int d, const int32_t* perm,
              const uint8_t* dead, bool, float* Wk) {
  const int gx = (d + 4 * 256 - 1) / (4 * 256);
  const int gy = std::max(1, std::min(m, (c->num_sms * 16 + gx - 1) / gx));
  const dim3 grid(gx, gy);
  if (w_dtype == GPTQ_F16)
    GPTQ_LAUNCH(c, k_init_work<__half>, grid, 256, 0, (const __half*)W, (long long)m, d, perm, dead, Wk);
  else if (w_dtype == GPTQ_BF16)
    GPTQ_LAUNCH(c, k_init_work<__nv_bfloat16>, grid, 256, 0, (const __nv_bfloat16*)W, (long long)m, d, perm, dead, Wk);
  else
    GPTQ_LAUNCH(c, k_init_work<float>, grid, 256, 0, (const float*)W, (long long)m, d, perm, dead, Wk);
  return GPTQ_OK;
}

// ------------------------------------------------------------------------------------------
// a5: one block of up to 128 columns for 48 rows per CTA (12 warps, 4 rows per warp, 8 lanes
// per row; two CTAs share an SM, so 12288 rows take one round on 148 SMs).  The block is walked in four 32-column sub-blocks; in a sub-block lane q of a row
// owns the 4 consecutive columns 4q .. 4q+3 in registers.  A column step fetches the column's
// value from its owner lane (width-8 shuffle), the 8 lanes run the sequential chain (divide,
// round, clip, residual, η) side by side, and each lane updates only its own later columns
// ([T] eq.(42)).  A sub-block first receives the residuals of the sub-blocks before it
// (E R, the lazy update of [T] eq.(46) at a finer grain, exact by eq.(47)-(49)).  R's block
// and the W block are staged with asynchronous copies; outputs leave through shared memory
// as coalesced row segments.
//
// The quotient w/Δ is the IEEE (correctly rounded) one, computed from y = RN(1/Δ), taken once
// per grid group: q0 = RN(w y), r = w - q0 Δ (exact, by FMA), u = RN(q0 + r y).  By
// Markstein's theorem (IBM J. Res. Dev. 34(1), 1990: y within half an ulp of 1/Δ and q0 within
// an ulp of w/Δ make RN(q0 + r y) = RN(w/Δ)) this is the same fp32 value as a division, at a
// third of its latency on the column chain.
constexpr int kColWarps = 12;                // 48 rows per CTA: two CTAs fit an SM
constexpr int kColLanes = 8;                 // lanes per row
constexpr int kColSub = 4 * kColLanes;       // sub-block width: 4 columns per lane
constexpr int kColCtaRows = 48;
constexpr int kColLd = 132;  // padded row of the staging buffers (16-byte rows)
constexpr int kColSmem = 128 * 128 * 4 + kColCtaRows * kColLd * 4 + kColWarps * 128 * 4;
static_assert(kColCtaRows == kColWarps * 32 / kColLanes && kColCtaRows == kColRows, "rows per CTA");

__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(gsrc),
               "r"(valid ? 4 : 0)
               : "memory");
}
// 16-byte copy of the first `bytes` (0..16) bytes, the rest zero-filled
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, int bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// y = RN(1/Δ) is used only while Δ lies in [2^-100, 2^100], where 1/Δ and the correction stay
// normal; a CTA with any row outside that range takes the division itself.
__device__ __forceinline__ bool quotient_fast(float delta) {
  return delta >= 0x1p-100f && delta <= 0x1p100f;
}
template <bool FAST>
__device__ __forceinline__ float quotient(float w, float delta, float y) {
  if (!FAST) return __fdiv_rn(w, delta);
  const float q0 = __fmul_rn(w, y);
  const float r = fmaf(-q0, delta, w);
  return fmaf(r, y, q0);
}

// The min-max fit of the static grid (the fp32 arithmetic of k_gridfit) from a row's range.
__device__ __forceinline__ void fit_from_range(float mn, float mx, float maxq, float& delta,
                                               float& z) {
  mn = fminf(mn, 0.f);
  mx = fmaxf(mx, 0.f);
  delta = (mx == mn) ? 1.f : __fdiv_rn(__fsub_rn(mx, mn), maxq);
  z = fminf(fmaxf(rintf(__fdiv_rn(-mn, delta)), 0.f), maxq);
}

// min and max over the 8 lanes that hold one row
__device__ __forceinline__ void row_range(float& mn, float& mx) {
#pragma unroll
  for (int o = 1; o < kColLanes; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
}

struct ColStepArgs {
  const float (*Rs)[128];
  const int* gs;
  const float* rinv;
  const float* scales;
  const int32_t* zeros;
  long long srow;  // row * ng
  int q;           // owner index of this lane
  unsigned src0;   // lane of owner 0 in this row's group
  bool active;
  float maxq, D0, Z0, Y0;
};

// One column step at block column off + J (J compile-time: owner lane J >> 2, slot J & 3).
// Columns past the block's end hold zeros with rinv = 0 and zero R rows, so their step is an
// exact no-op and needs no branch.  The code offset c - z is clipped to [-z, maxq - z]
// directly (integers in fp32: the same value as clipping c and subtracting z).
template <int J, bool UNIFORM, bool FAST>
__device__ __forceinline__ void col_step(float (&w)[4], float (&e4)[4], float (&c4)[4],
                                         const ColStepArgs& a, int off) {
  constexpr int TJ = J & 3, QJ = J >> 2;
  const int C = off + J;
  const float wj = __shfl_sync(0xffffffffu, w[TJ], a.src0 + QJ);
  float Dj = a.D0, Zj = a.Z0, Yj = a.Y0;
  if (!UNIFORM && a.active) {
    const int gj = a.gs[C];
    Dj = a.scales[a.srow + gj];
    Zj = (float)a.zeros[a.srow + gj];
    if (FAST) Yj = __frcp_rn(Dj);
  }
  const float u = quotient<FAST>(wj, Dj, Yj);
  const float co = fminf(fmaxf(rintf(u), -Zj), a.maxq - Zj);
  const float qv = __fmul_rn(Dj, co);
  const float eta = __fmul_rn(__fsub_rn(wj, qv), a.rinv[C]);
  const float4 r4 = *reinterpret_cast<const float4*>(&a.Rs[C][off + 4 * a.q]);
  const float rr[4] = {r4.x, r4.y, r4.z, r4.w};
  // later columns of this lane: all of them past the owner, the slots after TJ at the owner
  const float e_hi = (a.q >= QJ) ? eta : 0.f;
  const float e_lo = (a.q > QJ) ? eta : 0.f;
#pragma unroll
  for (int t = 0; t < 4; ++t) w[t] = fmaf(-(t > TJ ? e_hi : e_lo), rr[t], w[t]);
  if (a.q == QJ) {
    w[TJ] = qv;
    e4[TJ] = eta;
    c4[TJ] = co + Zj;
  }
}

template <bool UNIFORM, bool FAST, int... Js>
__device__ __forceinline__ void col_steps(float (&w)[4], float (&e4)[4], float (&c4)[4],
                                          const ColStepArgs& a, int off,
                                          std::integer_sequence<int, Js...>) {
  (col_step<Js, UNIFORM, FAST>(w, e4, c4, a, off), ...);
}

template <bool UNIFORM, bool FAST>
__device__ __forceinline__ void col_walk(float (*St)[kColLd], float (*lossw)[128],
                                         const ColStepArgs& args, int r, int row, int nb, int d,
                                         int i, int ldE, bool vec, float* __restrict__ Wk,
                                         float* __restrict__ E, float* __restrict__ Ehi,
                                         float* __restrict__ Elo, uint8_t* __restrict__ codes,
                                         int dyn, int ng, float* __restrict__ dscales,
                                         int32_t* __restrict__ dzeros) {
  const float(*Rs)[128] = args.Rs;
  const int q = args.q, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int off = 0; off < nb; off += kColSub) {
    float w[4], e4[4] = {0.f, 0.f, 0.f, 0.f}, c4[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const float4 w4 = *reinterpret_cast<const float4*>(&St[r][off + 4 * q]);
      w[0] = w4.x; w[1] = w4.y; w[2] = w4.z; w[3] = w4.w;
    }
    // residuals of the earlier sub-blocks: w -= η[0:off] R[0:off, my columns], 8 at a time
    for (int j = 0; j < off; j += 8) {
      const float4 ea = *reinterpret_cast<const float4*>(&St[r][j]);
      const float4 eb = *reinterpret_cast<const float4*>(&St[r][j + 4]);
      const float e[8] = {ea.x, ea.y, ea.z, ea.w, eb.x, eb.y, eb.z, eb.w};
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 r4 = *reinterpret_cast<const float4*>(&Rs[j + u][off + 4 * q]);
        w[0] = fmaf(-e[u], r4.x, w[0]);
        w[1] = fmaf(-e[u], r4.y, w[1]);
        w[2] = fmaf(-e[u], r4.z, w[2]);
        w[3] = fmaf(-e[u], r4.w, w[3]);
      }
    }
    ColStepArgs sa = args;
    if (dyn == kColSub) {
      // dynamic group = this sub-block: its grid is fitted per row from the current weights
      // (every earlier column's compensation is in w now)
      float mn = fminf(fminf(w[0], w[1]), fminf(w[2], w[3]));
      float mx = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
      row_range(mn, mx);
      float dlt, zz;
      fit_from_range(mn, mx, args.maxq, dlt, zz);
      sa.D0 = dlt;
      sa.Z0 = zz;
      if (q == 0 && args.active) {
        dscales[args.srow + (i + off) / kColSub] = dlt;
        dzeros[args.srow + (i + off) / kColSub] = (int32_t)zz;
      }
    }
    col_steps<UNIFORM, FAST>(w, e4, c4, sa, off, std::make_integer_sequence<int, kColSub>{});
    // the sub-block's η for later sub-blocks; outputs straight from registers
    __syncwarp();
    *reinterpret_cast<float4*>(&St[r][off + 4 * q]) = make_float4(e4[0], e4[1], e4[2], e4[3]);
    const int c = off + 4 * q;
    if (args.active) {
      // η's tf32 halves for the pair GEMM of the tail update, when it is used
      float eh[4], el[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        eh[t] = tc::tf32_rna(e4[t]);
        el[t] = tc::tf32_rna(e4[t] - eh[t]);
      }
      if (vec && c + 4 <= nb) {
        *reinterpret_cast<float4*>(E + (long long)row * ldE + c) =
            make_float4(e4[0], e4[1], e4[2], e4[3]);
        if (Ehi) {
          *reinterpret_cast<float4*>(Ehi + (long long)row * ldE + c) =
              make_float4(eh[0], eh[1], eh[2], eh[3]);
          *reinterpret_cast<float4*>(Elo + (long long)row * ldE + c) =
              make_float4(el[0], el[1], el[2], el[3]);
        }
        *reinterpret_cast<float4*>(Wk + (long long)row * d + i + c) =
            make_float4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uchar4*>(codes + (long long)row * d + i + c) =
            make_uchar4((uint8_t)c4[0], (uint8_t)c4[1], (uint8_t)c4[2], (uint8_t)c4[3]);
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (c + t < nb) {
            E[(long long)row * ldE + c + t] = e4[t];
            if (Ehi) {
              Ehi[(long long)row * ldE + c + t] = eh[t];
              Elo[(long long)row * ldE + c + t] = el[t];
            }
            Wk[(long long)row * d + i + c + t] = w[t];
            codes[(long long)row * d + i + c + t] = (uint8_t)c4[t];
          }
      }
    }
    // Σ η² over the warp's 4 rows (lanes q, q+8, q+16, q+24 share columns)
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float s2 = args.active ? e4[t] * e4[t] : 0.f;
      s2 += __shfl_xor_sync(0xffffffffu, s2, 8);
      s2 += __shfl_xor_sync(0xffffffffu, s2, 16);
      if (lane < kColLanes) lossw[warp][c + t] = s2;
    }
  }
}

template <bool UNIFORM>
__global__ void __launch_bounds__(32 * kColWarps, 2) k_colblock(
    float* __restrict__ Wk, int m, int d, int i, int nb, const float* __restrict__ R,
    float* __restrict__ scales, int32_t* __restrict__ zeros, int ng,
    const int32_t* __restrict__ gcol, int dyn, int maxq, float* __restrict__ E,
    float* __restrict__ Ehi,
    float* __restrict__ Elo, int ldE, uint8_t* __restrict__ codes,
    float* __restrict__ loss_part) {
  extern __shared__ __align__(16) unsigned char smem[];
  float(*Rs)[128] = reinterpret_cast<float(*)[128]>(smem);
  // St: the W block on entry, then sub-block by sub-block η (scaled residual) replaces w
  float(*St)[kColLd] = reinterpret_cast<float(*)[kColLd]>(smem + 128 * 128 * 4);
  float(*lossw)[128] =
      reinterpret_cast<float(*)[128]>(smem + 128 * 128 * 4 + kColCtaRows * kColLd * 4);
  __shared__ int gs[128];
  __shared__ float rinv[128];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * kColCtaRows;
  const int r = warp * (32 / kColLanes) + lane / kColLanes;  // row within the CTA
  const int q = lane % kColLanes;
  const int row = row0 + r;
  const bool active = row < m;

  // R[i:i+nb, i:i+nb] and W[rows, i:i+nb], zero-filled beyond nb; 16-byte copies when the
  // rows are 16-byte aligned
  const bool vec = (d % 4 == 0) && (i % 4 == 0) && (ldE % 4 == 0) &&
                   ((reinterpret_cast<uintptr_t>(R) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Wk) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(E) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Ehi) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(Elo) & 15) == 0) &&
                   ((reinterpret_cast<uintptr_t>(codes) & 3) == 0);
  // R was written before the previous kernel (the factorization, or an earlier block's
  // kernels), so its copies start before the wait; the W block is the previous kernel's output
  if (vec) {
    for (int e = tid; e < 128 * 32; e += blockDim.x) {
      const int a = e >> 5, b = (e & 31) * 4;
      const int bytes = (a < nb && b < nb) ? 4 * min(4, nb - b) : 0;
      cp_async16(&Rs[a][b], bytes ? R + (long long)(i + a) * d + i + b : R, bytes);
    }
  } else {
    for (int e = tid; e < 128 * 128; e += blockDim.x) {
      const int a = e >> 7, b = e & 127;
      const bool v = a < nb && b < nb;
      cp_async4(&Rs[a][b], v ? R + (long long)(i + a) * d + i + b : R, v);
    }
  }
  pdl_wait();
  pdl_release();
  if (vec) {
    for (int e = tid; e < kColCtaRows * 32; e += blockDim.x) {
      const int rr = e >> 5, t = (e & 31) * 4;
      const int gr = row0 + rr;
      const int bytes = (gr < m && t < nb) ? 4 * min(4, nb - t) : 0;
      cp_async16(&St[rr][t], bytes ? Wk + (long long)gr * d + i + t : Wk, bytes);
    }
  } else {
    for (int e = tid; e < kColCtaRows * 128; e += blockDim.x) {
      const int rr = e >> 7, t = e & 127;
      const int gr = row0 + rr;
      const bool v = gr < m && t < nb;
      cp_async4(&St[rr][t], v ? Wk + (long long)gr * d + i + t : Wk, v);
    }
  }
  for (int a = tid; a < 128; a += blockDim.x) gs[a] = (a < nb) ? gcol[i + a] : 0;
  cp_async_wait_all();
  __syncthreads();
  for (int a = tid; a < 128; a += blockDim.x) rinv[a] = (a < nb) ? 1.f / Rs[a][a] : 0.f;

  ColStepArgs args;
  args.Rs = Rs; args.gs = gs; args.rinv = rinv;
  args.scales = scales; args.zeros = zeros;
  args.srow = (long long)(active ? row : 0) * ng;
  args.q = q; args.src0 = lane & ~(unsigned)(kColLanes - 1);
  args.active = active;
  args.maxq = (float)maxq;
  args.D0 = 1.f; args.Z0 = 0.f; args.Y0 = 1.f;
  bool fast = true;
  if (UNIFORM && dyn == 128) {
    // dynamic group = this kernel block: its grid is fitted per row from the staged block,
    // which holds the current weights (zeros beyond nb leave the range, which contains 0, as is)
    float mn = 0.f, mx = 0.f;
#pragma unroll
    for (int sb = 0; sb < 128 / kColSub; ++sb) {
      const float4 v = *reinterpret_cast<const float4*>(&St[r][sb * kColSub + 4 * q]);
      mn = fminf(mn, fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
      mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
    row_range(mn, mx);
    float dlt, zz;
    fit_from_range(mn, mx, args.maxq, dlt, zz);
    args.D0 = dlt;
    args.Z0 = zz;
    args.Y0 = __frcp_rn(dlt);
    fast = quotient_fast(dlt);
    if (q == 0 && active) {
      scales[args.srow + i / 128] = dlt;
      zeros[args.srow + i / 128] = (int32_t)zz;
    }
  } else if (UNIFORM && dyn == kColSub) {
    fast = false;  // each sub-block fits its own grid inside the walk; Δ is divided by
  } else if (UNIFORM) {
    if (active) {
      args.D0 = scales[args.srow + gcol[i]];
      args.Z0 = (float)zeros[args.srow + gcol[i]];
      args.Y0 = __frcp_rn(args.D0);
      fast = quotient_fast(args.D0);
    }
  } else if (active) {
    for (int t = q; t < nb; t += kColLanes) fast &= quotient_fast(scales[args.srow + gcol[i + t]]);
  }
  fast = __syncthreads_and(fast);  // also publishes rinv and gs
  if (fast)
    col_walk<UNIFORM, true>(St, lossw, args, r, row, nb, d, i, ldE, vec, Wk, E, Ehi, Elo, codes,
                          dyn, ng, scales, zeros);
  else
    col_walk<UNIFORM, false>(St, lossw, args, r, row, nb, d, i, ldE, vec, Wk, E, Ehi, Elo, codes,
                          dyn, ng, scales, zeros);
  __syncthreads();
  // loss partial Σ_rows η² per column, the warps' sums in a fixed order
  for (int t = tid; t < nb; t += blockDim.x) {
    float sacc = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kColWarps; ++w8) sacc += lossw[w8][t];
    loss_part[(long long)blockIdx.x * d + i + t] = sacc;
  }
}

int column_block(Ctx* c, float* Wk, int m, int d, int i, int nb, const float* R, float* scales,
                 int32_t* zeros, int ng, const int32_t* gcol, bool uniform_grid, int dyn, int maxq,
                 float* E, float* Ehi, float* Elo, int ldE, uint8_t* codes, float* loss_part) {
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_colblock<true>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, kColSmem));
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_colblock<false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, kColSmem));
  const int blocks = (m + kColCtaRows - 1) / kColCtaRows;
  if (uniform_grid || dyn)
    GPTQ_LAUNCH(c, k_colblock<true>, blocks, 32 * kColWarps, kColSmem, Wk, m, d, i, nb, R, scales,
                zeros, ng, gcol, dyn, maxq, E, Ehi, Elo, ldE, codes, loss_part);
  else
    GPTQ_LAUNCH(c, k_colblock<false>, blocks, 32 * kColWarps, kColSmem, Wk, m, d, i, nb, R, scales,
                zeros, ng, gcol, 0, maxq, E, Ehi, Elo, ldE, codes, loss_part);
  return GPTQ_OK;
}

// ------------------------------------------------------------------------------------------
// a6: lazy update W[:, c0:c1] -= E[:, 0:k] R[i:i+k, c0:c1]  ([T] eq.(46)); fp32-accurate GEMM.
int trailing_update(Ctx* c, float* Wk, int m, int d, int i, int k, int c0, int c1,
                    const float* E, int ldE, const float* R) {
  const int n = c1 - c0;
  if (n <= 0 || k <= 0) return GPTQ_OK;
  int rc;
  GemmArgs g{m, n, k, E, ldE, 1, R + (long long)i * d + c0, d, 1, Wk + c0, d, -1.f, 1.f, 0};
  if ((rc = gemm_f32(c, g))) return rc;
  return GPTQ_OK;
}

// col_loss[j] = ½ Σ_parts Σ_rows η²  (= Σ_rows ρ² / (2 R_jj²), [T] eq.(43))
__global__ void k_loss_reduce(const float* __restrict__ part, int parts, int d,
                              float* __restrict__ out) {
  pdl_wait();
  pdl_release();
  int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  double s = 0.0;
  for (int p = 0; p < parts; ++p) s += (double)part[(long long)p * d + j];
  out[j] = (float)(0.5 * s);
}

int loss_reduce(Ctx* c, const float* loss_part, int parts, int d, float* loss_p) {
  GPTQ_LAUNCH(c, k_loss_reduce, (d + 255) / 256, 256, 0, loss_part, parts, d, loss_p);
  return GPTQ_OK;
}

// a7: back to original column order ([T] §10: undo the column permutation).  Grid: x over
// columns, y strided over rows.
__global__ void k_unpermute(long long m, int d, const int32_t* __restrict__ inv,
                            const uint8_t* __restrict__ codes_p, const float* __restrict__ Wk,
                            const float* __restrict__ loss_p, uint8_t* __restrict__ codes,
                            float* __restrict__ W_hat, float* __restrict__ col_loss) {
  pdl_wait();
  pdl_release();
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= d) return;
  const int src = inv[k];
  if (blockIdx.y == 0) col_loss[k] = loss_p[src];
  for (long long r = blockIdx.y; r < m; r += gridDim.y) {
    codes[r * d + k] = codes_p[r * d + src];
    W_hat[r * d + k] = Wk[r * d + src];
  }
}

int unpermute(Ctx* c, int m, int d, const int32_t* inv, const uint8_t* codes_p, const float* Wk,
              const float* loss_p, uint8_t* codes, float* W_hat, float* col_loss) {
  const int gx = (d + 255) / 256;
  const int gy = std::max(1, std::min(m, (c->num_sms * 16 + gx - 1) / gx));
  GPTQ_LAUNCH(c, k_unpermute, dim3(gx, gy), 256, 0, (long long)m, d, inv, codes_p, Wk, loss_p,
              codes, W_hat, col_loss);
  return GPTQ_OK;
}

}  // namespace gptq
