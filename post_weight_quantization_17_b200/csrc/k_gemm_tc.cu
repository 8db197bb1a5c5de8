// fp32-accurate GEMM on the 5th-generation tensor cores:
//   C[i, j] = alpha * sum_k A[i, k] B(k, j) + beta * C[i, j]
// A is [M, K] row-major (K contiguous); B is either [N, K] row-major ("K-major") or [K, N]
// row-major ("N-major").  Used by the factorization recursion and the lazy trailing update
// W[:, T] -= E R[B, T] ([T] eq.(46)).
//
// Each fp32 operand x is split as hi = tf32(x), lo = tf32(x - hi) (round to nearest) and the
// product is hi*hi + hi*lo + lo*hi: three tcgen05.mma.kind::tf32 per k-step into one TMEM
// accumulator (relative error ~2^-21 per product, against 2^-11 for plain TF32; clearing the
// low bits instead of rounding would double the error that the factorization's conditioning
// then amplifies).  The tensor
// core rounds its fp32 accumulator toward zero at every MMA, so partial sums of kp k-elements
// (128 by default, 32 in the factorization) are taken from TMEM and added in fp32 into a
// register accumulator by the epilogue warps.
//   warp 0       TMA producer: A box 128 x 32, B box 128 x 32 (K-major) or 4 x (32 x 32)
//                (N-major), 128-byte swizzle (32-byte atoms for the N-major tf32 operand, the
//                only smem layout the tensor core takes for it), 3-stage ring
//   warps 2..5   split: tf32 hi in place, lo into its own buffer (same swizzled layout),
//                then fence.proxy.async so the tensor core sees the writes
//   warp 1       MMA issuer, M = N = 128, K = 8 per instruction, two TMEM accumulators
//   warps 6..13  epilogue: TMEM -> registers (+= per partial) -> C
// Triangular-structure flags restrict each tile's k-range (the skipped values are zeros in
// memory, so rounding the range out to whole 32-element slabs is harmless).  Every wait is
// bounded (GPTQ_ERR_TIMEOUT, then the CTA drains its copies and frees TMEM).
#include "kernels.h"
#include "gemm_simt.cuh"
#include "tc_util.cuh"

namespace gptq {

constexpr int GT_BM = 128, GT_BN = 128, GT_BK = 32, GT_STAGES = 3;
constexpr int GT_TILE_BYTES = GT_BM * GT_BK * 4;  // 16 KB: one fp32 operand tile
constexpr int GT_STAGE_BYTES = 4 * GT_TILE_BYTES;  // A hi, A lo, B hi, B lo
constexpr int GT_SMEM = GT_STAGES * GT_STAGE_BYTES + 1024 + 256;
constexpr int GT_CONV_WARPS = 4, GT_EPI_WARPS = 8;
constexpr int GT_THREADS = 32 * (2 + GT_CONV_WARPS + GT_EPI_WARPS);

struct GemmTcParams {
  int M, N, K;
  float* C;
  long long ldc;
  float alpha, beta;
  int flags;
  int b_nmajor;
  int tiles_m, tiles_n, num_tiles;
  int kp;  // k-elements per TMEM partial
  uint32_t idesc;
};

// Tiles are visited in groups of GT_GROUP tile rows, column by column inside a group, so that
// the ~148 tiles of one wave form a near-square block (16 rows x ~9 columns) and share their A
// row slabs and B column slabs through L2; in plain row-major order a wave of a wide product
// spans one tile row and ~148 columns, and every B slab then streams from HBM.
constexpr int GT_GROUP = 16;

__device__ __forceinline__ bool gt_tile(const GemmTcParams& p, int t, int& i0, int& j0, int& kbeg,
                                        int& kend) {
  const int group = t / (GT_GROUP * p.tiles_n);
  const int first = group * GT_GROUP;
  const int rows = min(GT_GROUP, p.tiles_m - first);
  const int local = t - group * GT_GROUP * p.tiles_n;
  i0 = (first + local % rows) * GT_BM;
  j0 = (local / rows) * GT_BN;
  if ((p.flags & kCUpper) && i0 > j0 + GT_BN - 1) return false;
  if ((p.flags & kCLower) && j0 > i0 + GT_BM - 1) return false;
  kbeg = 0;
  kend = p.K;
  if (p.flags & kAUpper) kbeg = max(kbeg, i0);
  if (p.flags & kBLower) kbeg = max(kbeg, j0);
  if (p.flags & kALower) kend = min(kend, i0 + GT_BM);
  if (p.flags & kBUpper) kend = min(kend, j0 + GT_BN);
  kbeg = kbeg / GT_BK * GT_BK;
  return true;
}

__global__ void __launch_bounds__(GT_THREADS, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              GemmTcParams p, DeviceStatus* st, long long budget) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + GT_STAGES * GT_STAGE_BYTES);
  uint64_t* conv = full + GT_STAGES;
  uint64_t* empty = conv + GT_STAGES;
  uint64_t* tfull = empty + GT_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < GT_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&conv[s], 32 * GT_CONV_WARPS);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], 32 * GT_EPI_WARPS);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmA);
    tc::prefetch_tmap(&tmB);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the previous kernel; its outputs are read only from here on
  pdl_wait();
  pdl_release();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[GT_STAGES] = {};
      uint32_t issued_phase[GT_STAGES] = {};
      for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
        int i0, j0, kbeg, kend;
        if (!gt_tile(p, t, i0, j0, kbeg, kend)) continue;
        for (int k0 = kbeg; k0 < kend; k0 += GT_BK) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 11);
            *abort_flag = 1;
            break;
          }
          uint8_t* sA = smem + stage * GT_STAGE_BYTES;
          uint8_t* sB = sA + 2 * GT_TILE_BYTES;
          tc::mbar_expect_tx(&full[stage], 2 * GT_TILE_BYTES);
          tc::tma_load_2d(sA, &tmA, &full[stage], k0, i0);
          if (p.b_nmajor) {
#pragma unroll
            for (int a = 0; a < GT_BN / 32; ++a)
              tc::tma_load_2d(sB + a * (GT_TILE_BYTES / 4), &tmB, &full[stage], j0 + 32 * a, k0);
          } else {
            tc::tma_load_2d(sB, &tmB, &full[stage], k0, j0);
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == GT_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int s = 0; s < GT_STAGES; ++s)
        if (issued[s] && !tc::mbar_wait(&full[s], issued_phase[s], kDrainCycles))
          raise_error(st, GPTQ_ERR_TIMEOUT, 12);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any = false;
      for (int t = blockIdx.x; t < p.num_tiles && ok && !*abort_flag; t += gridDim.x) {
        int i0, j0, kbeg, kend;
        if (!gt_tile(p, t, i0, j0, kbeg, kend)) continue;
        for (int kp = kbeg; kp < kend && ok; kp += p.kp) {
          if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 13);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem + acc * GT_BN;
          const int kp1 = min(kend, kp + p.kp);
          for (int k0 = kp; k0 < kp1; k0 += GT_BK) {
            if (!tc::mbar_wait(&conv[stage], phase, budget)) {
              raise_error(st, GPTQ_ERR_TIMEOUT, 14);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc::fence_after_sync();
            const uint32_t ahi = tc::smem_u32(smem + stage * GT_STAGE_BYTES);
            const uint32_t alo = ahi + GT_TILE_BYTES;
            const uint32_t bhi = ahi + 2 * GT_TILE_BYTES;
            const uint32_t blo = ahi + 3 * GT_TILE_BYTES;
#pragma unroll
            for (int kk = 0; kk < GT_BK / 8; ++kk) {
              const uint64_t dah = tc::sdesc_sw128(ahi + kk * 32, 16, 1024);
              const uint64_t dal = tc::sdesc_sw128(alo + kk * 32, 16, 1024);
              uint64_t dbh, dbl;
              if (p.b_nmajor) {
                // MN-major tf32: 32-element atoms along N every 4 KB, 4-row K atoms of 512 B
                dbh = tc::sdesc_sw128_32b(bhi + kk * 1024, GT_TILE_BYTES / 4, 512);
                dbl = tc::sdesc_sw128_32b(blo + kk * 1024, GT_TILE_BYTES / 4, 512);
              } else {
                dbh = tc::sdesc_sw128(bhi + kk * 32, 16, 1024);
                dbl = tc::sdesc_sw128(blo + kk * 32, 16, 1024);
              }
              const uint32_t first = (k0 == kp && kk == 0) ? 0u : 1u;
              tc::mma_tf32(d_tmem, dah, dbh, p.idesc, first);
              tc::mma_tf32(d_tmem, dah, dbl, p.idesc, 1u);
              tc::mma_tf32(d_tmem, dal, dbh, p.idesc, 1u);
            }
            any = true;
            tc::mma_commit(&empty[stage]);
            if (++stage == GT_STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          tc::mma_commit(&tfull[acc]);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1;
          }
        }
      }
      // every MMA has completed before TMEM is freed (after an abort the epilogue may not have
      // waited for them)
      if (any) {
        tc::mma_commit(drain);
        if (!tc::mbar_wait(drain, 0, kDrainCycles)) raise_error(st, GPTQ_ERR_TIMEOUT, 16);
      }
    }
  } else if (warp < 2 + GT_CONV_WARPS) {
    // ---------------------------------------------------------------- tf32 hi / lo split
    const int ct = threadIdx.x - 64;  // 0 .. 127
    int stage = 0;
    uint32_t phase = 0;
    for (int t = blockIdx.x; t < p.num_tiles && !*abort_flag; t += gridDim.x) {
      int i0, j0, kbeg, kend;
      if (!gt_tile(p, t, i0, j0, kbeg, kend)) continue;
      bool ok = true;
      for (int k0 = kbeg; k0 < kend; k0 += GT_BK) {
        if (!tc::mbar_wait(&full[stage], phase, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 15);
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* base = smem + stage * GT_STAGE_BYTES;
#pragma unroll
        for (int op = 0; op < 2; ++op) {
          float4* hi = reinterpret_cast<float4*>(base + op * 2 * GT_TILE_BYTES);
          float4* lo = reinterpret_cast<float4*>(base + op * 2 * GT_TILE_BYTES + GT_TILE_BYTES);
#pragma unroll 4
          for (int c = ct; c < GT_TILE_BYTES / 16; c += 32 * GT_CONV_WARPS) {
            const float4 x = hi[c];
            float4 h, l;
            h.x = tc::tf32_rna(x.x);
            h.y = tc::tf32_rna(x.y);
            h.z = tc::tf32_rna(x.z);
            h.w = tc::tf32_rna(x.w);
            l.x = tc::tf32_rna(x.x - h.x);
            l.y = tc::tf32_rna(x.y - h.y);
            l.z = tc::tf32_rna(x.z - h.z);
            l.w = tc::tf32_rna(x.w - h.w);
            hi[c] = h;
            lo[c] = l;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc::mbar_arrive(&conv[stage]);
        if (++stage == GT_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int h = (warp - 2 - GT_CONV_WARPS) / 4;  // column half
    const int r = 32 * q + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok && !*abort_flag; t += gridDim.x) {
      int i0, j0, kbeg, kend;
      if (!gt_tile(p, t, i0, j0, kbeg, kend)) continue;
      float m[64];
#pragma unroll
      for (int u = 0; u < 64; ++u) m[u] = 0.f;
      for (int kp = kbeg; kp < kend; kp += p.kp) {
        if (!tc::mbar_wait_warp(&tfull[acc], acc_phase, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 17);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t base = tmem + acc * GT_BN + ((uint32_t)(32 * q) << 16) + h * 64;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t v[32];
          tc::tmem_ld32(base + cc * 32, v);
#pragma unroll
          for (int u = 0; u < 32; ++u) m[cc * 32 + u] += __uint_as_float(v[u]);
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&tempty[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok) break;
      const int gi = i0 + r;
      if (gi < p.M) {
        float* crow = p.C + (long long)gi * p.ldc;
        const int jb = j0 + h * 64;
        const bool vec = (jb + 64 <= p.N) && ((reinterpret_cast<uintptr_t>(crow + jb) & 15) == 0);
        if (vec) {
          float4* c4 = reinterpret_cast<float4*>(crow + jb);
          // C is read in batches of eight float4 before any store, so that the loads overlap
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            float4 o[8];
            if (p.beta != 0.f) {
#pragma unroll
              for (int u = 0; u < 8; ++u) o[u] = c4[8 * hb + u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int e = 4 * (8 * hb + u);
              float4 v = make_float4(p.alpha * m[e], p.alpha * m[e + 1], p.alpha * m[e + 2],
                                     p.alpha * m[e + 3]);
              if (p.beta != 0.f) {
                v.x = fmaf(p.beta, o[u].x, v.x); v.y = fmaf(p.beta, o[u].y, v.y);
                v.z = fmaf(p.beta, o[u].z, v.z); v.w = fmaf(p.beta, o[u].w, v.w);
              }
              c4[8 * hb + u] = v;
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < 64; ++u) {
            const int gj = jb + u;
            if (gj < p.N) {
              const float v = p.alpha * m[u];
              crow[gj] = (p.beta == 0.f) ? v : fmaf(p.beta, crow[gj], v);
            }
          }
        }
      }
    }
  }
  // the producer and MMA roles run on one lane of their warps: reconverge every warp before the
  // CTA barrier, so that TMEM is released only after the epilogue has read it
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

static bool make_map_f32(CUtensorMap* map, const void* base, long long inner, long long outer,
                         long long ld, int box_inner, int box_outer, CUtensorMapSwizzle swz) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// The tensor path takes fp32 operands whose rows are 16-byte aligned (TMA) and shapes of at
// least one tile; A must be K-contiguous and B either K- or N-contiguous.
bool gemm_tc_applies(const GemmArgs& g) {
  auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (g.sak != 1 || g.sai % 4 != 0 || !al(g.A)) return false;
  const bool bk = (g.sbk == 1), bn = (g.sbj == 1);
  if (!(bk || bn)) return false;
  const long long ldb = bk ? g.sbj : g.sbk;
  if (ldb % 4 != 0 || !al(g.B)) return false;
  return g.M >= 64 && g.N >= 64 && g.K >= 32;
}

int gemm_tc(Ctx* c, const GemmArgs& g) {
  CUtensorMap ma, mb;
  const bool b_nmajor = (g.sbj == 1) && (g.sbk != 1);
  if (!make_map_f32(&ma, g.A, g.K, g.M, g.sai, GT_BK, GT_BM, CU_TENSOR_MAP_SWIZZLE_128B))
    GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "tensor map for A failed");
  const bool okb =
      b_nmajor ? make_map_f32(&mb, g.B, g.N, g.K, g.sbk, 32, GT_BK,
                              CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)
               : make_map_f32(&mb, g.B, g.K, g.N, g.sbj, GT_BK, GT_BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!okb) GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "tensor map for B failed");
  GemmTcParams p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.C = g.C; p.ldc = g.ldc; p.alpha = g.alpha; p.beta = g.beta; p.flags = g.flags;
  p.b_nmajor = b_nmajor ? 1 : 0;
  p.tiles_n = (g.N + GT_BN - 1) / GT_BN;
  p.tiles_m = (g.M + GT_BM - 1) / GT_BM;
  p.num_tiles = p.tiles_n * p.tiles_m;
  p.kp = g.partial_k > 0 ? std::max(GT_BK, g.partial_k / GT_BK * GT_BK) : 128;
  p.idesc = tc::idesc_f32acc(2u, false, b_nmajor, GT_BM, GT_BN);
  const int grid = std::min(p.num_tiles, c->num_sms);
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          GT_SMEM));
  GPTQ_LAUNCH(c, k_gemm_tc, grid, GT_THREADS, GT_SMEM, ma, mb, p, c->status, c->timeout_cycles);
  return GPTQ_OK;
}

// fp32 GEMM entry used by the factorization and the trailing update: small products on CUDA
// cores with small tiles, tensor cores where the operands allow TMA, CUDA cores otherwise.
int gemm_f32(Ctx* c, const GemmArgs& g) {
  if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
  if (g.M <= kSmallGemmSide && g.N <= kSmallGemmSide) return gemm_small(c, g);
  if (gemm_tc_applies(g)) return gemm_tc(c, g);
  return gemm_simt(c, g);
}

}  // namespace gptq
