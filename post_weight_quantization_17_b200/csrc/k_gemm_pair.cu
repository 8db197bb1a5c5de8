// a6: the lazy trailing update W[:, T] -= E R[B, T] ([T] eq.(46)) on CTA pairs with operands
// already split for 3xTF32:
//   C[i, j] = alpha * sum_k A(i, k) B(k, j) + beta * C[i, j],   A = A_hi + A_lo, B = B_hi + B_lo
// with A [M, K] row-major (K contiguous) and B [K, N] row-major (N contiguous), each given as its
// tf32 halves hi = RN_tf32(x), lo = RN_tf32(x - hi) (the column kernel writes E's halves, a
// small kernel splits the super-block's slice of R).  The product is hi*hi + hi*lo + lo*hi:
// three tcgen05.mma.kind::tf32 per k-step (relative error ~2^-21 per product).
//
// Cluster of 2 (tcgen05 cta_group::2), 256 x 256 output tiles, M = N = 256, K = 8 per MMA.
// CTA r of the pair loads tile rows 128 r .. 128 r + 127 of A_hi and A_lo (K-major boxes of
// 128 x 32, 128-byte swizzle) and tile columns 128 r .. 128 r + 127 of B_hi and B_lo (four
// N-major boxes of 32 x 32 each, the 128-byte swizzle with 32-byte atoms that MN-major tf32
// operands need) into its own shared memory: 64 KB per 32-deep stage, 3 stages, no multicast.
// Both CTAs' copies complete on the leader's stage barrier, which the leader arms for both.
//   warp 0      both CTAs: TMA producer of its own halves
//   warp 1      leader (rank 0): MMA issuer; commits arrive on the barriers of both CTAs
//   warps 2..9  both CTAs: epilogue; TMEM partials of 128 k-elements are added in fp32 into a
//               row of 128 registers (the tensor core's own accumulation over many MMAs loses
//               low bits), then one read-modify-write of C per tile
// Every wait is bounded; a wait that runs out records GPTQ_ERR_TIMEOUT and the CTA unwinds;
// both CTAs pass a cluster barrier before TMEM is freed or either exits.
#include "kernels.h"
#include "tc_util.cuh"

#include <algorithm>

namespace gptq {

constexpr int GP_BK = 32, GP_STAGES = 3, GP_KBP = 4;     // 4 stages (128 k) per TMEM partial
constexpr int GP_BOX = 128 * GP_BK * 4;                   // 16 KB: one operand half per CTA
constexpr int GP_STAGE = 4 * GP_BOX;                      // A_hi, A_lo, B_hi, B_lo
constexpr int GP_SMEM = GP_STAGES * GP_STAGE + 1024 + 256;
constexpr int GP_EPI_WARPS = 8;
constexpr int GP_THREADS = 64 + 32 * GP_EPI_WARPS;

struct GemmPairParams {
  int M, N, K;
  float* C;
  long long ldc;
  float alpha, beta;
  int tiles_n, num_tiles;
  uint32_t idesc;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GP_THREADS, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmAh, const __grid_constant__ CUtensorMap tmAl,
                const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmBl,
                GemmPairParams p, DeviceStatus* st, long long budget) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + GP_STAGES * GP_STAGE);
  uint64_t* empty = full + GP_STAGES;
  uint64_t* tfull = empty + GP_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < GP_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], 2 * GP_EPI_WARPS);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmAh);
    tc::prefetch_tmap(&tmAl);
    tc::prefetch_tmap(&tmBh);
    tc::prefetch_tmap(&tmBl);
  }
  tc::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  if (warp == 1) tc::tmem_alloc_pair(tmem_slot, 512);
  tc::fence_before_sync();
  tc::cluster_sync();  // TMEM allocated in both CTAs before the leader's first MMA
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the previous kernel; its outputs are read only from here on
  pdl_wait();
  pdl_release();
  const int kblocks = (p.K + GP_BK - 1) / GP_BK;
  const int nparts = (kblocks + GP_KBP - 1) / GP_KBP;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[GP_STAGES] = {};
      uint32_t issued_phase[GP_STAGES] = {};
      const uint32_t leader_full = tc::map_to_rank(full, 0);
      for (int t = pair; t < p.num_tiles && !*abort_flag; t += npairs) {
        const int m0 = (t / p.tiles_n) * 256 + 128 * (int)rank;
        const int n0 = (t % p.tiles_n) * 256 + 128 * (int)rank;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait_cluster(&empty[stage], phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 31);
            *abort_flag = 1;
            break;
          }
          uint8_t* s0 = smem + stage * GP_STAGE;
          if (rank == 0) tc::mbar_expect_tx(&full[stage], 2 * GP_STAGE);
          const uint32_t bar = leader_full + 8u * stage;
          const int k0 = kb * GP_BK;
          tc::tma_load_2d_pair(s0, &tmAh, bar, k0, m0);
          tc::tma_load_2d_pair(s0 + GP_BOX, &tmAl, bar, k0, m0);
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            tc::tma_load_2d_pair(s0 + 2 * GP_BOX + a * (GP_BOX / 4), &tmBh, bar, n0 + 32 * a, k0);
            tc::tma_load_2d_pair(s0 + 3 * GP_BOX + a * (GP_BOX / 4), &tmBl, bar, n0 + 32 * a, k0);
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == GP_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: the leader's stage barriers count both CTAs' copies
      if (rank == 0)
        for (int s = 0; s < GP_STAGES; ++s)
          if (issued[s] && !tc::mbar_wait_cluster(&full[s], issued_phase[s], kDrainCycles))
            raise_error(st, GPTQ_ERR_TIMEOUT, 32);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any = false;
      for (int t = pair; t < p.num_tiles && ok && !*abort_flag; t += npairs) {
        for (int pp = 0; pp < nparts && ok; ++pp) {
          if (!tc::mbar_wait_cluster(&tempty[acc], acc_phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 33);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem + acc * 256;
          const int kb1 = min(kblocks, (pp + 1) * GP_KBP);
          for (int kb = pp * GP_KBP; kb < kb1; ++kb) {
            if (!tc::mbar_wait_cluster(&full[stage], phase, budget)) {
              raise_error(st, GPTQ_ERR_TIMEOUT, 34);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc::fence_after_sync();
            const uint32_t ah = tc::smem_u32(smem + stage * GP_STAGE);
            const uint32_t al = ah + GP_BOX, bh = ah + 2 * GP_BOX, bl = ah + 3 * GP_BOX;
#pragma unroll
            for (int kk = 0; kk < GP_BK / 8; ++kk) {
              const uint64_t dah = tc::sdesc_sw128(ah + kk * 32, 16, 1024);
              const uint64_t dal = tc::sdesc_sw128(al + kk * 32, 16, 1024);
              const uint64_t dbh = tc::sdesc_sw128_32b(bh + kk * 1024, GP_BOX / 4, 512);
              const uint64_t dbl = tc::sdesc_sw128_32b(bl + kk * 1024, GP_BOX / 4, 512);
              const uint32_t first = (kb == pp * GP_KBP && kk == 0) ? 0u : 1u;
              tc::mma_tf32_pair(d_tmem, dah, dbh, p.idesc, first);
              tc::mma_tf32_pair(d_tmem, dah, dbl, p.idesc, 1u);
              tc::mma_tf32_pair(d_tmem, dal, dbh, p.idesc, 1u);
            }
            any = true;
            tc::mma_commit_pair(&empty[stage]);
            if (++stage == GP_STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          tc::mma_commit_pair(&tfull[acc]);
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1;
          }
        }
      }
      if (any) {
        tc::mma_commit_pair(drain);
        if (!tc::mbar_wait(drain, 0, kDrainCycles)) raise_error(st, GPTQ_ERR_TIMEOUT, 35);
      }
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 and the 128-column half h
    const int q = warp & 3;
    const int h = (warp - 2) / 4;
    const int r = 32 * q + lane;
    const uint32_t leader_tempty = tc::map_to_rank(tempty, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = pair; t < p.num_tiles && ok && !*abort_flag; t += npairs) {
      float m[128];
#pragma unroll
      for (int u = 0; u < 128; ++u) m[u] = 0.f;
      for (int pp = 0; pp < nparts; ++pp) {
        if (!tc::mbar_wait_cluster_warp(&tfull[acc], acc_phase, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 36);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t base = tmem + acc * 256 + ((uint32_t)(32 * q) << 16) + h * 128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tc::tmem_ld32(base + cc * 32, v);
#pragma unroll
          for (int u = 0; u < 32; ++u) m[cc * 32 + u] += __uint_as_float(v[u]);
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            tc::mbar_arrive(&tempty[acc]);
          else
            tc::mbar_arrive_remote(leader_tempty + 8u * acc);
        }
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok) break;
      const int gi = (t / p.tiles_n) * 256 + 128 * (int)rank + r;
      if (gi < p.M) {
        float* crow = p.C + (long long)gi * p.ldc;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int gj0 = (t % p.tiles_n) * 256 + h * 128 + cc * 32;
          if (gj0 >= p.N) continue;
          float4* c4 = reinterpret_cast<float4*>(crow + gj0);
          if (gj0 + 32 <= p.N && ((reinterpret_cast<uintptr_t>(c4) & 15) == 0)) {
            float4 o[8];
            if (p.beta != 0.f) {
#pragma unroll
              for (int u = 0; u < 8; ++u) o[u] = c4[u];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int e = cc * 32 + 4 * u;
              float4 y = make_float4(p.alpha * m[e], p.alpha * m[e + 1], p.alpha * m[e + 2],
                                     p.alpha * m[e + 3]);
              if (p.beta != 0.f) {
                y.x = fmaf(p.beta, o[u].x, y.x); y.y = fmaf(p.beta, o[u].y, y.y);
                y.z = fmaf(p.beta, o[u].z, y.z); y.w = fmaf(p.beta, o[u].w, y.w);
              }
              c4[u] = y;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int gj = gj0 + u;
              if (gj < p.N) {
                const float y = p.alpha * m[cc * 32 + u];
                crow[gj] = (p.beta == 0.f) ? y : fmaf(p.beta, crow[gj], y);
              }
            }
          }
        }
      }
    }
  }
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  tc::cluster_sync();  // no CTA frees TMEM or leaves while its pair may still touch it
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, 512);
  }
}

// x -> (hi, lo) for a rows x cols block (row strides lds, ldd)
__global__ void k_split_tf32(const float* __restrict__ src, long long lds, int rows, int cols,
                             float* __restrict__ hi, float* __restrict__ lo, long long ldd) {
  pdl_wait();
  pdl_release();
  const long long total = (long long)rows * cols;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(e / cols), c = (int)(e - (long long)r * cols);
    const float x = src[r * lds + c];
    const float h = tc::tf32_rna(x);
    hi[r * ldd + c] = h;
    lo[r * ldd + c] = tc::tf32_rna(x - h);
  }
}

int split_tf32(Ctx* c, const float* src, long long lds, int rows, int cols, float* hi, float* lo,
               long long ldd) {
  const long long total = (long long)rows * cols;
  if (total <= 0) return GPTQ_OK;
  const int blocks = (int)std::min<long long>((total + 255) / 256, (long long)c->num_sms * 8);
  GPTQ_LAUNCH(c, k_split_tf32, blocks, 256, 0, src, lds, rows, cols, hi, lo, ldd);
  return GPTQ_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 pair_encode() {
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

static bool pair_map(CUtensorMap* map, const float* base, long long inner, long long outer,
                     long long ld, int box_inner, int box_outer, CUtensorMapSwizzle swz) {
  auto enc = pair_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
             box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemm_pair_applies(int M, int N, int K, const float* Ah, long long lda, const float* Bh,
                       long long ldb, int num_sms) {
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  return num_sms >= 2 && M >= 256 && N >= 128 && K >= GP_BK && lda % 4 == 0 && ldb % 4 == 0 &&
         al(Ah) && al(Bh);
}

int gemm_pair(Ctx* c, int M, int N, int K, const float* Ah, const float* Al, long long lda,
              const float* Bh, const float* Bl, long long ldb, float* C, long long ldc, float alpha,
              float beta) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  CUtensorMap mah, mal, mbh, mbl;
  const bool ok = pair_map(&mah, Ah, K, M, lda, GP_BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  pair_map(&mal, Al, K, M, lda, GP_BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
                  pair_map(&mbh, Bh, N, K, ldb, 32, GP_BK, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) &&
                  pair_map(&mbl, Bl, N, K, ldb, 32, GP_BK, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
  if (!ok) GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "pair GEMM: tensor map encoding failed");
  GemmPairParams p;
  p.M = M; p.N = N; p.K = K;
  p.C = C; p.ldc = ldc; p.alpha = alpha; p.beta = beta;
  p.tiles_n = (N + 255) / 256;
  p.num_tiles = p.tiles_n * ((M + 255) / 256);
  p.idesc = tc::idesc_f32acc(2u, false, true, 256, 256);
  const int npairs = std::min(p.num_tiles, c->num_sms / 2);
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_gemm_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          GP_SMEM));
  // CTA pairs keep the default wait budget (a pair whose CTAs gave up at different stages could
  // not drain every copy completing on the leader's barriers)
  GPTQ_LAUNCH(c, k_gemm_pair, 2 * npairs, GP_THREADS, GP_SMEM, mah, mal, mbh, mbl, p, c->status,
              kDefaultWaitCycles);
  return GPTQ_OK;
}

}  // namespace gptq
