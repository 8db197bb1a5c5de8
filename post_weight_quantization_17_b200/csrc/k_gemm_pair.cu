// fp32-accurate GEMM on CTA pairs with operands already split for 3xTF32:
//   C[i, j] = alpha * sum_k A(i, k) B(k, j) + beta * C[i, j],   A = A_hi + A_lo, B = B_hi + B_lo
// with A [M, K] row-major (K contiguous) and B either [K, N] row-major (N contiguous) or given
// K-major (B(k, j) = Bmem[j ldb + k], e.g. the transpose of a row-major matrix), each as its tf32
// halves hi = RN_tf32(x), lo = RN_tf32(x - hi).  The product is hi*hi + hi*lo + lo*hi: three
// tcgen05.mma.kind::tf32 per k-step (relative error ~2^-21 per product).  It serves
//   a6  the lazy trailing update W[:, T] -= E R[B, T] ([T] eq.(46)), E's halves from the column
//       kernel, R's slice split by k_split_tf32;
//   a3  the factorization's large products ([T] eq.(37)-(40) by block recursion), whose zero
//       triangles are skipped by k-range flags, whose symmetric update computes only the tiles
//       that touch the upper triangle, and whose temporaries (U12, T2) are written directly as
//       tf32 halves for the next product (split output).
//
// Cluster of 2 (tcgen05 cta_group::2), 256 x 256 output tiles, M = N = 256, K = 8 per MMA.
// CTA r of the pair loads tile rows 128 r .. 128 r + 127 of A_hi and A_lo (K-major boxes of
// 128 x 32, 128-byte swizzle) and tile columns 128 r .. 128 r + 127 of B_hi and B_lo (N-major:
// four boxes of 32 x 32 each in the 128-byte swizzle with 32-byte atoms that MN-major tf32
// operands need; K-major: one box of 128 x 32 like A) into its own shared memory: 64 KB per
// 32-deep stage, 3 stages, no multicast.  Both CTAs' copies complete on the leader's stage
// barrier, which the leader arms for both.
//   warp 0      both CTAs: TMA producer of its own halves
//   warp 1      leader (rank 0): MMA issuer; commits arrive on the barriers of both CTAs
//   warps 2..9  both CTAs: epilogue; TMEM partials of 32 kbp k-elements are added in fp32 into a
//               row of 128 registers (the tensor core's own accumulation over many MMAs loses
//               low bits), then one read-modify-write of C (or the split write) per tile
// Every wait is bounded; a wait that runs out records GPTQ_ERR_TIMEOUT and the CTA unwinds;
// both CTAs pass a cluster barrier before TMEM is freed or either exits.
#include "kernels.h"
#include "gemm_simt.cuh"
#include "tc_util.cuh"
#include "tile_upper.h"

#include <algorithm>

namespace gptq {

constexpr int GP_BK = 32, GP_STAGES = 3;
constexpr int GP_BOX = 128 * GP_BK * 4;                   // 16 KB: one operand half per CTA
constexpr int GP_STAGE = 4 * GP_BOX;                      // A_hi, A_lo, B_hi, B_lo
constexpr int GP_SMEM = GP_STAGES * GP_STAGE + 1024 + 256;
constexpr int GP_EPI_WARPS = 8;
constexpr int GP_THREADS = 64 + 32 * GP_EPI_WARPS;

struct GemmPairParams {
  int M, N, K;
  float* C;              // beta / output (row-major, ldc), unless the split output is given
  float* Ch;             // split output: tf32 halves of alpha A B + beta C (same ldc), or null
  float* Cl;
  long long ldc;
  float alpha, beta;
  int flags;             // kAUpper / kALower / kBUpper / kBLower (k-ranges), kCUpper (tiles)
  int b_kmajor;
  int vec;               // C (or Ch and Cl) and ldc allow 16-byte row segments
  int kbp;               // 32-deep stages per TMEM partial
  int tiles_m, tiles_n, num_tiles;
  uint32_t idesc;
};

// Tile t -> (tile row, tile column), in groups of GP_GROUP tile rows walked column by column, so
// that the 74 tiles of one wave form a near-square block (8 x ~9) and share operand slabs through
// L2 (row-major order would give each tile of a wave its own B slab).
// A product computed only where C touches the upper triangle (kCUpper) enumerates just those
// tiles, in the same grouped order (tile_upper.h).
constexpr int GP_GROUP = 8;
__device__ __forceinline__ void gp_tile(const GemmPairParams& p, int t, int& tm, int& tn) {
  if (p.flags & kCUpper) {
    upper_tile(p.tiles_m, p.tiles_n, GP_GROUP, t, tm, tn);
    return;
  }
  const int group = t / (GP_GROUP * p.tiles_n);
  const int first = group * GP_GROUP;
  const int rows = min(GP_GROUP, p.tiles_m - first);
  const int local = t - group * GP_GROUP * p.tiles_n;
  tm = first + local % rows;
  tn = local / rows;
}

// The tile's coordinates and its range of 32-deep k-blocks [kb0, kb1) after the structure flags
// (the values the flags exclude are zeros in memory, so rounding the range out to whole blocks is
// harmless); false for a tile that kCUpper skips.  Every role calls this with the same arguments.
// The blocks are walked from the end of the range when only its start depends on the tile
// (kBLower, kAUpper): the tiles of a wave then all begin at the same k-slab and keep walking it in
// step, so each slab they share is fetched from HBM once and served to the rest from L2.
__device__ __forceinline__ bool gp_tile_range(const GemmPairParams& p, int t, int& tm, int& tn,
                                              int& kb0, int& kb1) {
  gp_tile(p, t, tm, tn);
  const int i0 = tm * 256, j0 = tn * 256;
  if ((p.flags & kCUpper) && i0 > j0 + 255) return false;
  int kbeg = 0, kend = p.K;
  if (p.flags & kAUpper) kbeg = max(kbeg, i0);
  if (p.flags & kBLower) kbeg = max(kbeg, j0);
  if (p.flags & kALower) kend = min(kend, i0 + 256);
  if (p.flags & kBUpper) kend = min(kend, j0 + 256);
  kb0 = kbeg / GP_BK;
  kb1 = max(kb0, (kend + GP_BK - 1) / GP_BK);
  return true;
}
__device__ __forceinline__ bool gp_reverse(const GemmPairParams& p) {
  return (p.flags & (kBLower | kAUpper)) && !(p.flags & (kBUpper | kALower));
}
// the s-th k-block of a tile's walk
__device__ __forceinline__ int gp_kb(bool rev, int kb0, int kb1, int s) {
  return rev ? kb1 - 1 - s : kb0 + s;
}

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

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[GP_STAGES] = {};
      uint32_t issued_phase[GP_STAGES] = {};
      const uint32_t leader_full = tc::map_to_rank(full, 0);
      for (int t = pair; t < p.num_tiles && !*abort_flag; t += npairs) {
        int tm, tn, kb0, kb1;
        if (!gp_tile_range(p, t, tm, tn, kb0, kb1)) continue;
        const int m0 = tm * 256 + 128 * (int)rank;
        const int n0 = tn * 256 + 128 * (int)rank;
        const bool rev = gp_reverse(p);
        for (int s = 0; s < kb1 - kb0; ++s) {
          const int kb = gp_kb(rev, kb0, kb1, s);
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
          if (p.b_kmajor) {
            tc::tma_load_2d_pair(s0 + 2 * GP_BOX, &tmBh, bar, k0, n0);
            tc::tma_load_2d_pair(s0 + 3 * GP_BOX, &tmBl, bar, k0, n0);
          } else {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              tc::tma_load_2d_pair(s0 + 2 * GP_BOX + a * (GP_BOX / 4), &tmBh, bar, n0 + 32 * a, k0);
              tc::tma_load_2d_pair(s0 + 3 * GP_BOX + a * (GP_BOX / 4), &tmBl, bar, n0 + 32 * a, k0);
            }
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
        int tm, tn, kb0, kb1;
        if (!gp_tile_range(p, t, tm, tn, kb0, kb1)) continue;
        const int nparts = (kb1 - kb0 + p.kbp - 1) / p.kbp;
        for (int pp = 0; pp < nparts && ok; ++pp) {
          if (!tc::mbar_wait_cluster(&tempty[acc], acc_phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 33);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem + acc * 256;
          const int se = min(kb1 - kb0, (pp + 1) * p.kbp);
          for (int s = pp * p.kbp; s < se; ++s) {   // the k-block gp_kb(..., s) of the tile
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
              // K-major B is laid out like A; N-major B in 32-column atoms every 4 KB
              const uint64_t dbh = p.b_kmajor ? tc::sdesc_sw128(bh + kk * 32, 16, 1024)
                                              : tc::sdesc_sw128_32b(bh + kk * 1024, GP_BOX / 4, 512);
              const uint64_t dbl = p.b_kmajor ? tc::sdesc_sw128(bl + kk * 32, 16, 1024)
                                              : tc::sdesc_sw128_32b(bl + kk * 1024, GP_BOX / 4, 512);
              const uint32_t first = (s == pp * p.kbp && kk == 0) ? 0u : 1u;
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
      int tm, tn, kb0, kb1;
      if (!gp_tile_range(p, t, tm, tn, kb0, kb1)) continue;
      const int nparts = (kb1 - kb0 + p.kbp - 1) / p.kbp;
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
        // two 32-column loads in flight per wait: half the TMEM round trips of one per load
#pragma unroll
        for (int cc = 0; cc < 4; cc += 2) {
          uint32_t v[32], w[32];
          tc::tmem_ld32_async(base + cc * 32, v);
          tc::tmem_ld32_async(base + cc * 32 + 32, w);
          tc::tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            m[cc * 32 + u] += __uint_as_float(v[u]);
            m[cc * 32 + 32 + u] += __uint_as_float(w[u]);
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            tc::mbar_arrive_relaxed(&tempty[acc]);
          else
            tc::mbar_arrive_remote_relaxed(leader_tempty + 8u * acc);
        }
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok) break;
      const int gi = tm * 256 + 128 * (int)rank + r;
      if (gi < p.M) {
        // y = alpha m + beta C written to C, or (beta = 0) alpha m split into tf32 halves and
        // written to Ch / Cl
        const long long roff = (long long)gi * p.ldc;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int gj0 = tn * 256 + h * 128 + cc * 32;
          if (gj0 >= p.N) continue;
          if (p.vec && gj0 + 32 <= p.N) {
            if (p.Ch) {
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const int e = cc * 32 + 4 * u;
                const float4 y = make_float4(p.alpha * m[e], p.alpha * m[e + 1],
                                             p.alpha * m[e + 2], p.alpha * m[e + 3]);
                const float4 hi = make_float4(tc::tf32_rna(y.x), tc::tf32_rna(y.y),
                                              tc::tf32_rna(y.z), tc::tf32_rna(y.w));
                reinterpret_cast<float4*>(p.Ch + roff + gj0)[u] = hi;
                reinterpret_cast<float4*>(p.Cl + roff + gj0)[u] =
                    make_float4(tc::tf32_rna(y.x - hi.x), tc::tf32_rna(y.y - hi.y),
                                tc::tf32_rna(y.z - hi.z), tc::tf32_rna(y.w - hi.w));
              }
            } else {
              float4* c4 = reinterpret_cast<float4*>(p.C + roff + gj0);
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
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int gj = gj0 + u;
              if (gj < p.N) {
                const float y = p.alpha * m[cc * 32 + u];
                if (p.Ch) {
                  const float hi = tc::tf32_rna(y);
                  p.Ch[roff + gj] = hi;
                  p.Cl[roff + gj] = tc::tf32_rna(y - hi);
                } else {
                  p.C[roff + gj] = (p.beta == 0.f) ? y : fmaf(p.beta, p.C[roff + gj], y);
                }
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

// x -> (hi, lo) for a rows x cols block (row strides lds, ldd); with upper set, the halves of
// the elements below the block's diagonal (column < row) are written as zeros whatever src holds.
// Grid: x over 1024-column slices of a row (256 threads, 4 columns each), y over rows
// (grid-strided); 16-byte accesses when the block's rows are 16-byte aligned.
__global__ void k_split_tf32(const float* __restrict__ src, long long lds, int rows, int cols,
                             float* __restrict__ hi, float* __restrict__ lo, long long ldd,
                             int vec, int upper) {
  pdl_wait();
  pdl_release();
  const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (c0 >= cols) return;
  for (int r = blockIdx.y; r < rows; r += gridDim.y) {
    const float* s = src + (long long)r * lds + c0;
    float* h = hi + (long long)r * ldd + c0;
    float* l = lo + (long long)r * ldd + c0;
    if (vec && c0 + 4 <= cols) {
      float4 x = *reinterpret_cast<const float4*>(s);
      if (upper && c0 < r) {
        x.x = 0.f;
        if (c0 + 1 < r) x.y = 0.f;
        if (c0 + 2 < r) x.z = 0.f;
        if (c0 + 3 < r) x.w = 0.f;
      }
      const float4 xh = make_float4(tc::tf32_rna(x.x), tc::tf32_rna(x.y), tc::tf32_rna(x.z),
                                    tc::tf32_rna(x.w));
      *reinterpret_cast<float4*>(h) = xh;
      *reinterpret_cast<float4*>(l) =
          make_float4(tc::tf32_rna(x.x - xh.x), tc::tf32_rna(x.y - xh.y),
                      tc::tf32_rna(x.z - xh.z), tc::tf32_rna(x.w - xh.w));
    } else {
      for (int u = 0; u < 4 && c0 + u < cols; ++u) {
        const float x = (upper && c0 + u < r) ? 0.f : s[u];
        const float xh = tc::tf32_rna(x);
        h[u] = xh;
        l[u] = tc::tf32_rna(x - xh);
      }
    }
  }
}

int split_tf32(Ctx* c, const float* src, long long lds, int rows, int cols, float* hi, float* lo,
               long long ldd, bool upper) {
  if (rows <= 0 || cols <= 0) return GPTQ_OK;
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  const int vec = (lds % 4 == 0) && (ldd % 4 == 0) && al(src) && al(hi) && al(lo);
  const int gx = (cols + 1023) / 1024;
  const int gy = std::min(rows, std::max(1, c->num_sms * 16 / gx));
  GPTQ_LAUNCH(c, k_split_tf32, dim3(gx, gy), 256, 0, src, lds, rows, cols, hi, lo, ldd, vec,
              upper ? 1 : 0);
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

int gemm_pair(Ctx* c, const GemmPairArgs& g) {
  if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  if (!al(g.Ah) || !al(g.Al) || !al(g.Bh) || !al(g.Bl) || g.lda % 4 || g.ldb % 4 || g.K < 1 ||
      (g.Ch && (!g.Cl || g.beta != 0.f)) || (!g.Ch && !g.C))
    GPTQ_SET_ERR(c, GPTQ_ERR_ARG, "pair GEMM: bad operands");
  CUtensorMap mah, mal, mbh, mbl;
  bool ok = pair_map(&mah, g.Ah, g.K, g.M, g.lda, GP_BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
            pair_map(&mal, g.Al, g.K, g.M, g.lda, GP_BK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (g.b_kmajor)
    ok = ok && pair_map(&mbh, g.Bh, g.K, g.N, g.ldb, GP_BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
         pair_map(&mbl, g.Bl, g.K, g.N, g.ldb, GP_BK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok &&
         pair_map(&mbh, g.Bh, g.N, g.K, g.ldb, 32, GP_BK, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B) &&
         pair_map(&mbl, g.Bl, g.N, g.K, g.ldb, 32, GP_BK, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
  if (!ok) GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "pair GEMM: tensor map encoding failed");
  GemmPairParams p;
  p.M = g.M; p.N = g.N; p.K = g.K;
  p.C = g.C; p.Ch = g.Ch; p.Cl = g.Cl; p.ldc = g.ldc;
  p.alpha = g.alpha; p.beta = g.beta; p.flags = g.flags;
  p.b_kmajor = g.b_kmajor ? 1 : 0;
  p.vec = (g.ldc % 4 == 0) && (g.Ch ? (al(g.Ch) && al(g.Cl)) : al(g.C));
  p.kbp = g.partial_k > 0 ? std::max(1, g.partial_k / GP_BK) : 4;
  p.tiles_n = (g.N + 255) / 256;
  p.tiles_m = (g.M + 255) / 256;
  p.num_tiles = (g.flags & kCUpper) ? upper_tiles(p.tiles_m, p.tiles_n, GP_GROUP)
                                     : p.tiles_n * p.tiles_m;
  p.idesc = tc::idesc_f32acc(2u, false, !g.b_kmajor, 256, 256);
  const int npairs = std::min(p.num_tiles, c->num_sms / 2);
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_gemm_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          GP_SMEM));
  // CTA pairs keep the default wait budget (a pair whose CTAs gave up at different stages could
  // not drain every copy completing on the leader's barriers)
  GPTQ_LAUNCH(c, k_gemm_pair, 2 * npairs, GP_THREADS, GP_SMEM, mah, mal, mbh, mbl, p, c->status,
              kDefaultWaitCycles);
  return GPTQ_OK;
}

int gemm_pair(Ctx* c, int M, int N, int K, const float* Ah, const float* Al, long long lda,
              const float* Bh, const float* Bl, long long ldb, float* C, long long ldc, float alpha,
              float beta) {
  GemmPairArgs g{};
  g.M = M; g.N = N; g.K = K;
  g.Ah = Ah; g.Al = Al; g.lda = lda;
  g.Bh = Bh; g.Bl = Bl; g.ldb = ldb; g.b_kmajor = false;
  g.C = C; g.ldc = ldc; g.alpha = alpha; g.beta = beta; g.flags = 0;
  return gemm_pair(c, g);
}

}  // namespace gptq
