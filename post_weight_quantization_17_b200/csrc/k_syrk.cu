// a1: Hessian statistic S += Xc^T Xc over one token chunk ([T] eq.(9); accumulated in batches,
// [T] §9.4).  Only the lower triangle of S is produced.
//
// Tensor-core path (bf16 / f16 X, d % 8 == 0): a persistent kernel over 128 x 256 output
// tiles that touch the lower triangle.  X is token-major, so for a tile (I, J) both MMA
// operands are MN-major slices of the same chunk: A[i, t] = X[t, 128 I + i] and
// B[j, t] = X[t, 256 J + j].  Products of two 16-bit values are exact in fp32.
//   warp 0      TMA producer: 64-token slabs of A (2 boxes) and B (4 boxes), 4-stage ring
//   warp 1      MMA issuer: tcgen05.mma kind::f16, M=128 N=256 K=16, fp32 partial sums in TMEM
//   warps 2..9  epilogue: every SY_KP (512) tokens the TMEM partial is added (fp32, round to
//               nearest) into a 128 x 256 accumulator held in the epilogue warps' registers
//               (each thread: one row, 128 columns); at the end of the tile it goes to S.
// The tensor core's own fp32 accumulation loses precision roughly in proportion to the number
// of MMA steps it sums, so partial sums are kept short (512 tokens) and the long sum over all
// tokens is done with IEEE adds.  Measured H error against fp64: <= 1.4e-6 with 512-token
// partials on the parity cases (<= 7e-7 with 256, 1.2e-5 with 4096); 512 halves the hand-offs
// between MMA and epilogue.  Two TMEM partial buffers let the MMA run ahead of the adds.
// Every wait is bounded; a wait that runs out records GPTQ_ERR_TIMEOUT and the CTA unwinds
// (drains its own TMA copies, frees TMEM) instead of hanging.
//
// CUDA-core path: fp32 X, or shapes the tensor path does not take.
#include "kernels.h"
#include "gemm_simt.cuh"
#include "tc_util.cuh"

namespace gptq {

constexpr int SY_BM = 128, SY_BN = 256, SY_BK = 64, SY_STAGES = 4;
constexpr int SY_KP = 512;                               // tokens per TMEM partial sum
constexpr int SY_KB_PER_PART = SY_KP / SY_BK;
constexpr int SY_BOX_BYTES = SY_BK * 64 * 2;             // one 64 x 64 box of 16-bit values
constexpr int SY_A_BYTES = (SY_BM / 64) * SY_BOX_BYTES;  // 16 KB
constexpr int SY_B_BYTES = (SY_BN / 64) * SY_BOX_BYTES;  // 32 KB
constexpr int SY_STAGE_BYTES = SY_A_BYTES + SY_B_BYTES;
constexpr int SY_SMEM = SY_STAGES * SY_STAGE_BYTES + 1024 + 256;
constexpr int SY_EPI_WARPS = 8;
constexpr int SY_THREADS = 64 + 32 * SY_EPI_WARPS;

__device__ __forceinline__ void syrk_tile_coords(int t, int& I, int& J) {
  int i = 0;
  for (;;) {
    const int cnt = i / 2 + 1;  // tiles of row-block i touching j <= i: J = 0 .. floor(i/2)
    if (t < cnt) {
      I = i;
      J = t;
      return;
    }
    t -= cnt;
    ++i;
  }
}

__global__ void __launch_bounds__(SY_THREADS, 1)
    k_syrk_tc(const __grid_constant__ CUtensorMap tmap, float* __restrict__ S, int d,
              int n_tokens, int accumulate, int num_tiles, uint32_t idesc, DeviceStatus* st,
              long long budget) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SY_STAGES * SY_STAGE_BYTES);
  uint64_t* empty = full + SY_STAGES;
  uint64_t* tfull = empty + SY_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SY_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], 32 * SY_EPI_WARPS);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&tmap);
  if (warp == 1) tc::tmem_alloc(tmem_slot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the previous kernel; its outputs are read only from here on
  pdl_wait();
  pdl_release();
  const int kblocks = (n_tokens + SY_BK - 1) / SY_BK;
  const int nparts = (kblocks + SY_KB_PER_PART - 1) / SY_KB_PER_PART;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[SY_STAGES] = {};
      uint32_t issued_phase[SY_STAGES] = {};
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        int I, J;
        syrk_tile_coords(t, I, J);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 1);
            *abort_flag = 1;
            break;
          }
          uint8_t* sA = smem + stage * SY_STAGE_BYTES;
          uint8_t* sB = sA + SY_A_BYTES;
          tc::mbar_expect_tx(&full[stage], SY_STAGE_BYTES);
          const int y = kb * SY_BK;
          tc::tma_load_2d(sA, &tmap, &full[stage], I * SY_BM, y);
          tc::tma_load_2d(sA + SY_BOX_BYTES, &tmap, &full[stage], I * SY_BM + 64, y);
#pragma unroll
          for (int b = 0; b < SY_BN / 64; ++b)
            tc::tma_load_2d(sB + b * SY_BOX_BYTES, &tmap, &full[stage], J * SY_BN + 64 * b, y);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == SY_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: every copy this thread issued has landed before the CTA may exit
      for (int s = 0; s < SY_STAGES; ++s)
        if (issued[s] && !tc::mbar_wait(&full[s], issued_phase[s], kDrainCycles))
          raise_error(st, GPTQ_ERR_TIMEOUT, 2);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any = false;
      for (int t = blockIdx.x; t < num_tiles && ok && !*abort_flag; t += gridDim.x) {
        for (int p = 0; p < nparts && ok; ++p) {
          if (!tc::mbar_wait(&tempty[acc], acc_phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 3);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem + acc * SY_BN;
          const int kb1 = min(kblocks, (p + 1) * SY_KB_PER_PART);
          for (int kb = p * SY_KB_PER_PART; kb < kb1; ++kb) {
            if (!tc::mbar_wait(&full[stage], phase, budget)) {
              raise_error(st, GPTQ_ERR_TIMEOUT, 4);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc::fence_after_sync();
            const uint32_t a0 = tc::smem_u32(smem + stage * SY_STAGE_BYTES);
            const uint32_t b0 = a0 + SY_A_BYTES;
            const bool first = (kb == p * SY_KB_PER_PART);
#pragma unroll
            for (int kk = 0; kk < SY_BK / 16; ++kk) {
              const uint64_t ad = tc::sdesc_sw128(a0 + kk * 2048, SY_BOX_BYTES, 1024);
              const uint64_t bd = tc::sdesc_sw128(b0 + kk * 2048, SY_BOX_BYTES, 1024);
              tc::mma_f16(d_tmem, ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
            }
            any = true;
            tc::mma_commit(&empty[stage]);
            if (++stage == SY_STAGES) {
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
        if (!tc::mbar_wait(drain, 0, kDrainCycles)) raise_error(st, GPTQ_ERR_TIMEOUT, 6);
      }
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (tile rows of that quarter) and
    // the 128-column half h of the tile
    const int q = warp & 3;
    const int h = (warp - 2) / 4;
    const int r = 32 * q + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok && !*abort_flag; t += gridDim.x) {
      int I, J;
      syrk_tile_coords(t, I, J);
      float m[128];
#pragma unroll
      for (int u = 0; u < 128; ++u) m[u] = 0.f;
      for (int p = 0; p < nparts; ++p) {
        if (!tc::mbar_wait_warp(&tfull[acc], acc_phase, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 5);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t base = tmem + acc * SY_BN + ((uint32_t)(32 * q) << 16) + h * 128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
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
      const int gi = I * SY_BM + r;
      if (gi < d) {
        float* srow = S + (long long)gi * d;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int gj0 = J * SY_BN + h * 128 + cc * 32;
          if (gj0 > gi) continue;
          if (gj0 + 31 <= gi && gj0 + 32 <= d) {
            float4* p4 = reinterpret_cast<float4*>(srow + gj0);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              float4 x = make_float4(m[cc * 32 + 4 * u], m[cc * 32 + 4 * u + 1],
                                     m[cc * 32 + 4 * u + 2], m[cc * 32 + 4 * u + 3]);
              if (accumulate) {
                const float4 o = p4[u];
                x.x += o.x; x.y += o.y; x.z += o.z; x.w += o.w;
              }
              p4[u] = x;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int gj = gj0 + u;
              if (gj <= gi && gj < d) {
                const float x = m[cc * 32 + u];
                srow[gj] = accumulate ? srow[gj] + x : x;
              }
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
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// The same statistic on CTA pairs (cluster of 2, tcgen05 cta_group::2): 256 x 256 output tiles
// touching the lower triangle, M = N = 256 per MMA.  CTA r of the pair loads tile rows
// 128 r .. 128 r + 127 (A) and tile columns 128 r .. 128 r + 127 (its half of B) into its own
// shared memory; the tensor cores of both SMs read both halves of B, so each SM moves 32 KB
// per 64-token stage for the work that took 48 KB on one SM (shared-memory bandwidth was the
// single-SM limit).  Each CTA's TMEM receives its 128 rows of the tile and its own epilogue
// warps fold them into S exactly as above.
//   warp 0      both CTAs: TMA producer of its own halves (no multicast), 6-stage ring; the
//               copies of both CTAs complete on the leader's (rank 0) stage barrier, which the
//               leader arms for the bytes of both
//   warp 1      leader: MMA issuer; commits arrive on the barriers of both CTAs
//   warps 2..9  both CTAs: epilogue; a finished TMEM buffer is released to the leader by one
//               arrive per warp (remote for the peer)
// Every wait is bounded; both CTAs pass a cluster barrier before TMEM is freed or either exits
// (the leader has then seen every stage of both CTAs land).
constexpr int S2_BM = 128;                                // tile rows per CTA (256 per pair)
constexpr int S2_BN = 256;                                // tile columns (128 per CTA's B half)
constexpr int S2_STAGES = 6;
constexpr int S2_A_BYTES = (S2_BM / 64) * SY_BOX_BYTES;   // 16 KB
constexpr int S2_B_BYTES = (S2_BN / 128) * SY_BOX_BYTES;  // 16 KB: this CTA's 128 columns
constexpr int S2_STAGE_BYTES = S2_A_BYTES + S2_B_BYTES;
constexpr int S2_SMEM = S2_STAGES * S2_STAGE_BYTES + 1024 + 256;

// Tile t -> (I, J), J <= I, of the lower triangle of 256 x 256 tiles (nI row blocks).  Tiles go
// in groups of SY2_GROUP row blocks walked column by column (rows I of the group with I >= J), so
// that the 74 tiles of one wave cover ~8 row blocks and ~9 column blocks of X: every pair walks
// the token axis in lockstep, and a wave's X slabs are then fetched from HBM once for ~17
// feature blocks instead of once per tile (in row-major order a wave of a wide triangle spans one
// row block and ~74 column blocks).
constexpr int SY2_GROUP = 8;
__device__ __forceinline__ void syrk2_tile_coords(int t, int nI, int& I, int& J) {
  int first = 0;
  for (;;) {
    const int last = min(first + SY2_GROUP, nI) - 1;
    const int rows = last - first + 1;
    const int below = rows * first;                      // columns J < first: all rows
    const int cnt = below + rows * (rows + 1) / 2;       // + the group's own triangle
    if (t < cnt) {
      if (t < below) {
        J = t / rows;
        I = first + t % rows;
        return;
      }
      t -= below;
      for (int j = first;; ++j) {                        // column j holds rows j .. last
        const int c = last - j + 1;
        if (t < c) {
          J = j;
          I = j + t;
          return;
        }
        t -= c;
      }
    }
    t -= cnt;
    first += SY2_GROUP;
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SY_THREADS, 1)
    k_syrk_tc2(const __grid_constant__ CUtensorMap tmap, float* __restrict__ S, int d,
               int n_tokens, int accumulate, int num_tiles, uint32_t idesc, DeviceStatus* st,
               long long budget) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S2_STAGES * S2_STAGE_BYTES);
  uint64_t* empty = full + S2_STAGES;
  uint64_t* tfull = empty + S2_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S2_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&tfull[a], 1);
      tc::mbar_init(&tempty[a], 2 * SY_EPI_WARPS);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) tc::prefetch_tmap(&tmap);
  tc::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  if (warp == 1) tc::tmem_alloc_pair(tmem_slot, 512);
  tc::fence_before_sync();
  tc::cluster_sync();  // TMEM allocated in both CTAs before the leader's first MMA
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // set-up above overlaps the previous kernel; its outputs are read only from here on
  pdl_wait();
  pdl_release();
  const int kblocks = (n_tokens + SY_BK - 1) / SY_BK;
  const int nparts = (kblocks + SY_KB_PER_PART - 1) / SY_KB_PER_PART;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[S2_STAGES] = {};
      uint32_t issued_phase[S2_STAGES] = {};
      const uint32_t leader_full = tc::map_to_rank(full, 0);
      for (int t = pair; t < num_tiles && !*abort_flag; t += npairs) {
        int I, J;
        syrk2_tile_coords(t, (d + 255) / 256, I, J);
        const int ra = 256 * I + S2_BM * rank, rb = 256 * J + 128 * rank;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!tc::mbar_wait_cluster(&empty[stage], phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 21);
            *abort_flag = 1;
            break;
          }
          uint8_t* sA = smem + stage * S2_STAGE_BYTES;
          uint8_t* sB = sA + S2_A_BYTES;
          if (rank == 0) tc::mbar_expect_tx(&full[stage], 2 * S2_STAGE_BYTES);
          const uint32_t bar = leader_full + 8u * stage;
          const int y = kb * SY_BK;
          tc::tma_load_2d_pair(sA, &tmap, bar, ra, y);
          tc::tma_load_2d_pair(sA + SY_BOX_BYTES, &tmap, bar, ra + 64, y);
          tc::tma_load_2d_pair(sB, &tmap, bar, rb, y);
          tc::tma_load_2d_pair(sB + SY_BOX_BYTES, &tmap, bar, rb + 64, y);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == S2_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: the leader's stage barriers count both CTAs' copies
      if (rank == 0)
        for (int s = 0; s < S2_STAGES; ++s)
          if (issued[s] && !tc::mbar_wait_cluster(&full[s], issued_phase[s], kDrainCycles))
            raise_error(st, GPTQ_ERR_TIMEOUT, 22);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---- leader: MMA issuer for the pair
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, any = false;
      for (int t = pair; t < num_tiles && ok && !*abort_flag; t += npairs) {
        for (int p = 0; p < nparts && ok; ++p) {
          if (!tc::mbar_wait_cluster(&tempty[acc], acc_phase ^ 1, budget)) {
            raise_error(st, GPTQ_ERR_TIMEOUT, 23);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t d_tmem = tmem + acc * S2_BN;
          const int kb1 = min(kblocks, (p + 1) * SY_KB_PER_PART);
          for (int kb = p * SY_KB_PER_PART; kb < kb1; ++kb) {
            if (!tc::mbar_wait_cluster(&full[stage], phase, budget)) {
              raise_error(st, GPTQ_ERR_TIMEOUT, 24);
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc::fence_after_sync();
            const uint32_t a0 = tc::smem_u32(smem + stage * S2_STAGE_BYTES);
            const uint32_t b0 = a0 + S2_A_BYTES;
            const bool first = (kb == p * SY_KB_PER_PART);
#pragma unroll
            for (int kk = 0; kk < SY_BK / 16; ++kk) {
              const uint64_t ad = tc::sdesc_sw128(a0 + kk * 2048, SY_BOX_BYTES, 1024);
              const uint64_t bd = tc::sdesc_sw128(b0 + kk * 2048, SY_BOX_BYTES, 1024);
              tc::mma_f16_pair(d_tmem, ad, bd, idesc, (first && kk == 0) ? 0u : 1u);
            }
            any = true;
            tc::mma_commit_pair(&empty[stage]);
            if (++stage == S2_STAGES) {
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
      // every MMA of the pair has completed before either CTA may free TMEM or exit
      if (any) {
        tc::mma_commit_pair(drain);
        if (!tc::mbar_wait(drain, 0, kDrainCycles)) raise_error(st, GPTQ_ERR_TIMEOUT, 25);
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
    for (int t = pair; t < num_tiles && ok && !*abort_flag; t += npairs) {
      int I, J;
      syrk2_tile_coords(t, (d + 255) / 256, I, J);
      float m[128];
#pragma unroll
      for (int u = 0; u < 128; ++u) m[u] = 0.f;
      for (int p = 0; p < nparts; ++p) {
        if (!tc::mbar_wait_cluster_warp(&tfull[acc], acc_phase, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 27);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t base = tmem + acc * S2_BN + ((uint32_t)(32 * q) << 16) + h * 128;
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
      const int gi = 256 * I + S2_BM * rank + r;
      if (gi < d) {
        float* srow = S + (long long)gi * d;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int gj0 = 256 * J + h * 128 + cc * 32;
          if (gj0 > gi) continue;
          if (gj0 + 31 <= gi && gj0 + 32 <= d) {
            float4* p4 = reinterpret_cast<float4*>(srow + gj0);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              float4 x = make_float4(m[cc * 32 + 4 * u], m[cc * 32 + 4 * u + 1],
                                     m[cc * 32 + 4 * u + 2], m[cc * 32 + 4 * u + 3]);
              if (accumulate) {
                const float4 o = p4[u];
                x.x += o.x; x.y += o.y; x.z += o.z; x.w += o.w;
              }
              p4[u] = x;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              const int gj = gj0 + u;
              if (gj <= gi && gj < d) {
                const float x = m[cc * 32 + u];
                srow[gj] = accumulate ? srow[gj] + x : x;
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

// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int syrk_tc(Ctx* c, const void* X, int dtype, long long n, int d, float* S, bool overwrite) {
  auto encode = get_encode();
  if (!encode) GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)n};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, SY_BK};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&map, dtype == GPTQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                      2, const_cast<void*>(X), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  const uint32_t fmt = dtype == GPTQ_BF16 ? 1u : 0u;
  if (d >= 256 && c->num_sms >= 2) {
    // CTA pairs over 256 x 256 tiles
    const int nI = (d + 255) / 256;
    const int num_tiles = nI * (nI + 1) / 2;
    const int grid = 2 * std::min(num_tiles, c->num_sms / 2);
    GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_syrk_tc2,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, S2_SMEM));
    const uint32_t idesc = tc::idesc_f32acc(fmt, true, true, 2 * S2_BM, S2_BN);
    // a pair's two CTAs could give up at different stages, after which copies of one CTA that
    // complete on the other's barriers could not all be drained: pairs keep the default budget
    GPTQ_LAUNCH(c, k_syrk_tc2, grid, SY_THREADS, S2_SMEM, map, S, d, (int)n, overwrite ? 0 : 1,
                num_tiles, idesc, c->status, kDefaultWaitCycles);
    return GPTQ_OK;
  }
  const int nI = (d + SY_BM - 1) / SY_BM;
  int num_tiles = 0;
  for (int i = 0; i < nI; ++i) num_tiles += i / 2 + 1;
  const int grid = std::min(num_tiles, c->num_sms);
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_syrk_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SY_SMEM));
  const uint32_t idesc = tc::idesc_f32acc(fmt, true, true, SY_BM, SY_BN);
  GPTQ_LAUNCH(c, k_syrk_tc, grid, SY_THREADS, SY_SMEM, map, S, d, (int)n, overwrite ? 0 : 1,
                                                      num_tiles, idesc, c->status,
                                                      c->timeout_cycles);
  return GPTQ_OK;
}

int syrk_simt(Ctx* c, const void* X, int dtype, long long n, int d, float* S, bool overwrite) {
  GemmArgs g{d, d, (int)n, X, 1, d, X, d, 1, S, d, 1.f, overwrite ? 0.f : 1.f, kCLower};
  if (dtype == GPTQ_BF16) return gemm_simt<__nv_bfloat16, __nv_bfloat16>(c, g);
  if (dtype == GPTQ_F16) return gemm_simt<__half, __half>(c, g);
  return gemm_simt<float, float>(c, g);
}

// The tensor path needs 16-byte aligned rows for TMA (d % 8 == 0, aligned base) and takes
// shapes at least one box wide; smaller or fp32 inputs use the CUDA-core kernel.
static bool syrk_tc_applies(const void* X, int dtype, long long n, int d) {
  return (dtype == GPTQ_BF16 || dtype == GPTQ_F16) && d % 8 == 0 && d >= 128 && n >= SY_BK &&
         (reinterpret_cast<uintptr_t>(X) & 15) == 0;
}

int syrk_accumulate(Ctx* c, const void* X, int dtype, long long n, int d, float* S,
                    bool overwrite) {
  if (!syrk_tc_applies(X, dtype, n, d)) return syrk_simt(c, X, dtype, n, d, S, overwrite);
  return syrk_tc(c, X, dtype, n, d, S, overwrite);
}

}  // namespace gptq
