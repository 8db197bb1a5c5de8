// The consumer of the packed format: Y = X Ŵᵀ with Ŵ[r, k] = Δ[r, g(k)] (c[r, k] - z[r, g(k)]),
// the product a W4A16 linear layer computes at inference ([T] §1.2: the weights are stored as
// codes while the activations stay FP16/BF16; [A] "how it works": the codes are dequantized on
// the fly inside a fused kernel instead of being expanded in global memory).
//
// Tensor path (4-bit codes, 16-bit X, one grid per row or per 128 k columns):
//   Y[t, r] = sum_g Δ[r, g] · sum_{k in g} X[t, k] (c[r, k] - z[r, g])
// The inner sums run on tcgen05 with A = (c - z) as an exact 16-bit integer held in TMEM and
// B = X staged by TMA.  (c - z) comes from a magic-number conversion: OR-ing the code into the
// mantissa of 128.0 (bf16) or 1024.0 (fp16) gives 128 + c exactly, and subtracting 128 + z is
// exact too.  Every 128-column step's partial sum is read from TMEM and scaled by its Δ in fp32,
// so Ŵ is never rounded to 16 bits.
// The codes are read in runs of NB x 128 bytes per row (NB 128-byte-swizzle boxes of 128 rows,
// 2 NB steps) and the ring keeps up to CST - 1 such stages in flight per SM, which is what the
// HBM latency needs; a warp arrives on the per-step barriers through one elected lane.
//   warp 0        TMA producer of the codes ring (CST stages)
//   warp 1        MMA issuer (M = 128 rows, N = BN tokens, K = 16 per instruction), TMEM owner
//   warp 2        TMA producer of the X ring: [BN tokens x 128 columns] per step (two
//                 128-byte-swizzle boxes), XST stages
//   dequantize    DQW warps: row 32 (warp % 4) + lane, 4 / (DQW / 4) of the step's four 16-byte
//                 chunks per warp; (c - z) pairs into TMEM (A, four buffers, so that dequantizing
//                 runs up to three steps ahead of the MMAs)
//   epilogue      EPW warps: TMEM partial (ND buffers) -> acc[t] += Δ · partial for BN / (EPW / 4)
//                 tokens -> Y, or a split-K partial summed in a fixed order by k_dqmm_reduce
// Every wait is bounded (GPTQ_ERR_TIMEOUT, then the CTA drains its copies and frees TMEM) and
// suspends the waiting thread in hardware rather than polling, so that the many waiting warps
// leave the issue slots to the dequantize warps.
// Other formats (bits != 4, fp32 X, groups not a multiple of 128, per-column group ids, unaligned
// rows) run k_dqmm_simt on CUDA cores with the same definition.
#include "kernels.h"
#include "tc_util.cuh"

#include <algorithm>
#include <cstring>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace gptq {

constexpr int DQ_BM = 128;                 // rows (output features) per CTA
constexpr int DQ_KS = 128;                 // columns per MMA step
constexpr int DQ_BOX = DQ_BM * 128;        // one codes box: 128 rows x 128 bytes (2 steps)
constexpr int DQ_A_COLS = DQ_KS / 2;       // TMEM columns of one A buffer (two 16-bit per column)
constexpr int DQ_NA = 4;                   // A buffers in TMEM
constexpr int DQ_THREADS = 32 * 15;

template <int BN>
struct DqCfg {
  static constexpr int NB = 2;                      // codes boxes per stage (256 B per row)
  static constexpr int SPS = 2 * NB;                // MMA steps per codes stage
  static constexpr int CST = BN <= 16 ? 6 : (BN <= 64 ? 5 : 3);  // codes stages
  static constexpr int XST = 4;                     // X stages
  static constexpr int X_BYTES = BN * DQ_KS * 2;
  static constexpr int C_BYTES = NB * DQ_BOX;
  static constexpr int SMEM = CST * C_BYTES + XST * X_BYTES + 1024 + 512;
  static constexpr int DQW = BN >= 128 ? 4 : 8;     // dequantize warps
  static constexpr int EPW = 12 - DQW;              // epilogue warps
  static constexpr int CPT = 4 / (DQW / 4);         // 16-byte chunks per dequantize thread
  static constexpr int EBN = BN / (EPW / 4);        // tokens per epilogue thread
  static constexpr int ND = BN >= 128 ? 2 : 4;      // D buffers (partial sums) in TMEM
  static constexpr int TMEM_COLS = 512;
  static constexpr int CTAS_PER_SM = 1;
  static_assert(DQ_NA * DQ_A_COLS + ND * BN <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(3 + DQW + EPW == DQ_THREADS / 32, "warp roles");
  // the ring starts on a 1024-byte boundary (rounded up at run time) and every codes box, codes
  // stage and X stage is a whole number of 1024-byte swizzle repeats, so the tiled layout's
  // pre-applied 128-byte swizzle (chunk ^ (row & 7)) lines up with the hardware's
  static_assert(DQ_BOX % 1024 == 0 && C_BYTES % 1024 == 0 && X_BYTES % 1024 == 0,
                "swizzle alignment of the rings");
};

struct DqParams {
  int m, d, T, ng;
  int group_steps;  // steps per grid column (group / 128); 0: one grid per row
  int steps_total, steps_per_split;
  const float* scales;
  const int32_t* zeros;
  float* out;              // Y [T, m], or the split-K partials [splits, T, m]
  const uint32_t* tiled;   // codes in the tile-contiguous layout (gptq_retile_codes), or null
  int ktiles;              // 256-code tiles per row block in that layout
  long long split_stride;  // T * m when partials are written, else 0
  uint32_t idesc;
};

__device__ __forceinline__ void mma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Whole warp: its 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// As mbar_wait, but each try suspends the thread in hardware (up to `hint_ns`) until the phase
// completes, instead of returning at once: waiting warps then take no issue slots from the
// warps that compute.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity,
                                                   uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(tc::smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, long long budget) {
  if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_hint(bar, parity, 20000u)) {
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

// One contiguous global -> shared copy of `bytes` (16-byte aligned, a multiple of 16) whose
// completion is counted on `bar` (no multicast).
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// (c - z) for the 8 codes of one word as four 16-bit pairs in K order (code 2p in the low half
// of out[p], code 2p + 1 in the high half).  y = word >> 4 puts code 2p + 1 in the low nibble of
// byte p, so one byte permute per pair brings both codes to the low nibbles of the two halves.
template <bool BF16>
__device__ __forceinline__ void dequant_word(uint32_t word, uint32_t zz, uint32_t (&out)[4]) {
  constexpr uint32_t magic = BF16 ? 0x43004300u : 0x64006400u;  // 128.0 / 1024.0 in each half
  const uint32_t y = word >> 4;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t sel = (uint32_t)p | ((uint32_t)p << 4) | ((uint32_t)(4 + p) << 8) |
                         ((uint32_t)(4 + p) << 12);
    const uint32_t t = (prmt(word, y, sel) & 0x000F000Fu) | magic;
    if (BF16) {
      const __nv_bfloat162 d = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&t),
                                       *reinterpret_cast<const __nv_bfloat162*>(&zz));
      out[p] = *reinterpret_cast<const uint32_t*>(&d);
    } else {
      const __half2 d = __hsub2(*reinterpret_cast<const __half2*>(&t),
                                *reinterpret_cast<const __half2*>(&zz));
      out[p] = *reinterpret_cast<const uint32_t*>(&d);
    }
  }
}

template <int BN, bool BF16, bool TILED>
__global__ void __launch_bounds__(DQ_THREADS)
    k_dqmm_tc(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmX,
              DqParams p, DeviceStatus* st, long long budget) {
  using Cfg = DqCfg<BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* cbuf = smem;                                // codes ring
  uint8_t* xbuf = smem + Cfg::CST * Cfg::C_BYTES;      // X ring
  uint64_t* full_c = reinterpret_cast<uint64_t*>(xbuf + Cfg::XST * Cfg::X_BYTES);
  uint64_t* empty_c = full_c + Cfg::CST;
  uint64_t* full_x = empty_c + Cfg::CST;
  uint64_t* empty_x = full_x + Cfg::XST;
  uint64_t* a_full = empty_x + Cfg::XST;
  uint64_t* a_free = a_full + DQ_NA;
  uint64_t* d_full = a_free + DQ_NA;
  uint64_t* d_empty = d_full + Cfg::ND;
  uint64_t* drain = d_empty + Cfg::ND;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * DQ_BM, tok0 = blockIdx.y * BN;
  const int k_begin = blockIdx.z * p.steps_per_split;
  const int n = min(p.steps_total, k_begin + p.steps_per_split) - k_begin;
  const int nst = (n + Cfg::SPS - 1) / Cfg::SPS;  // codes stages of this CTA
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::CST; ++s) {
      tc::mbar_init(&full_c[s], 1);
      tc::mbar_init(&empty_c[s], Cfg::DQW);
    }
    for (int s = 0; s < Cfg::XST; ++s) {
      tc::mbar_init(&full_x[s], 1);
      tc::mbar_init(&empty_x[s], 1);
    }
    for (int b = 0; b < DQ_NA; ++b) {
      tc::mbar_init(&a_full[b], Cfg::DQW);
      tc::mbar_init(&a_free[b], 1);
    }
    for (int b = 0; b < Cfg::ND; ++b) {
      tc::mbar_init(&d_full[b], 1);
      tc::mbar_init(&d_empty[b], Cfg::EPW);
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    if (!TILED) tc::prefetch_tmap(&tmC);
    tc::prefetch_tmap(&tmX);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t a_col = 0, d_col = DQ_NA * DQ_A_COLS;
  pdl_wait();
  pdl_release();

  if (warp == 0) {
    // ---------------------------------------------------------------- codes producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nst && !*abort_flag; ++j) {
        const int s = j % Cfg::CST;
        const uint32_t ph = (uint32_t)(j / Cfg::CST) & 1u;
        if (!mbar_wait_sleep(&empty_c[s], ph ^ 1u, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 41);
          *abort_flag = 1;
          break;
        }
        if (TILED) {
          // whole 16 KB tiles, already in the swizzled order the reads below expect; a tile past
          // the row's end is not loaded (its steps are never processed)
          const int kt0 = (k_begin + j * Cfg::SPS) / 2;
          int nbox = 0;
#pragma unroll
          for (int bx = 0; bx < Cfg::NB; ++bx) nbox += (kt0 + bx < p.ktiles) ? 1 : 0;
          tc::mbar_expect_tx(&full_c[s], nbox * DQ_BOX);
#pragma unroll
          for (int bx = 0; bx < Cfg::NB; ++bx)
            if (kt0 + bx < p.ktiles)
              bulk_load_1d(cbuf + s * Cfg::C_BYTES + bx * DQ_BOX,
                           p.tiled + ((size_t)blockIdx.x * p.ktiles + kt0 + bx) * (DQ_BOX / 4),
                           DQ_BOX, &full_c[s]);
        } else {
          tc::mbar_expect_tx(&full_c[s], Cfg::C_BYTES);
          const int x0 = (k_begin + j * Cfg::SPS) * 16;  // in 32-bit words
#pragma unroll
          for (int bx = 0; bx < Cfg::NB; ++bx)
            tc::tma_load_2d(cbuf + s * Cfg::C_BYTES + bx * DQ_BOX, &tmC, &full_c[s], x0 + 32 * bx,
                            row0);
        }
        issued = j + 1;
      }
      for (int j = max(0, issued - Cfg::CST); j < issued; ++j)
        if (!mbar_wait_sleep(&full_c[j % Cfg::CST], (uint32_t)(j / Cfg::CST) & 1u, kDrainCycles))
          raise_error(st, GPTQ_ERR_TIMEOUT, 42);
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- X producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < n && !*abort_flag; ++i) {
        const int s = i % Cfg::XST;
        const uint32_t ph = (uint32_t)(i / Cfg::XST) & 1u;
        if (!mbar_wait_sleep(&empty_x[s], ph ^ 1u, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 47);
          *abort_flag = 1;
          break;
        }
        uint8_t* base = xbuf + s * Cfg::X_BYTES;
        const int kx = (k_begin + i) * DQ_KS;
        tc::mbar_expect_tx(&full_x[s], Cfg::X_BYTES);
        tc::tma_load_2d(base, &tmX, &full_x[s], kx, tok0);
        tc::tma_load_2d(base + BN * 128, &tmX, &full_x[s], kx + 64, tok0);
        issued = i + 1;
      }
      for (int i = max(0, issued - Cfg::XST); i < issued; ++i)
        if (!mbar_wait_sleep(&full_x[i % Cfg::XST], (uint32_t)(i / Cfg::XST) & 1u, kDrainCycles))
          raise_error(st, GPTQ_ERR_TIMEOUT, 48);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool any = false;
      for (int i = 0; i < n && !*abort_flag; ++i) {
        const int s = i % Cfg::XST, a = i % DQ_NA, b = i % Cfg::ND;
        const uint32_t ph = (uint32_t)(i / Cfg::XST) & 1u;
        const uint32_t aph = (uint32_t)(i / DQ_NA) & 1u, dph = (uint32_t)(i / Cfg::ND) & 1u;
        if (!mbar_wait_sleep(&d_empty[b], dph ^ 1u, budget) ||
            !mbar_wait_sleep(&a_full[a], aph, budget) || !mbar_wait_sleep(&full_x[s], ph, budget)) {
          raise_error(st, GPTQ_ERR_TIMEOUT, 43);
          *abort_flag = 1;
          break;
        }
        tc::fence_after_sync();
        const uint32_t xs = tc::smem_u32(xbuf + s * Cfg::X_BYTES);
#pragma unroll
        for (int kk = 0; kk < DQ_KS / 16; ++kk) {
          const uint64_t bd = tc::sdesc_sw128(xs + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16,
                                              1024);
          mma_f16_tmem_a(tmem + d_col + b * BN, tmem + a_col + a * DQ_A_COLS + kk * 8, bd,
                         p.idesc, kk > 0 ? 1u : 0u);
        }
        any = true;
        tc::mma_commit(&empty_x[s]);
        tc::mma_commit(&a_free[a]);
        tc::mma_commit(&d_full[b]);
      }
      // every MMA has completed before TMEM is freed (after an abort the epilogue may not have
      // waited for them)
      if (any) {
        tc::mma_commit(drain);
        if (!mbar_wait_sleep(drain, 0, kDrainCycles)) raise_error(st, GPTQ_ERR_TIMEOUT, 49);
      }
    }
  } else if (warp < 3 + Cfg::DQW) {
    // ---------------------------------------------------------------- dequantize into TMEM
    const int q = warp & 3, h = (warp - 3) >> 2, r = 32 * q + lane, row = row0 + r;
    const bool active = row < p.m;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + a_col + h * Cfg::CPT * 16;
    const int swz = r & 7;  // 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r & 7)
    const int32_t* zrow = p.zeros + (long long)(active ? row : 0) * p.ng;
    int32_t z_next = active ? zrow[p.group_steps ? k_begin / p.group_steps : 0] : 0;
    for (int i = 0; i < n && !*abort_flag; ++i) {
      const int j = i / Cfg::SPS, within = i % Cfg::SPS;
      const int cs = j % Cfg::CST, a = i % DQ_NA;
      const uint32_t cph = (uint32_t)(j / Cfg::CST) & 1u, aph = (uint32_t)(i / DQ_NA) & 1u;
      int32_t z = z_next;
      if (active && i + 1 < n)
        z_next = zrow[p.group_steps ? (k_begin + i + 1) / p.group_steps : 0];
      if (z < 0 || z > 15) {  // (c - z) would not be exact in 16 bits; a 4-bit grid has z <= 15
        raise_error(st, GPTQ_ERR_ARG, row);
        z = 0;
      }
      // 128 + z (or 1024 + z) in both halves
      uint32_t zz;
      if (BF16) {
        const __nv_bfloat16 hz = __float2bfloat16_rn(128.f + (float)z);
        const uint16_t u = *reinterpret_cast<const uint16_t*>(&hz);
        zz = (uint32_t)u | ((uint32_t)u << 16);
      } else {
        const __half hz = __float2half_rn(1024.f + (float)z);
        const uint16_t u = *reinterpret_cast<const uint16_t*>(&hz);
        zz = (uint32_t)u | ((uint32_t)u << 16);
      }
      if (within == 0 && !__all_sync(0xffffffffu, mbar_wait_sleep(&full_c[cs], cph, budget))) {
        raise_error(st, GPTQ_ERR_TIMEOUT, 44);
        *abort_flag = 1;
        break;
      }
      // this step's 64 bytes of the row: chunks 4 (i & 1) .. + 3 of the box's 128-byte row
      const uint8_t* rowp = cbuf + cs * Cfg::C_BYTES + (within >> 1) * DQ_BOX + r * 128;
      uint4 v[Cfg::CPT];
#pragma unroll
      for (int c = 0; c < Cfg::CPT; ++c) {
        const int chunk = 4 * (i & 1) + h * Cfg::CPT + c;
        v[c] = *reinterpret_cast<const uint4*>(rowp + ((chunk ^ swz) << 4));
      }
      if (within == Cfg::SPS - 1) {  // the warp is done with this codes stage
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty_c[cs]);
      }
      // A buffer a was last read by the MMAs of step i - 4
      if (i >= DQ_NA && !__all_sync(0xffffffffu, mbar_wait_sleep(&a_free[a], aph ^ 1u, budget))) {
        raise_error(st, GPTQ_ERR_TIMEOUT, 45);
        *abort_flag = 1;
        break;
      }
      tc::fence_after_sync();
#pragma unroll
      for (int c = 0; c < Cfg::CPT; ++c) {
        const uint32_t words[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
        uint32_t o[16];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t pr[4];
          dequant_word<BF16>(words[w], zz, pr);
#pragma unroll
          for (int u = 0; u < 4; ++u) o[4 * w + u] = pr[u];
        }
        tmem_st16(lane_base + a * DQ_A_COLS + c * 16, o);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&a_full[a]);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3, e = (warp - 3 - Cfg::DQW) >> 2, r = 32 * q + lane, row = row0 + r;
    const bool active = row < p.m;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + d_col + e * Cfg::EBN;
    const float* srow = p.scales + (long long)(active ? row : 0) * p.ng;
    float acc[Cfg::EBN];
#pragma unroll
    for (int t = 0; t < Cfg::EBN; ++t) acc[t] = 0.f;
    bool ok = true;
    float delta_next = active ? srow[p.group_steps ? k_begin / p.group_steps : 0] : 0.f;
    for (int i = 0; i < n && !*abort_flag; ++i) {
      const int b = i % Cfg::ND;
      const uint32_t dph = (uint32_t)(i / Cfg::ND) & 1u;
      const float delta = delta_next;
      if (active && i + 1 < n)
        delta_next = srow[p.group_steps ? (k_begin + i + 1) / p.group_steps : 0];
      if (!__all_sync(0xffffffffu, mbar_wait_sleep(&d_full[b], dph, budget))) {
        raise_error(st, GPTQ_ERR_TIMEOUT, 46);
        *abort_flag = 1;
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t dbase = lane_base + b * BN;
      if (Cfg::EBN == 16) {
        uint32_t v[16];
        tmem_ld16(dbase, v);
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = fmaf(delta, __uint_as_float(v[t]), acc[t]);
      } else {
#pragma unroll
        for (int cc = 0; cc < Cfg::EBN / 32; ++cc) {
          uint32_t v[32];
          tc::tmem_ld32(dbase + cc * 32, v);
#pragma unroll
          for (int t = 0; t < 32; ++t)
            acc[cc * 32 + t] = fmaf(delta, __uint_as_float(v[t]), acc[cc * 32 + t]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&d_empty[b]);
    }
    if (ok && active) {
      float* out = p.out + (long long)blockIdx.z * p.split_stride + row;
      const int t0 = tok0 + e * Cfg::EBN;
#pragma unroll
      for (int t = 0; t < Cfg::EBN; ++t)
        if (t0 + t < p.T) out[(long long)(t0 + t) * p.m] = acc[t];
    }
  }
  __syncwarp();
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// Y = sum over splits of the partials, in split order.
__global__ void k_dqmm_reduce(const float* __restrict__ part, int splits, long long n,
                              float* __restrict__ Y) {
  pdl_wait();
  pdl_release();
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float s = part[e];
  for (int k = 1; k < splits; ++k) s += part[(long long)k * n + e];
  Y[e] = s;
}

// CUDA cores, any format: CTA = 128 rows x 8 tokens, K in chunks of 32 columns (whole words of
// every width: a 32-code chunk is `bits` words).  Ŵ is formed exactly as the quantizer defines it
// (Δ (c - z) in fp32) and accumulated in fp32.
template <class TX>
__global__ void __launch_bounds__(128)
    k_dqmm_simt(const TX* __restrict__ X, int T, int d, const uint32_t* __restrict__ packed,
                int wpr, int m, int bits, int group, const int32_t* __restrict__ group_id, int ng,
                const float* __restrict__ scales, const int32_t* __restrict__ zeros,
                float* __restrict__ Y, DeviceStatus* st) {
  pdl_wait();
  pdl_release();
  __shared__ float xs[8][33];
  const int r = blockIdx.x * 128 + threadIdx.x, tok0 = blockIdx.y * 8;
  const bool active = r < m;
  const uint32_t mask = (1u << bits) - 1u;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  bool bad = false;
  for (int k0 = 0; k0 < d; k0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 8 * 32; e += 128) {
      const int t = e >> 5, j = e & 31;
      xs[t][j] = (tok0 + t < T && k0 + j < d)
                     ? to_f32<TX>(X[(long long)(tok0 + t) * d + k0 + j])
                     : 0.f;
    }
    __syncthreads();
    if (!active) continue;
    const int w0 = (k0 / 32) * bits;
    const uint32_t* src = packed + (long long)r * wpr + w0;
    const int nwords = min(bits, wpr - w0);
    unsigned long long bitsbuf = 0;
    int nbits = 0, win = 0;
    const int nj = min(32, d - k0);
    for (int j = 0; j < nj; ++j) {
      if (nbits < bits) {
        if (win < nwords) bitsbuf |= (unsigned long long)src[win++] << nbits;
        nbits += 32;
      }
      const int code = (int)(bitsbuf & mask);
      bitsbuf >>= bits;
      nbits -= bits;
      const int col = k0 + j;
      int gi = group_id ? group_id[col] : (group == -1 ? 0 : col / group);
      if (gi < 0 || gi >= ng) {
        bad = true;
        gi = 0;
      }
      const long long gidx = (long long)r * ng + gi;
      const float w = __fmul_rn(scales[gidx], (float)(code - zeros[gidx]));
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t] = fmaf(xs[t][j], w, acc[t]);
    }
  }
  if (bad) raise_error(st, GPTQ_ERR_ARG, r);
  if (!active) return;
#pragma unroll
  for (int t = 0; t < 8; ++t)
    if (tok0 + t < T) Y[(long long)(tok0 + t) * m + r] = acc[t];
}

// ------------------------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 dq_encode() {
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

static bool dq_map(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base,
                   long long inner, long long outer, long long ld, int box_inner, int box_outer,
                   CUtensorMapSwizzle swz) {
  auto enc = dq_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * esize)};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool dequant_matmul_tc_applies(const void* X, int x_dtype, int d, const uint32_t* packed,
                               int bits, int group, const int32_t* group_id) {
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  return bits == 4 && (x_dtype == GPTQ_BF16 || x_dtype == GPTQ_F16) && d % 32 == 0 && al(X) &&
         al(packed) && (group == -1 || group % DQ_KS == 0) && group_id == nullptr;
}

template <int BN, bool BF16, bool TILED>
static int launch_dqmm_tc(Ctx* c, const void* X, int T, int d, const uint32_t* packed, int m,
                          int group, int ng, const float* scales, const int32_t* zeros, float* Y,
                          float* part_ws, size_t part_floats) {
  using Cfg = DqCfg<BN>;
  const int wpr = d / 8;
  CUtensorMap mc, mx;
  memset(&mc, 0, sizeof(mc));
  if (!TILED && !dq_map(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, packed, wpr, m, wpr, 32, DQ_BM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
    GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "dequant_matmul: tensor map for the codes failed");
  if (!dq_map(&mx, BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
              X, d, T, d, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    GPTQ_SET_ERR(c, GPTQ_ERR_CUDA, "dequant_matmul: tensor map for X failed");
  const int rt = (m + DQ_BM - 1) / DQ_BM, tt = (T + BN - 1) / BN;
  const int ks = (d + DQ_KS - 1) / DQ_KS;
  // Split K (small token counts only, where the partials are small): choose the steps per CTA
  // that minimize waves x (steps + a fixed start-up cost of about 4 steps) on the GPU's SMs.
  const long long slots = (long long)c->num_sms * Cfg::CTAS_PER_SM;
  int per = ks;
  if (BN <= 64) {
    long long best = -1;
    for (int cand = ks; cand >= 1; --cand) {
      if (TILED && cand != ks && cand % 2) continue;  // splits start on whole 256-code tiles
      const long long sp = (ks + cand - 1) / cand;
      if (sp > 1 && (size_t)sp * T * m > part_floats) break;
      const long long waves = (rt * tt * sp + slots - 1) / slots;
      const long long cost = waves * (cand + 4);
      if (best < 0 || cost < best) {
        best = cost;
        per = cand;
      }
    }
  }
  const int splits = (ks + per - 1) / per;
  DqParams p;
  p.m = m; p.d = d; p.T = T; p.ng = ng;
  p.group_steps = (group == -1) ? 0 : group / DQ_KS;
  p.steps_total = ks;
  p.steps_per_split = per;
  p.scales = scales;
  p.zeros = zeros;
  p.out = (splits > 1) ? part_ws : Y;
  p.split_stride = (splits > 1) ? (long long)T * m : 0;
  p.tiled = TILED ? packed : nullptr;
  p.ktiles = (d + 255) / 256;
  p.idesc = tc::idesc_f32acc(BF16 ? 1u : 0u, false, false, DQ_BM, BN);
  GPTQ_CUDA_CHECK(c, cudaFuncSetAttribute(k_dqmm_tc<BN, BF16, TILED>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM));
  GPTQ_LAUNCH(c, k_dqmm_tc<BN, BF16, TILED>, dim3(rt, tt, splits), DQ_THREADS, Cfg::SMEM, mc, mx,
              p, c->status, c->timeout_cycles);
  if (splits > 1) {
    const long long nel = (long long)T * m;
    GPTQ_LAUNCH(c, k_dqmm_reduce, (int)((nel + 255) / 256), 256, 0, (const float*)part_ws, splits,
                nel, Y);
  }
  return GPTQ_OK;
}

template <bool TILED>
static int dispatch_dqmm_tc(Ctx* c, const void* X, int x_dtype, int T, int d,
                            const uint32_t* codes, int m, int group, int ng, const float* scales,
                            const int32_t* zeros, float* Y, float* part_ws, size_t part_floats) {
  const bool bf = (x_dtype == GPTQ_BF16);
  if (T <= 16)
    return bf ? launch_dqmm_tc<16, true, TILED>(c, X, T, d, codes, m, group, ng, scales, zeros,
                                                Y, part_ws, part_floats)
              : launch_dqmm_tc<16, false, TILED>(c, X, T, d, codes, m, group, ng, scales, zeros,
                                                 Y, part_ws, part_floats);
  if (T <= 64)
    return bf ? launch_dqmm_tc<64, true, TILED>(c, X, T, d, codes, m, group, ng, scales, zeros,
                                                Y, part_ws, part_floats)
              : launch_dqmm_tc<64, false, TILED>(c, X, T, d, codes, m, group, ng, scales, zeros,
                                                 Y, part_ws, part_floats);
  return bf ? launch_dqmm_tc<128, true, TILED>(c, X, T, d, codes, m, group, ng, scales, zeros, Y,
                                               part_ws, part_floats)
            : launch_dqmm_tc<128, false, TILED>(c, X, T, d, codes, m, group, ng, scales, zeros, Y,
                                                part_ws, part_floats);
}

int dequant_matmul_tiled(Ctx* c, const void* X, int x_dtype, int T, int d,
                         const uint32_t* tiled, int m, int group, int ng, const float* scales,
                         const int32_t* zeros, float* Y, float* part_ws, size_t part_floats) {
  return dispatch_dqmm_tc<true>(c, X, x_dtype, T, d, tiled, m, group, ng, scales, zeros, Y,
                                part_ws, part_floats);
}

// 16-byte chunk o of the tile-contiguous layout: tile o / 1024 (row block rt, 256-code column
// block kt), row r = (o % 1024) / 8 of the tile, stored chunk pc = o % 8 holding the row's
// logical chunk pc ^ (r & 7) (the 128-byte swizzle); rows and columns past the matrix are zero.
__global__ void k_retile_w4(const uint32_t* __restrict__ packed, int m, int wpr, int ktiles,
                            long long nchunks, uint32_t* __restrict__ tiled) {
  pdl_wait();
  pdl_release();
  const long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= nchunks) return;
  const long long tile = o / 1024;
  const int q = (int)(o % 1024), r = q / 8, pc = q % 8, cidx = pc ^ (r & 7);
  const long long rt = tile / ktiles, kt = tile % ktiles;
  const long long row = rt * DQ_BM + r, word = kt * 32 + cidx * 4;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (row < m && word + 4 <= wpr) v = *reinterpret_cast<const uint4*>(packed + row * wpr + word);
  reinterpret_cast<uint4*>(tiled)[o] = v;
}

long long retile_words(long long m, long long d) {
  return ((m + DQ_BM - 1) / DQ_BM) * ((d + 255) / 256) * (DQ_BOX / 4);
}

int retile_codes(Ctx* c, const uint32_t* packed, int m, int d, uint32_t* tiled) {
  const long long nchunks = retile_words(m, d) / 4;
  GPTQ_LAUNCH(c, k_retile_w4, (int)((nchunks + 255) / 256), 256, 0, packed, m, d / 8,
              (d + 255) / 256, nchunks, tiled);
  return GPTQ_OK;
}

int dequant_matmul(Ctx* c, const void* X, int x_dtype, int T, int d, const uint32_t* packed,
                   int m, int bits, int group, const int32_t* group_id, int ng,
                   const float* scales, const int32_t* zeros, float* Y, float* part_ws,
                   size_t part_floats) {
  if (dequant_matmul_tc_applies(X, x_dtype, d, packed, bits, group, group_id))
    return dispatch_dqmm_tc<false>(c, X, x_dtype, T, d, packed, m, group, ng, scales, zeros, Y,
                                   part_ws, part_floats);
  const int wpr = (int)(((long long)d * bits + 31) / 32);
  const dim3 grid((m + 127) / 128, (T + 7) / 8);
  if (x_dtype == GPTQ_BF16)
    GPTQ_LAUNCH(c, k_dqmm_simt<__nv_bfloat16>, grid, 128, 0, (const __nv_bfloat16*)X, T, d, packed,
                wpr, m, bits, group, group_id, ng, scales, zeros, Y, c->status);
  else if (x_dtype == GPTQ_F16)
    GPTQ_LAUNCH(c, k_dqmm_simt<__half>, grid, 128, 0, (const __half*)X, T, d, packed, wpr, m,
                bits, group, group_id, ng, scales, zeros, Y, c->status);
  else
    GPTQ_LAUNCH(c, k_dqmm_simt<float>, grid, 128, 0, (const float*)X, T, d, packed, wpr, m, bits,
                group, group_id, ng, scales, zeros, Y, c->status);
  return GPTQ_OK;
}

}  // namespace gptq
