// a8: dense bit-packing of the codes ([T] §3.1 output table, §9.4).  Per row a little-endian
// bitstream: code k occupies bits [b k, b k + b); word w holds bits [32 w, 32 w + 32).
// 32 codes of b bits fill exactly b words, so a thread that packs whole 32-code chunks owns
// whole output words and no two threads touch the same word.
#include "kernels.h"

namespace gptq {

// Packs one 32-code chunk held in v[32] into `bits` words at dst (n valid codes).
__device__ __forceinline__ void pack_chunk(const uint8_t (&v)[32], int n, int bits,
                                           uint32_t* __restrict__ dst) {
  const uint32_t mask = (1u << bits) - 1u;
  uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  unsigned long long acc = 0;
  int nacc = 0, wout = 0;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    if (q < n) {
      acc |= (unsigned long long)(v[q] & mask) << nacc;
      nacc += bits;
      if (nacc >= 32) {
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k == wout) w[k] = (uint32_t)acc;
        ++wout;
        acc >>= 32;
        nacc -= 32;
      }
    }
  }
  if (nacc > 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k == wout) w[k] = (uint32_t)acc;
    ++wout;
  }
  const uintptr_t a = reinterpret_cast<uintptr_t>(dst);
  if (n == 32 && bits == 4 && (a & 15) == 0) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (n == 32 && bits == 2 && (a & 7) == 0) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if (n == 32 && bits == 8 && (a & 15) == 0) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < wout) dst[k] = w[k];
  }
}

// Four codes (the bytes of x, code k in byte k) as a 4 b-bit field, for b = 2 or 4.
template <int B>
__device__ __forceinline__ uint32_t squeeze4(uint32_t x) {
  constexpr uint32_t m = (1u << B) - 1u;
  uint32_t t = x & (m * 0x01010101u);             // c0 | c1 << 8 | c2 << 16 | c3 << 24
  t = (t | (t >> (8 - B))) & ((1u << (2 * B)) - 1u) * 0x00010001u;  // pairs in bytes 0 and 2
  return (t | (t >> (16 - 2 * B))) & ((1u << (4 * B)) - 1u);        // c0 | c1 << B | ...
}

// One 32-code chunk per thread.  For 2-, 4- and 8-bit codes in dense rows (d % 32 == 0) the
// words come from the 32 loaded bytes by independent mask-and-shift steps (8-bit words are the
// bytes themselves); other widths run the bit accumulator of pack_chunk.
__global__ void k_pack(const uint8_t* __restrict__ codes, int m, int d, int bits,
                       uint32_t* __restrict__ packed, int wpr) {
  pdl_wait();
  pdl_release();
  const int chunks = (d + 31) / 32;
  const long long total = (long long)m * chunks;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const bool linear = (d % 32 == 0) && ((reinterpret_cast<uintptr_t>(codes) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(packed) & 15) == 0);
  if (linear && (bits == 2 || bits == 4 || bits == 8)) {
    // the (row, chunk) space is linear in both codes and packed words
    const uint4* src = reinterpret_cast<const uint4*>(codes + t * 32);
    const uint4 a = src[0], b = src[1];
    const uint32_t x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t* dst = packed + t * bits;
    if (bits == 8) {
      reinterpret_cast<uint4*>(dst)[0] = a;
      reinterpret_cast<uint4*>(dst)[1] = b;
    } else if (bits == 4) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) w[k] = squeeze4<4>(x[2 * k]) | (squeeze4<4>(x[2 * k + 1]) << 16);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
      uint32_t w[2];
#pragma unroll
      for (int k = 0; k < 2; ++k)
        w[k] = squeeze4<2>(x[4 * k]) | (squeeze4<2>(x[4 * k + 1]) << 8) |
               (squeeze4<2>(x[4 * k + 2]) << 16) | (squeeze4<2>(x[4 * k + 3]) << 24);
      *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    }
    return;
  }
  const int r = (int)(t / chunks), ch = (int)(t % chunks);
  const int k0 = ch * 32, n = min(32, d - k0);
  const uint8_t* src = codes + (long long)r * d + k0;
  uint8_t v[32];
  if (n == 32 && ((reinterpret_cast<uintptr_t>(src) & 15) == 0)) {
    *reinterpret_cast<uint4*>(&v[0]) = reinterpret_cast<const uint4*>(src)[0];
    *reinterpret_cast<uint4*>(&v[16]) = reinterpret_cast<const uint4*>(src)[1];
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = (q < n) ? src[q] : 0;
  }
  pack_chunk(v, n, bits, packed + (long long)r * wpr + (long long)ch * bits);
}

__global__ void k_unpack(const uint32_t* __restrict__ packed, int m, int d, int bits,
                         uint8_t* __restrict__ codes, int wpr) {
  pdl_wait();
  pdl_release();
  const int chunks = (d + 31) / 32;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)m * chunks) return;
  const int r = (int)(t / chunks), ch = (int)(t % chunks);
  const int k0 = ch * 32, n = min(32, d - k0);
  const uint32_t mask = (1u << bits) - 1u;
  const uint32_t* src = packed + (long long)r * wpr + (long long)ch * bits;
  const int nwords = (n * bits + 31) / 32;
  unsigned long long acc = 0;
  int nacc = 0, win = 0;
  uint8_t* dst = codes + (long long)r * d + k0;
  for (int q = 0; q < n; ++q) {
    if (nacc < bits) {
      if (win < nwords) acc |= (unsigned long long)src[win++] << nacc;
      nacc += 32;
    }
    dst[q] = (uint8_t)(acc & mask);
    acc >>= bits;
    nacc -= bits;
  }
}

int pack_codes(Ctx* c, const uint8_t* codes, int m, int d, int bits, uint32_t* packed) {
  const int wpr = (int)(((long long)d * bits + 31) / 32);
  const long long chunks = (long long)m * ((d + 31) / 32);
  GPTQ_LAUNCH(c, k_pack, (int)((chunks + 255) / 256), 256, 0, codes, m, d, bits, packed, wpr);
  return GPTQ_OK;
}

int unpack_codes(Ctx* c, const uint32_t* packed, int m, int d, int bits, uint8_t* codes) {
  const int wpr = (int)(((long long)d * bits + 31) / 32);
  const long long threads = (long long)m * ((d + 31) / 32);
  GPTQ_LAUNCH(c, k_unpack, (int)((threads + 255) / 256), 256, 0, packed, m, d, bits, codes, wpr);
  return GPTQ_OK;
}

}  // namespace gptq
