// a8: dense bit-packing of the codes ([T] §3.1 output table, §9.4).  Per row a little-endian
// bitstream: code k occupies bits [b k, b k + b); word w holds bits [32 w, 32 w + 32).
// One thread per 32 codes: 32 codes of b bits fill exactly b words, so every thread owns
// whole output words and no two threads touch the same word.
#include "kernels.h"

namespace gptq {

__global__ void k_pack(const uint8_t* __restrict__ codes, int m, int d, int bits,
                       uint32_t* __restrict__ packed, int wpr) {
  pdl_wait();
  pdl_release();
  const int chunks = (d + 31) / 32;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)m * chunks) return;
  const int r = (int)(t / chunks), ch = (int)(t % chunks);
  const int k0 = ch * 32, n = min(32, d - k0);
  const uint32_t mask = (1u << bits) - 1u;
  const uint8_t* src = codes + (long long)r * d + k0;
  uint32_t* dst = packed + (long long)r * wpr + (long long)ch * bits;
  uint8_t v[32];
  if (n == 32 && ((reinterpret_cast<uintptr_t>(src) & 15) == 0)) {
    uint4 a = reinterpret_cast<const uint4*>(src)[0];
    uint4 b = reinterpret_cast<const uint4*>(src)[1];
    *reinterpret_cast<uint4*>(&v[0]) = a;
    *reinterpret_cast<uint4*>(&v[16]) = b;
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = (q < n) ? src[q] : 0;
  }
  unsigned long long acc = 0;
  int nacc = 0, wout = 0;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    if (q < n) {
      acc |= (unsigned long long)(v[q] & mask) << nacc;
      nacc += bits;
      if (nacc >= 32) {
        dst[wout++] = (uint32_t)acc;
        acc >>= 32;
        nacc -= 32;
      }
    }
  }
  if (nacc > 0) dst[wout] = (uint32_t)acc;
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
  const long long threads = (long long)m * ((d + 31) / 32);
  GPTQ_LAUNCH(c, k_pack, (int)((threads + 255) / 256), 256, 0, codes, m, d, bits, packed, wpr);
  return GPTQ_OK;
}

int unpack_codes(Ctx* c, const uint32_t* packed, int m, int d, int bits, uint8_t* codes) {
  const int wpr = (int)(((long long)d * bits + 31) / 32);
  const long long threads = (long long)m * ((d + 31) / 32);
  GPTQ_LAUNCH(c, k_unpack, (int)((threads + 255) / 256), 256, 0, packed, m, d, bits, codes, wpr);
  return GPTQ_OK;
}

}  // namespace gptq
