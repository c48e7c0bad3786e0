// Device helpers shared by the tensor-core decode and prefill kernels:
// 16-channel value groups dequantised straight to fp16 pairs, and a fast exp2.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace starkv {

// ---------------------------------------------------------------------------
// 16-channel value group of one token -> fp16 z_hat = code * s + zp, as two
// 16-byte chunks.  Codes become fp16 (1024 + code) by OR-ing them under the
// exponent of 1024 (0x6400); subtracting 1024 is exact, and one half2 fma
// applies the scale and zero.  The pairs come out as (c, c+4) per nibble word
// and (c, c+8) per 3-bit plane, so the 16 positions hold channels
//   4-bit: 0 4 1 5 2 6 3 7 | 8 12 9 13 10 14 11 15
//   3-bit: 0 8 1 9 2 10 3 11 | 4 12 5 13 6 14 7 15
// (value_channel_of_position undoes this).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ void scale_zero(uint32_t mw, __half2& s2, __half2& z2) {
  s2 = bits2h(__byte_perm(mw, mw, 0x1010));
  z2 = bits2h(__byte_perm(mw, mw, 0x3232));
}

__device__ __forceinline__ uint32_t deq_pair(uint32_t magic_bits, __half2 s2, __half2 z2) {
  const __half2 k1024 = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
  return h2bits(__hfma2(__hsub2(bits2h(magic_bits), k1024), s2, z2));
}

__device__ __forceinline__ void dequant16_4bit(const uint8_t* p, uint32_t mw, uint4& c0, uint4& c1) {
  __half2 s2, z2;
  scale_zero(mw, s2, z2);
  const uint2 w = *reinterpret_cast<const uint2*>(p);
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[i] = deq_pair(((w.x >> (4 * i)) & 0x000F000Fu) | 0x64006400u, s2, z2);
    o[4 + i] = deq_pair(((w.y >> (4 * i)) & 0x000F000Fu) | 0x64006400u, s2, z2);
  }
  c0 = make_uint4(o[0], o[1], o[2], o[3]);
  c1 = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ void dequant16_3bit(const uint8_t* tile, int t16, uint32_t mw, uint4& c0, uint4& c1) {
  __half2 s2, z2;
  scale_zero(mw, s2, z2);
  const uint32_t lo = *reinterpret_cast<const uint32_t*>(tile + 4 * t16);
  const uint32_t hi16 = *reinterpret_cast<const uint16_t*>(tile + 64 + 2 * t16);
  const uint32_t hs = __byte_perm(hi16, 0u, 0x4140);  // bits 0-7 stay, bits 8-15 -> 16-23
  uint32_t o[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t l = ((lo >> (2 * c)) & 0x00030003u) | 0x64006400u;
    const uint32_t h = (c >= 2 ? (hs >> (c - 2)) : (hs << (2 - c))) & 0x00040004u;
    o[c] = deq_pair(l | h, s2, z2);
  }
  c0 = make_uint4(o[0], o[1], o[2], o[3]);
  c1 = make_uint4(o[4], o[5], o[6], o[7]);
}

__host__ __device__ __forceinline__ int value_channel_of_position(int p, bool top) {
  const int k = p >> 3, e = p & 7;
  return top ? 8 * k + (e >> 1) + 4 * (e & 1) : 4 * k + (e >> 1) + 8 * (e & 1);
}


// 2^x on the special-function unit (relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace starkv
