// nf4_device.cuh -- device helpers shared by the codec and GEMM kernels:
// bf16 / E4M3 unpacking, the two-level block constant, and the byte-permute
// expansion of packed NF4 codes into bf16 (a 16-entry table per 64-block).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace qlora {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// E4M3 ("fn") byte -> float, exact (every E4M3 value is a float).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float v = (e == 0) ? __int2float_rn(static_cast<int>(m)) * 0.001953125f            // m * 2^-9
                     : __uint_as_float(((e + 120u) << 23) | (m << 20));              // (1+m/8) 2^(e-7)
  if (e == 15 && m == 7) v = __uint_as_float(0x7FC00000u);
  return (b & 0x80u) ? -v : v;
}

// Builds the 16-entry bf16 table T[c] = bf16(L[c] * c1') of a block, split
// into byte planes so that a byte-permute picks four entries at once.
struct ByteTables {
  uint32_t ha0, ha1, hb0, hb1;   // high bytes of T[0..3], T[4..7], T[8..11], T[12..15]
  uint32_t la0, la1, lb0, lb1;   // low bytes, same grouping
};

__device__ __forceinline__ ByteTables make_tables(const float* L, float c1p) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const __nv_bfloat162 t = __floats2bfloat162_rn(__fmul_rn(L[2 * j], c1p), __fmul_rn(L[2 * j + 1], c1p));
    p[j] = *reinterpret_cast<const uint32_t*>(&t);        // T[2j] low half, T[2j+1] high half
  }
  ByteTables b;
  b.ha0 = __byte_perm(p[0], p[1], 0x7531); b.la0 = __byte_perm(p[0], p[1], 0x6420);
  b.ha1 = __byte_perm(p[2], p[3], 0x7531); b.la1 = __byte_perm(p[2], p[3], 0x6420);
  b.hb0 = __byte_perm(p[4], p[5], 0x7531); b.lb0 = __byte_perm(p[4], p[5], 0x6420);
  b.hb1 = __byte_perm(p[6], p[7], 0x7531); b.lb1 = __byte_perm(p[6], p[7], 0x6420);
  return b;
}

// Four codes (the 16 low bits of `w16`, nibble k -> output byte k) -> two
// bf16x2 words in element order.  Nibble k holds element k^1 (high nibble first).
__device__ __forceinline__ void lookup4(uint32_t w16, const ByteTables& t, uint32_t& out01,
                                        uint32_t& out23) {
  const uint32_t s = w16 & 0x7777u;                          // low 3 bits of each code
  const uint32_t s2 = ((w16 >> 1) & 0x4444u) | 0x3210u;      // bit 3 picks the upper table
  const uint32_t h = __byte_perm(__byte_perm(t.ha0, t.ha1, s), __byte_perm(t.hb0, t.hb1, s), s2);
  const uint32_t l = __byte_perm(__byte_perm(t.la0, t.la1, s), __byte_perm(t.lb0, t.lb1, s), s2);
  out01 = __byte_perm(l, h, 0x4051);   // element 0 (nibble 1), element 1 (nibble 0)
  out23 = __byte_perm(l, h, 0x6273);   // element 2 (nibble 3), element 3 (nibble 2)
}

// The two byte-permute stages of lookup4 given their selectors: s holds the
// low 3 bits of each code (table half index), s2 picks the half by code bit 3.
__device__ __forceinline__ void lookup4_sel(uint32_t s, uint32_t s2, const ByteTables& t, uint32_t& out01,
                                            uint32_t& out23) {
  const uint32_t h = __byte_perm(__byte_perm(t.ha0, t.ha1, s), __byte_perm(t.hb0, t.hb1, s), s2);
  const uint32_t l = __byte_perm(__byte_perm(t.la0, t.la1, s), __byte_perm(t.lb0, t.lb1, s), s2);
  out01 = __byte_perm(l, h, 0x4051);
  out23 = __byte_perm(l, h, 0x6273);
}

// Eight codes -> four bf16x2 words: the selectors of all eight codes are
// built at once (byte-permute reads only the low 16 bits of a selector).
__device__ __forceinline__ uint4 expand8(uint32_t w, const ByteTables& t) {
  const uint32_t s = w & 0x77777777u;
  const uint32_t s2 = ((w >> 1) & 0x44444444u) | 0x32103210u;
  uint4 o;
  lookup4_sel(s, s2, t, o.x, o.y);
  lookup4_sel(s >> 16, s2 >> 16, t, o.z, o.w);
  return o;
}

__device__ __forceinline__ float block_constant(uint32_t qbyte, float c2_over_448, float mu) {
  return __fmaf_rn(e4m3_to_f32(qbyte), c2_over_448, mu);
}

}  // namespace qlora
