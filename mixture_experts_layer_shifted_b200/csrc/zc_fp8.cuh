// Block-scaled FP8 helpers shared by the quantizers and the FP8 GEMM.
//
// LongCat-Flash technical summary (zhangjingwei.cn), 六 推理與部署, 定制內核
// "量化": DeepSeek-V3's fine-grained block quantization, one scale per [1,128]
// block of activations and per [128,128] block of weights.  Codes are FP8 E4M3
// (round to nearest even, saturating at 448); a block's scale is the smallest
// power of two 2^E with amax <= 448 * 2^E, stored as the E8M0 byte E + 127
// (clamped to [0, 254]; an all-zero block takes 2^0), which is the scale format
// the tensor cores' block-scaled MMA reads.
//
// Scale atoms.  The block-scaled MMA takes its scales from tensor memory, one
// byte per operand row per 32-deep K slice; tcgen05.cp (32x128b, broadcast to
// the four lane quarters) fills them from a 512-byte shared-memory atom that
// holds 128 operand rows x 4 K-blocks: byte 16*(r%32) + 4*(r/32) + j is the
// scale of row r in the j-th 128-deep K-block of the atom.  Scales are stored in
// global memory as these atoms, atom (R, G) covering rows [128R, 128R+128) and
// K-blocks [4G, 4G+4), at byte offset (R * groups + G) * 512.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace zc {

constexpr int kAtomBytes = 512;

// E8M0 code of a block's largest magnitude (amax >= 0, finite).
__device__ __forceinline__ uint32_t e8m0_code(float amax) {
  const uint32_t b = __float_as_uint(amax);
  if (b == 0u) return 127u;
  const int ef = (int)(b >> 23);
  if (ef == 0) return 0u;  // subnormal block maximum: the smallest scale suffices
  const int k = ef - 127;  // amax in [2^k, 2^(k+1))
  // 448 = 1.75 * 2^8: amax <= 1.75 * 2^k  <=>  mantissa fraction <= 0.75
  const int E = ((b & 0x7FFFFFu) <= 0x600000u) ? k - 8 : k - 7;
  const int c = E + 127;
  return (uint32_t)(c < 0 ? 0 : (c > 254 ? 254 : c));
}

// 2^(127 - code) as fp32 (code <= 253).
__device__ __forceinline__ float e8m0_inverse(uint32_t code) { return __uint_as_float((254u - code) << 23); }

// Four E4M3 codes packed little-endian (byte i = code of v_i).
__device__ __forceinline__ uint32_t pack_e4m3x4(float v0, float v1, float v2, float v3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(v1), "f"(v0));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(v3), "f"(v2));
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

// ---------------------------------------------------------------- W4A4 (MXFP4)
// A LongCat-Flash news page (gate.com post) reports W4A4 serving (expert
// weights and activations in 4 bits) without naming the format; here MXFP4:
// E2M1 codes (0, 0.5, 1, 1.5, 2, 3, 4, 6), round to nearest even, saturating;
// one E8M0 scale per 32 elements along K, the smallest 2^E with amax <= 6 * 2^E.
// Two codes per byte, the even element in the low nibble.  Scale atoms as above
// with j indexing the 32-element blocks of a 128-element K group (so `kb` in
// atom_offset is the 32-block index and `groups` = ceil(K / 128)).

__device__ __forceinline__ uint32_t mx4_code(float amax) {
  const uint32_t b = __float_as_uint(amax);
  if (b == 0u) return 127u;
  const int ef = (int)(b >> 23);
  if (ef == 0) return 0u;
  const int k = ef - 127;
  // 6 = 1.5 * 2^2: amax <= 1.5 * 2^k  <=>  mantissa fraction <= 0.5
  const int E = ((b & 0x7FFFFFu) <= 0x400000u) ? k - 2 : k - 1;
  const int c = E + 127;
  return (uint32_t)(c < 0 ? 0 : (c > 254 ? 254 : c));
}

// Two E2M1 codes in one byte: v_lo in bits 0..3, v_hi in bits 4..7.
__device__ __forceinline__ uint32_t pack_e2m1x2(float v_lo, float v_hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}\n"
      : "=r"(r)
      : "f"(v_hi), "f"(v_lo));
  return r;
}

// Eight E2M1 codes (v[0] lowest nibble) of v * inv.
__device__ __forceinline__ uint32_t pack_e2m1x8(const float* v, float inv) {
  return pack_e2m1x2(v[0] * inv, v[1] * inv) | (pack_e2m1x2(v[2] * inv, v[3] * inv) << 8) |
         (pack_e2m1x2(v[4] * inv, v[5] * inv) << 16) | (pack_e2m1x2(v[6] * inv, v[7] * inv) << 24);
}

// ---------------------------------------------------------------- W4A4 (NVFP4)
// The same E2M1 codes with a finer, two-level scale: one unsigned E4M3 value
// (UE4M3: the positive E4M3 values 2^-9 .. 448) per 16 elements along K and one
// fp32 scale g per tensor (value = code * s * g).  The block scale is the
// smallest UE4M3 value s with amax <= 6 s g, decided in fp32 on
// t = fl32(amax / fl32(6 g)); codes are e2m1(fl32(x * fl32(1 / fl32(s g)))).
// Weights take g = fl32(amax(matrix) / 2688) (so their largest block scale is
// 448), activations g = 1.  Scale atoms as above with j indexing the 16-element
// blocks of a 64-element K group (`groups` = ceil(K / 64)).

// The value of a positive E4M3 code (exact in fp32).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  return e == 0 ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// The smallest positive E4M3 value >= t (t > 0), as its code; 0x7E (448) for t > 448.
__device__ __forceinline__ uint32_t ue4m3_ceil(float t) {
  if (t > 448.0f) return 0x7Eu;
  const uint32_t b = __float_as_uint(t);
  const int ef = (int)(b >> 23);
  if (ef < 121) return (uint32_t)ceilf(t * 512.0f);  // below 2^-6: multiples of 2^-9 (code 8 is 2^-6)
  const uint32_t mant = b & 0x7FFFFFu;
  const uint32_t m3 = (mant >> 20) + ((mant & 0xFFFFFu) != 0u);  // 8 carries into the exponent
  return ((uint32_t)(ef - 120) << 3) + m3;
}

// UE4M3 block-scale code for a block maximum amax (finite, >= 0) under tensor scale g.
__device__ __forceinline__ uint32_t nv4_code(float amax, float g) {
  if (!(amax > 0.0f)) return 0x38u;  // 1.0
  return ue4m3_ceil(__fdiv_rn(amax, __fmul_rn(6.0f, g)));
}

// fl32(1 / fl32(s g)): the multiplier that takes a block's elements to code space.
__device__ __forceinline__ float nv4_inverse(uint32_t code, float g) {
  return __frcp_rn(__fmul_rn(e4m3_value(code), g));
}

// Byte offset of (row, K-block) in a scale-atom array with `groups` atoms per 128 rows.
__host__ __device__ __forceinline__ int64_t atom_offset(int64_t row, int kb, int groups) {
  const int64_t R = row >> 7;
  const int r = (int)(row & 127);
  return (R * groups + (kb >> 2)) * kAtomBytes + 16 * (r & 31) + 4 * (r >> 5) + (kb & 3);
}

}  // namespace zc
