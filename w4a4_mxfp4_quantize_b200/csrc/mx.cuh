// Per-block arithmetic of the MACAQ activation prologue and of the offline
// weight preparation, and the shared-memory operand image layout.
//
// Steps (MACAQ page, summary; latency section for the MX rule):
//   activations: r = RN32(1/D); xs = RNE_bf16(RN32(x*r));
//                u = RNE_bf16(FWHT32(xs)) (FP32 butterfly, order h = 1..16);
//   weights:     t = FWHT32(RN32(W*D)) in FP32 (offline, no BF16 rounding);
//   both:        E8M0 scale = floor(log2 amax) - 2 + 127 clamped at 0
//                (OCP MX scale_alg = 0); E2M1 code = RNE with saturation of
//                value * 2^(127 - scale); sign bit copied from the value.
// One thread owns one 32-element block, so the whole rotation and the block
// amax stay in registers (no shuffles, no shared memory).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace macaq {

constexpr int kBlk = 32;         // elements per MX block
constexpr int kKTile = 256;      // K elements per operand tile row (128 bytes of E2M1)
constexpr int kRowsTile = 128;   // rows per operand tile image
constexpr int kTileCodeBytes = kRowsTile * kKTile / 2;  // 16384
constexpr int kTileSfBytes = kRowsTile * kKTile / kBlk; // 1024

// Byte offset of the 16-byte code chunk of (row r, block c) inside a 128-row x
// 256-K operand image: rows of 128 bytes, chunk index XOR-swizzled with r mod 8
// (the 128-byte swizzle the tensor core's K-major descriptor expects).
__host__ __device__ __forceinline__ uint32_t code_chunk_offset(uint32_t r, uint32_t c) {
  return r * 128u + ((c ^ (r & 7u)) << 4);
}
// Byte offset of the E8M0 scale of (row r, block c) in the 1024-byte scale
// image of the same tile: two 512-byte groups of four K-blocks; inside one,
// row r sits at 16*(r mod 32) + 4*(r / 32), one byte per K-block.
__host__ __device__ __forceinline__ uint32_t sf_offset(uint32_t r, uint32_t c) {
  return (c >> 2) * 512u + (r & 31u) * 16u + (r >> 5) * 4u + (c & 3u);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round two floats to bf16 (nearest-even) and return them widened back.
__device__ __forceinline__ void round_pair_bf16(float& a, float& b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // .x = a (low half), .y = b
  uint32_t w = *reinterpret_cast<uint32_t*>(&h);
  a = bf16lo(w);
  b = bf16hi(w);
}

// Unnormalised Walsh-Hadamard transform of 32 floats; each output of each
// stage is one IEEE binary32 rounding (no contraction possible: no products).
__device__ __forceinline__ void fwht32(float (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i & h) continue;
      const float a = v[i], b = v[i + h];
      v[i] = __fadd_rn(a, b);
      v[i + h] = __fsub_rn(a, b);
    }
  }
}

// Eight values -> eight E2M1 codes in one 32-bit word, element 0 in the
// lowest nibble.  cvt puts its first source operand in the high nibble.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return out;
}

// E8M0 code from the bit pattern of a non-negative float amax:
// floor(log2 amax) + 127 is the biased exponent field e (0 for zero and
// subnormals, which clamp to 0 anyway); minus emax(E2M1) = 2.
__device__ __forceinline__ uint32_t e8m0_from_amax_bits(uint32_t amax_bits) {
  const uint32_t e = amax_bits >> 23;  // sign is clear
  if (e == 0xFFu) return 0xFFu;        // non-finite input (precondition violated)
  return e >= 2u ? e - 2u : 0u;
}

// MX-encode a block already in registers: 16 code bytes (element 2j in the low
// nibble of byte j) and the E8M0 scale.
__device__ __forceinline__ void mx_encode_block(const float (&u)[32], uint4& codes, uint32_t& scale) {
  uint32_t amax = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = max(amax, __float_as_uint(u[i]) & 0x7FFFFFFFu);
  const uint32_t c = e8m0_from_amax_bits(amax);
  // 2^(127 - c) for c in [0, 252] is a normal float; multiplying by it is exact
  // except where the product falls below 2^-126, far under the code-0 bound.
  const float s = __uint_as_float((254u - min(c, 253u)) << 23);
  float q[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) q[i] = __fmul_rn(u[i], s);
  codes.x = e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
  codes.y = e2m1x8(q[8], q[9], q[10], q[11], q[12], q[13], q[14], q[15]);
  codes.z = e2m1x8(q[16], q[17], q[18], q[19], q[20], q[21], q[22], q[23]);
  codes.w = e2m1x8(q[24], q[25], q[26], q[27], q[28], q[29], q[30], q[31]);
  scale = c;
}

// Activation block: 32 bf16 values (four 16-byte words) and the 32
// reciprocals r = RN32(1/D) of their channels.
__device__ __forceinline__ void act_block(const uint4 (&xv)[4], const float* __restrict__ r, uint4& codes,
                                          uint32_t& scale) {
  float v[32];
  const uint32_t* w = reinterpret_cast<const uint32_t*>(xv);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float a = __fmul_rn(bf16lo(w[j]), r[2 * j]);
    float b = __fmul_rn(bf16hi(w[j]), r[2 * j + 1]);
    round_pair_bf16(a, b);
    v[2 * j] = a;
    v[2 * j + 1] = b;
  }
  fwht32(v);
#pragma unroll
  for (int j = 0; j < 16; ++j) round_pair_bf16(v[2 * j], v[2 * j + 1]);
  mx_encode_block(v, codes, scale);
}

// Weight block: 32 fp32 weights and their 32 channel factors D (offline).
__device__ __forceinline__ void weight_block(const float (&wv)[32], const float (&dv)[32], uint4& codes,
                                             uint32_t& scale) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(wv[i], dv[i]);
  fwht32(v);
  mx_encode_block(v, codes, scale);
}

}  // namespace macaq
