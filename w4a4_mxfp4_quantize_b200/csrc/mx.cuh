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
// Every kernel gives each thread whole 32-element blocks (act_block: the
// rotation and the block amax stay in its registers).
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

// Reciprocals 1/D of one 256-wide K tile in shared memory: blocks 36 floats
// apart, so each block starts on a 16-byte boundary and a warp's 16-byte loads of
// the same element of the eight blocks cover all 32 banks once.
constexpr int kQRcpStride = kBlk + 4;
constexpr int kQRcpTile = 8 * kQRcpStride;
__host__ __device__ constexpr int qrcp_index(int k) { return (k >> 5) * kQRcpStride + (k & 31); }

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

// ---- packed two-lane FP32 arithmetic (sm_100 f32x2 through CUDA's float2
// intrinsics): each lane one IEEE rounding to nearest, never contracted ----
__device__ __forceinline__ float2 f2(float lo, float hi) { return make_float2(lo, hi); }
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as a + (-b): the negation is exact, so the sum is the IEEE difference
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) { return __fadd2_rn(a, make_float2(-b.x, -b.y)); }
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
// Round both lanes to bf16 (nearest-even); low lane in the low half.
__device__ __forceinline__ uint32_t f2_to_bf16x2(float2 v) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(v.y), "f"(v.x));
  return r;
}
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// Four lane pairs -> eight E2M1 codes in one word, element 0 in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8_f2(float2 a, float2 b, float2 c, float2 d) {
  return e2m1x8(a.x, a.y, b.x, b.y, c.x, c.y, d.x, d.y);
}

// The 32 reciprocals of one block (16-byte aligned, e.g. in shared memory) as
// 16 lane pairs: pair j holds channels 2j and 2j + 1.
__device__ __forceinline__ void load_rcp_block(const float* __restrict__ r, float2 (&r2)[16]) {
  const uint4* r4 = reinterpret_cast<const uint4*>(r);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 rq = r4[i];  // four reciprocals per 16-byte load
    r2[2 * i] = f2(__uint_as_float(rq.x), __uint_as_float(rq.y));
    r2[2 * i + 1] = f2(__uint_as_float(rq.z), __uint_as_float(rq.w));
  }
}

// Activation block: 32 bf16 values (four 16-byte words) and the 32
// reciprocals r = RN32(1/D) of their channels as lane pairs (load_rcp_block).
// Same arithmetic as the scalar definition, two lanes per instruction:
//   xs = RNE_bf16(RN32(x * r)); FP32 butterfly h = 1, 2, 4, 8, 16;
//   u = RNE_bf16(.); E8M0 from the block amax of |u|; E2M1 of u * 2^(127-c).
__device__ __forceinline__ void act_block(const uint4 (&xv)[4], const float2 (&r2)[16], uint4& codes,
                                          uint32_t& scale) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(xv);
  float2 P[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t xs = f2_to_bf16x2(f2_mul(bf16x2_to_f2(w[j]), r2[j]));  // channel scaling, BF16
    // butterfly stage h = 1 inside the pair: (v0 + v1, v0 - v1)
    const float v0 = bf16lo(xs), v1 = bf16hi(xs);
    P[j] = f2(__fadd_rn(v0, v1), __fsub_rn(v0, v1));
  }
  // stages h = 2, 4, 8, 16: pairs of pairs (P[i], P[i + h/2])
#pragma unroll
  for (int hp = 1; hp < 16; hp <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & hp) continue;
      const float2 a = P[i], b = P[i + hp];
      P[i] = f2_add(a, b);
      P[i + hp] = f2_sub(a, b);
    }
  }
  uint32_t u[16];
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    u[j] = f2_to_bf16x2(P[j]);
    m = max_u16x2(m, u[j] & 0x7FFF7FFFu);
  }
  const uint32_t amax16 = max(m & 0xFFFFu, m >> 16);
  const uint32_t c = e8m0_from_amax_bits(amax16 << 16);
  const float s = __uint_as_float((254u - min(c, 253u)) << 23);
  const float2 s2 = f2(s, s);
  uint32_t out[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    out[q] = e2m1x8_f2(f2_mul(bf16x2_to_f2(u[4 * q]), s2), f2_mul(bf16x2_to_f2(u[4 * q + 1]), s2),
                       f2_mul(bf16x2_to_f2(u[4 * q + 2]), s2), f2_mul(bf16x2_to_f2(u[4 * q + 3]), s2));
  codes = make_uint4(out[0], out[1], out[2], out[3]);
  scale = c;
}

// Plain MXFP4 (no D, no Hadamard): the block's BF16 values are encoded as they
// are.  amax over |x| in BF16 (exact), E8M0 and E2M1 as in act_block.
__device__ __forceinline__ void act_block_plain(const uint4 (&xv)[4], uint4& codes, uint32_t& scale) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(xv);
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) m = max_u16x2(m, w[j] & 0x7FFF7FFFu);
  const uint32_t amax16 = max(m & 0xFFFFu, m >> 16);
  const uint32_t c = e8m0_from_amax_bits(amax16 << 16);
  const float s = __uint_as_float((254u - min(c, 253u)) << 23);
  const float2 s2 = f2(s, s);
  uint32_t out[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    out[q] = e2m1x8_f2(f2_mul(bf16x2_to_f2(w[4 * q]), s2), f2_mul(bf16x2_to_f2(w[4 * q + 1]), s2),
                       f2_mul(bf16x2_to_f2(w[4 * q + 2]), s2), f2_mul(bf16x2_to_f2(w[4 * q + 3]), s2));
  codes = make_uint4(out[0], out[1], out[2], out[3]);
  scale = c;
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
