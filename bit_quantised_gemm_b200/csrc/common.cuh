// Shared definitions for the BitLinear kernels: launch parameters, the
// ternary-weight unpack, and small numeric helpers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace blt {

constexpr float kEps = 1e-5f;  // floor of every absmax scale

// ----------------------------------------------------------- bf16 helpers
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// Integer code of one activation: clamp(rne(h * inv), lo, hi), fp32 multiply.
// The rounding runs on the FMA pipe rather than the quarter-rate conversion
// unit: for |v| < 2^22, v + 1.5 * 2^23 rounds v to the nearest integer (ties
// to even) and that integer is the low bits of the sum. Every caller has
// |h * inv| <= Q (1 + 2^-23) with Q <= 127 (|h| never exceeds the absmax
// its scale comes from).
__device__ __forceinline__ int quant_code(float h, float inv, float lo, float hi) {
  const float r = __fadd_rn(__fmul_rn(h, inv), 12582912.f);
  const int c = __float_as_int(r) - 0x4B400000;
  return min(max(c, static_cast<int>(lo)), static_cast<int>(hi));
}

// v <- fl(fl(v * s) + bias) for both values: two IEEE roundings each. The
// products come from one paired fp32 multiply; the adds stay scalar IEEE adds,
// which are never contracted with it into a fused multiply-add (a fused
// x * s + bias rounds once and can land on the other integer at a .5 tie).
__device__ __forceinline__ void mul_then_add_rn(float& lo, float& hi, float s, float bias) {
  const float2 p = __fmul2_rn(make_float2(lo, hi), make_float2(s, s));
  lo = __fadd_rn(p.x, bias);
  hi = __fadd_rn(p.y, bias);
}

__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

// h of the activation quantisers: x, or the ReLU^2-gated product
// (r * r) * up with r = max(x, 0), both multiplies in fp32.
__device__ __forceinline__ void act_vals8(const uint4& xv, const uint4& uv, bool relu2, float (&h)[8]) {
  bf16x8_to_f32(xv, h);
  if (relu2) {
    float u[8];
    bf16x8_to_f32(uv, u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float r = h[i] > 0.f ? h[i] : 0.f;
      h[i] = __fmul_rn(__fmul_rn(r, r), u[i]);
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------------------ ternary unpacking
// A 32-bit word of the packed weights holds 16 consecutive k: element 8h+i
// sits in bits [4i+2h, 4i+2h+2) as code c = w + 1 (0, 1, 2). Masking with
// 0x33333333 after a shift of 2h leaves one code per nibble, which PRMT
// then uses as a byte selector into a 4-entry lookup table.
__device__ __forceinline__ uint32_t codes_lo(uint32_t w) { return w & 0x33333333u; }
__device__ __forceinline__ uint32_t codes_hi(uint32_t w) { return (w >> 2) & 0x33333333u; }

// 16 weights -> 16 signed int8 bytes in k order (-1 -> 0xFF, 0, +1 -> 0x01).
__device__ __forceinline__ uint4 unpack16_s8(uint32_t w) {
  constexpr uint32_t kLut = 0x000100FFu;  // code 0 -> -1, 1 -> 0, 2 -> +1, 3 -> 0
  const uint32_t x0 = codes_lo(w), x1 = codes_hi(w);
  uint4 o;
  o.x = __byte_perm(kLut, 0u, x0);
  o.y = __byte_perm(kLut, 0u, x0 >> 16);
  o.z = __byte_perm(kLut, 0u, x1);
  o.w = __byte_perm(kLut, 0u, x1 >> 16);
  return o;
}

// 16 weights -> two words of 8 e2m1 nibbles each (elements 0-7 and 8-15,
// even k in the low nibble): code 0 -> 0xA (-1.0), 1 -> 0x0, 2 -> 0x2 (+1.0).
// Eight logic ops: for the code bits (c1 c0) of element 8h + i, nibble i of
// the result gets bit 1 = !c0 (a non-zero weight) and bit 3 = !c0 & !c1
// (weight -1). For h = 0 those bits sit 1 and 3 places above c0 and 2 above
// c1; for h = 1, 1 below and 1 above c0 and at c1 itself.
__device__ __forceinline__ void e2m1_words(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t t1 = w << 1, t2 = w << 2, t3 = w << 3, r1 = w >> 1;
  lo = (~t1 & 0x22222222u) | (~t3 & ~t2 & 0x88888888u);
  hi = (~r1 & 0x22222222u) | (~t1 & ~w & 0x88888888u);
}

// 16 weights -> one 16-byte e2m1 group in the padded shared-memory form the
// f8f6f4 MMA reads: 16 nibbles (even k low) in the first 8 bytes, 8 zero bytes.
__device__ __forceinline__ uint4 unpack16_e2m1(uint32_t w) {
  uint4 o;
  e2m1_words(w, o.x, o.y);
  o.z = 0u;
  o.w = 0u;
  return o;
}

// --------------------------------------------------------- status words
__device__ __forceinline__ void report_status(int* status, int code) {
  if (status) atomicOr(status, code);
}

}  // namespace blt
