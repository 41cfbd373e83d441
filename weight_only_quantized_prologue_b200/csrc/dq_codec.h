// dq_codec.h -- scalar number-format codecs and the per-group / per-block
// weight quantizers, compiled both for the host packer and for the GPU
// packer so the two are bit-identical.  All arithmetic is IEEE fp32 with
// round-to-nearest-even (explicit __fdiv_rn / __fmul_rn on the device; the
// host build uses SSE fp32 and no FMA contraction).
//
// Formats: E2M1 (bias 1, values 0, .5, 1, 1.5, 2, 3, 4, 6), E4M3 "fn" (bias 7,
// max 448, S.1111.111 NaN), E8M0 (2^(e-127)), bf16, as named on the NVFP4,
// MXFP4 and FP8 tutorial pages (intro sections).
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define DQ_HD __host__ __device__ __forceinline__
#else
#define DQ_HD inline
#endif

namespace dq {

DQ_HD float fdiv(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fdiv_rn(a, b);
#else
  volatile float r = a / b;   // keep it an fp32 division
  return r;
#endif
}
DQ_HD float fmul(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);
#else
  volatile float r = a * b;
  return r;
#endif
}
DQ_HD float frint(float a) {   // round half to even
#if defined(__CUDA_ARCH__)
  return rintf(a);
#else
  return nearbyintf(a);
#endif
}
DQ_HD uint32_t f2u(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}
DQ_HD float u2f(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// fp32 -> bf16 bits, round to nearest even; NaN stays a quiet NaN.
DQ_HD uint16_t bf16_bits_rn(float f) {
  uint32_t u = f2u(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
DQ_HD float bf16_to_f(uint16_t b) { return u2f((uint32_t)b << 16); }

// floor(log2(a)) for finite a > 0, exact (subnormals included).
DQ_HD int ilog2f(float a) {
  const uint32_t u = f2u(a);
  const int e = (int)((u >> 23) & 0xFF);
  if (e) return e - 127;
  uint32_t m = u & 0x7FFFFFu;   // subnormal: value = m * 2^-149
  int l = -150;
  while (m) { m >>= 1; ++l; }
  return l;
}

DQ_HD float pow2f(int e) {   // 2^e for -149 <= e <= 127, exact
  if (e >= -126) return u2f((uint32_t)(e + 127) << 23);
  return u2f(1u << (e + 149));
}

// E4M3: saturating round to nearest even; the sign is kept (-0 -> 0x80).
DQ_HD uint8_t e4m3_encode_sat(float v) {
  const uint32_t sign = (f2u(v) >> 24) & 0x80u;
  const float a = fabsf(v);
  if (a != a) return 0x7F;
  if (a >= 448.f) return (uint8_t)(sign | 0x7E);
  if (a < 0x1p-6f) return (uint8_t)(sign | (uint32_t)frint(fmul(a, 512.f)));   // 0..8 (8 = 2^-6)
  const int E = ilog2f(a);                                                      // -6..8
  const float m = fmul(a, pow2f(-E)) - 1.f;                                      // [0, 1), exact
  const uint32_t n = (uint32_t)frint(m * 8.f);                                   // 0..8 (carry ok)
  return (uint8_t)(sign | ((uint32_t)((E + 7) << 3) + n));
}
DQ_HD float e4m3_decode(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  float v = e ? fmul(pow2f(e - 7), 1.f + m * 0.125f) : m * 0x1p-9f;
  if ((c & 0x7F) == 0x7F) v = u2f(0x7FC00000u);
  return (c & 0x80) ? -v : v;
}

// E2M1: saturating round to nearest even; the sign is kept (-0 -> 0x8).
DQ_HD uint8_t e2m1_encode_sat(float v) {
  const uint32_t sign = (f2u(v) >> 28) & 0x8u;
  const float a = fabsf(v);
  if (a >= 6.f) return (uint8_t)(sign | 7u);
  if (a < 1.f) return (uint8_t)(sign | (uint32_t)frint(a * 2.f));       // 0, 1, or 2 (= 1.0)
  const int E = ilog2f(a);                                              // 0..2
  const float m = fmul(a, pow2f(-E)) - 1.f;
  const uint32_t n = (uint32_t)frint(m * 2.f);                          // 0..2 (carry ok)
  return (uint8_t)(sign | ((uint32_t)((E + 1) << 1) + n));
}
DQ_HD float e2m1_decode(uint8_t c) {
  const int mag = c & 7, e = mag >> 1, m = mag & 1;
  const float v = e ? pow2f(e - 1) * (1.f + 0.5f * m) : 0.5f * m;
  return (c & 8) ? -v : v;
}

// ---------------------------------------------------------------------------
// quantizers of one group / block (elements at w[0..n), stride 1)
// ---------------------------------------------------------------------------

// INT4 symmetric, zero-point 0: s = bf16(amax/7), c = clamp(rne(w/s), -8, 7).
// Writes n codes (int8) and returns the scale's bf16 bits.
DQ_HD uint16_t quant_int4_group(const float* w, int n, int8_t* codes) {
  float a = 0.f;
  for (int i = 0; i < n; ++i) a = fmaxf(a, fabsf(w[i]));
  const uint16_t sb = bf16_bits_rn(fdiv(a, 7.f));
  const float s = bf16_to_f(sb);
  for (int i = 0; i < n; ++i) {
    float q = s > 0.f ? frint(fdiv(w[i], s)) : 0.f;
    q = q < -8.f ? -8.f : (q > 7.f ? 7.f : q);
    codes[i] = (int8_t)q;
  }
  return sb;
}

// INT4 asymmetric: lo = min(0, min w), hi = max(0, max w),
// s = bf16((hi - lo)/15), z = clamp(rne(-lo/s), 0, 15),
// c = clamp(rne(w/s) + z, 0, 15) (unsigned); a group with s == 0 has codes
// 0 and z 0.  Writes n codes and *zero, returns the scale's bf16 bits.
DQ_HD uint16_t quant_int4_asym_group(const float* w, int n, uint8_t* codes, uint8_t* zero) {
  float lo = 0.f, hi = 0.f;
  for (int i = 0; i < n; ++i) {
    lo = fminf(lo, w[i]);
    hi = fmaxf(hi, w[i]);
  }
  const uint16_t sb = bf16_bits_rn(fdiv(hi - lo, 15.f));
  const float s = bf16_to_f(sb);
  float z = 0.f;
  if (s > 0.f) {
    z = frint(fdiv(-lo, s));
    z = z < 0.f ? 0.f : (z > 15.f ? 15.f : z);
  }
  for (int i = 0; i < n; ++i) {
    float q = s > 0.f ? frint(fdiv(w[i], s)) + z : 0.f;
    q = q < 0.f ? 0.f : (q > 15.f ? 15.f : q);
    codes[i] = (uint8_t)q;
  }
  *zero = (uint8_t)z;
  return sb;
}

DQ_HD float nvfp4_global_scale(float amax) { return amax > 0.f ? fdiv(amax, 2688.f) : 1.f; }

// NVFP4 block of 16: sb = e4m3((amax/6)/g), c = e2m1(w / (dec(sb)*g)).
DQ_HD uint8_t quant_nvfp4_block(const float* w, int n, float g, uint8_t* codes) {
  float a = 0.f;
  for (int i = 0; i < n; ++i) a = fmaxf(a, fabsf(w[i]));
  const uint8_t sb = e4m3_encode_sat(fdiv(fdiv(a, 6.f), g));
  const float d = fmul(e4m3_decode(sb), g);
  for (int i = 0; i < n; ++i) codes[i] = d > 0.f ? e2m1_encode_sat(fdiv(w[i], d)) : 0;
  return sb;
}

// MXFP4 block of 32: e = floor(log2 amax) - 2 in [-127, 127], code e + 127
// (0 for a zero block), c = e2m1(w * 2^-e).
DQ_HD uint8_t quant_mxfp4_block(const float* w, int n, uint8_t* codes) {
  float a = 0.f;
  for (int i = 0; i < n; ++i) a = fmaxf(a, fabsf(w[i]));
  if (!(a > 0.f)) {
    for (int i = 0; i < n; ++i) codes[i] = 0;
    return 0;
  }
  int e = ilog2f(a) - 2;
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  for (int i = 0; i < n; ++i) {
    // w * 2^-e in two exact steps (2^-e may not be an fp32 normal)
    const int e1 = -e > 127 ? 127 : -e;
    const float t = fmul(fmul(w[i], pow2f(e1)), pow2f(-e - e1));
    codes[i] = e2m1_encode_sat(t);
  }
  return (uint8_t)(e + 127);
}

// FP8 per channel: s = max(|min|, |max|)/448, c = e4m3(w/s); zero row -> 0.
DQ_HD float quant_fp8_row(const float* w, int n, uint8_t* codes) {
  float a = 0.f;
  for (int i = 0; i < n; ++i) a = fmaxf(a, fabsf(w[i]));
  const float s = fdiv(a, 448.f);
  for (int i = 0; i < n; ++i) codes[i] = s > 0.f ? e4m3_encode_sat(fdiv(w[i], s)) : 0;
  return s;
}

}  // namespace dq
