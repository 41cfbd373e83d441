// dq_aux.cuh -- the non-GEMM kernels: debug dequantization through the
// GEMM's own unpack code, the static-FP8 activation quantizer, the GPU weight
// packer, and the bounded-wait self test.
#pragma once

#include "dq_codec.h"
#include "dq_gemm.cuh"

namespace dq {

// ---------------------------------------------------------------------------
// debug dequantization: one CTA per (tile, stage), 256 threads = 128 rows x
// 2 k-halves, exactly the prologue's thread mapping.  The chunk is staged in
// shared memory and unpacked by prologue_stage, then multiplied by the
// epilogue factor of its channel: out = bf16(f32(operand) * sigma_n).
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* wchunks, const float* col_scale, float sigma,
                                                      int mx_bias, int N, int K, int k_stages,
                                                      __nv_bfloat16* out) {
  __shared__ __align__(16) uint8_t chunk[chunk_bytes(FMT)];
  const int t = blockIdx.x, s = blockIdx.y;
  const uint8_t* src = wchunks + ((size_t)t * k_stages + s) * chunk_bytes(FMT);
  for (int i = threadIdx.x * 16; i < chunk_bytes(FMT); i += 256 * 16)
    *reinterpret_cast<uint4*>(chunk + i) = *reinterpret_cast<const uint4*>(src + i);
  __syncthreads();
  const int r = threadIdx.x & 127, h = threadIdx.x >> 7;
  const int n = t * TILE_N + r;
  if (n >= N) return;
  const float sig = col_scale ? sigma * col_scale[n] : sigma;
  if constexpr (FMT == FMT_FP8S) {
    for (int kl = h * 64; kl < h * 64 + 64; ++kl) {
      const int k = s * STAGE_K + kl;
      if (k >= K) break;
      const uint8_t c = chunk[r * 128 + (((kl >> 4) ^ (r & 7)) << 4) + (kl & 15)];
      out[(size_t)n * K + k] = __float2bfloat16_rn(__fmul_rn(e4m3_decode(c), sig));
    }
  } else {
    uint32_t o[32];
    prologue_stage<FMT, 16>(chunk, r, h, mx_bias, o);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int k = s * STAGE_K + h * 64 + 2 * i;
      const float lo = __uint_as_float(o[i] << 16), hi = __uint_as_float(o[i] & 0xFFFF0000u);
      if (k < K) out[(size_t)n * K + k] = __float2bfloat16_rn(__fmul_rn(lo, sig));
      if (k + 1 < K) out[(size_t)n * K + k + 1] = __float2bfloat16_rn(__fmul_rn(hi, sig));
    }
  }
}

// ---------------------------------------------------------------------------
// static FP8 activation quantization: q = e4m3(f32(x / s_x)), saturating
// ---------------------------------------------------------------------------
template <bool FAST>
__device__ __forceinline__ uint32_t act_code_t(float v, float s, float r) {
  return e4m3_code(FAST ? e4m3_quotient(v, s, r) : __fdiv_rn(v, s));
}

template <bool FAST>
__device__ __forceinline__ void act_quant_loop(const __nv_bfloat16* x, long long count, float s_x, float r_x,
                                               uint8_t* q) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x)
    q[i] = (uint8_t)act_code_t<FAST>(__bfloat162float(x[i]), s_x, r_x);
}

__global__ void act_quant_kernel(const __nv_bfloat16* x, long long count, float s_x, uint8_t* q) {
  const float r_x = __frcp_rn(s_x);
  if (e4m3_quotient_ok(r_x))
    act_quant_loop<true>(x, count, s_x, r_x, q);
  else
    act_quant_loop<false>(x, count, s_x, r_x, q);
}

// The same, 16 elements per thread: two 16-byte loads of bf16, one 16-byte
// store of codes (x and q 16-byte aligned; `groups` = count / 16, the tail
// goes to act_quant_kernel).  Each code is the same function of the same
// value, so the result is bit-identical with the element-wise kernel.
template <bool FAST>
__device__ __forceinline__ void act_quant16_loop(const uint4* x, long long groups, float s_x, float r_x, uint4* q) {
  for (long long g = blockIdx.x * (long long)blockDim.x + threadIdx.x; g < groups;
       g += (long long)gridDim.x * blockDim.x) {
    const uint4 a = x[2 * g], b = x[2 * g + 1];
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t word = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t v = in[2 * w + k];
        const uint32_t lo = act_code_t<FAST>(__uint_as_float(v << 16), s_x, r_x);
        const uint32_t hi = act_code_t<FAST>(__uint_as_float(v & 0xFFFF0000u), s_x, r_x);
        word |= (lo | (hi << 8)) << (16 * k);
      }
      out[w] = word;
    }
    q[g] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

__global__ void act_quant16_kernel(const uint4* x, long long groups, float s_x, uint4* q) {
  const float r_x = __frcp_rn(s_x);
  if (e4m3_quotient_ok(r_x))
    act_quant16_loop<true>(x, groups, s_x, r_x, q);
  else
    act_quant16_loop<false>(x, groups, s_x, r_x, q);
}

// ---------------------------------------------------------------------------
// GPU packer (bit-identical with the host packer: same dq_codec.h routines)
// ---------------------------------------------------------------------------
__global__ void pack_int4_kernel(const float* W, int N, int K, uint8_t* packed, uint16_t* scales) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int groups = K / 128;
  if (gid >= (long long)N * groups) return;
  const int n = (int)(gid / groups), g = (int)(gid % groups);
  int8_t c[128];
  scales[gid] = quant_int4_group(W + (size_t)n * K + g * 128, 128, c);
  uint8_t* dst = packed + (size_t)n * (K / 2) + g * 64;
  for (int i = 0; i < 64; ++i) dst[i] = (uint8_t)((c[2 * i] & 0xF) | ((c[2 * i + 1] & 0xF) << 4));
}

// asymmetric INT4: scales bf16 [N, K/128] then zero points u8 [N, K/128],
// one buffer (the canonical storage)
__global__ void pack_int4a_kernel(const float* W, int N, int K, uint8_t* packed, uint8_t* scales) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int groups = K / 128;
  const long long G = (long long)N * groups;
  if (gid >= G) return;
  const int n = (int)(gid / groups), g = (int)(gid % groups);
  uint8_t c[128], z;
  const uint16_t sb = quant_int4_asym_group(W + (size_t)n * K + g * 128, 128, c, &z);
  scales[gid * 2] = (uint8_t)(sb & 0xFF);
  scales[gid * 2 + 1] = (uint8_t)(sb >> 8);
  scales[2 * G + gid] = z;
  uint8_t* dst = packed + (size_t)n * (K / 2) + g * 64;
  for (int i = 0; i < 64; ++i) dst[i] = (uint8_t)((c[2 * i] & 0xF) | ((c[2 * i + 1] & 0xF) << 4));
}

__global__ void amax_kernel(const float* W, long long count, unsigned int* amax_bits) {
  float a = 0.f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x)
    a = fmaxf(a, fabsf(W[i]));
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(a));   // a >= 0: bit order = value order
}

__global__ void pack_nvfp4_kernel(const float* W, int N, int K, const unsigned int* amax_bits, uint8_t* packed,
                                  uint8_t* scales, float* g_out) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int blocks = K / 16;
  const float g = nvfp4_global_scale(__uint_as_float(*amax_bits));
  if (gid == 0 && g_out) *g_out = g;
  if (gid >= (long long)N * blocks) return;
  const int n = (int)(gid / blocks), b = (int)(gid % blocks);
  uint8_t c[16];
  scales[gid] = quant_nvfp4_block(W + (size_t)n * K + b * 16, 16, g, c);
  uint8_t* dst = packed + (size_t)n * (K / 2) + b * 8;
  for (int i = 0; i < 8; ++i) dst[i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
}

__global__ void pack_mxfp4_kernel(const float* W, int N, int K, uint8_t* packed, uint8_t* scales) {
  const long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const int blocks = K / 32;
  if (gid >= (long long)N * blocks) return;
  const int n = (int)(gid / blocks), b = (int)(gid % blocks);
  uint8_t c[32];
  scales[gid] = quant_mxfp4_block(W + (size_t)n * K + b * 32, 32, c);
  uint8_t* dst = packed + (size_t)n * (K / 2) + b * 16;
  for (int i = 0; i < 16; ++i) dst[i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
}

// one warp per row: amax by shuffle, then the codes
__global__ void pack_fp8_kernel(const float* W, int N, int K, uint8_t* codes, float* scales) {
  const int n = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (n >= N) return;
  const float* w = W + (size_t)n * K;
  float a = 0.f;
  for (int k = lane; k < K; k += 32) a = fmaxf(a, fabsf(w[k]));
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  const float s = fdiv(a, 448.f);
  if (lane == 0) scales[n] = s;
  for (int k = lane; k < K; k += 32) codes[(size_t)n * K + k] = s > 0.f ? e4m3_encode_sat(fdiv(w[k], s)) : 0;
}

// two-pass tensor amax over fixed-size chunks (used by the allocation-free
// packer): pass 1 writes one partial maximum per chunk, pass 2 reduces them
__global__ void amax_partials_kernel(const float* W, long long count, long long chunk, float* partials) {
  const long long b0 = blockIdx.x * chunk;
  const long long b1 = b0 + chunk < count ? b0 + chunk : count;
  float a = 0.f;
  for (long long i = b0 + threadIdx.x; i < b1; i += blockDim.x) a = fmaxf(a, fabsf(W[i]));
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  __shared__ float wmax[32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) a = fmaxf(a, wmax[w]);
    partials[blockIdx.x] = a;
  }
}

__global__ void amax_final_kernel(const float* partials, int n, unsigned int* amax_bits) {
  float a = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) a = fmaxf(a, partials[i]);
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  __shared__ float wmax[32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) a = fmaxf(a, wmax[w]);
    *amax_bits = __float_as_uint(a);
  }
}

// ---------------------------------------------------------------------------
// FP4 x FP4: dynamic activation quantization ("TorchAO MXFP4 Dynamic
// Activation + MX Weight (Linear)", intro: MX-quantized activations and
// weights for the native FP4 MMA).  One thread per (row, 64 k): the two MX
// blocks (E8M0 per 32) or the four NVFP4 blocks (E4M3 per 16, under the
// call's global scale g_x) of those 64 k, quantized with the weight packer's
// codec, so that activations and weights follow the same recipe.
// GEMM layout (sfw set): codes [rows][kp / 2], the even k in the low nibble,
// rows >= M and k >= K zero; scale words [m_tile][k_stage][t][bn] (k-stage
// of 256, k-step t of 64; the word layout of the weight chunks).
// Canonical layout (sfw null): codes [M][K / 2], scale bytes [M][K / VS].
// ---------------------------------------------------------------------------
// E2M1 codes of two magnitudes, a at k (low nibble) and b at k + 1: the
// hardware conversion, round to nearest even, saturating at 6
__device__ __forceinline__ uint32_t e2m1x2_mag(float a, float b) {
  uint16_t r;
  asm("{ .reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "mov.b16 %0, {t, 0};\n\t}"
      : "=h"(r)
      : "f"(a), "f"(b));
  return r;
}

// f32(v / d), correctly rounded, for the E2M1 rounding that follows (v >= 0,
// r = f32(1 / d) correctly rounded and normal): Markstein's correction step,
// as e4m3_quotient.  Below 2^-4 every E2M1 code is 0 and from 8 on it is 6,
// whatever the quotient's last bits, so q0 is used as it is there.
__device__ __forceinline__ float e2m1_quotient(float v, float d, float r) {
  const float q0 = __fmul_rn(v, r);
  if (!(q0 >= 0x1p-4f && q0 < 8.f)) return q0;
  return __fmaf_rn(__fmaf_rn(-q0, d, v), r, q0);
}

// The codes of one word of two bf16 values (low half at k), the sign bit of
// the input kept (so -0 gives code 8, as the packer's codec does); returns
// the byte of the two codes.  DIV = 0: each magnitude times f (MXFP4: the
// block's 2^-e, a product exact in fp32); 1: divided by f (NVFP4: the
// block's dec(sb) * g) through e2m1_quotient with r = f32(1 / f); 2: by the
// IEEE division.
template <int DIV>
__device__ __forceinline__ uint32_t e2m1_pair(uint32_t w, float f, float r) {
  const float lo = __uint_as_float((w & 0x7FFFu) << 16), hi = __uint_as_float(w & 0x7FFF0000u);
  const uint32_t mag = DIV == 0 ? e2m1x2_mag(__fmul_rn(lo, f), __fmul_rn(hi, f))
                     : DIV == 1 ? e2m1x2_mag(e2m1_quotient(lo, f, r), e2m1_quotient(hi, f, r))
                                : e2m1x2_mag(__fdiv_rn(lo, f), __fdiv_rn(hi, f));
  return mag | ((w >> 12) & 0x8u) | ((w >> 24) & 0x80u);
}

// the codes of a block's words (WB / 4 packed words of 8 codes)
template <int DIV, int WB>
__device__ __forceinline__ void e2m1_block(const uint32_t (&w)[WB], float f, float r, uint32_t* packed) {
#pragma unroll
  for (int q = 0; q < WB / 4; ++q) {
    uint32_t pk = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) pk |= e2m1_pair<DIV>(w[4 * q + e], f, r) << (8 * e);
    packed[q] = pk;
  }
}

template <bool MX>
__global__ void __launch_bounds__(256) w4a4_act_quant_kernel(const __nv_bfloat16* __restrict__ x, int M, int K,
                                                             int rows, int kp, int bn, const float* gx,
                                                             uint8_t* codes, uint32_t* sfw, uint8_t* scales) {
  // (the GEMM after this kernel may start now and stream its weights; it
  // reads what this kernel writes only after waiting for it to complete)
  pdl_launch_dependents();
  pdl_wait();   // x may be the previous grid's output, and that grid may still read the workspace
  constexpr int VS = MX ? 32 : 16;   // elements per block
  constexpr int WB = VS / 2;         // bf16x2 words per block
  const float g = MX ? 1.f : *reinterpret_cast<const volatile float*>(gx);
  const int slices = kp / 64;
  const long long total = (long long)rows * slices;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(i / slices), sl = (int)(i - (long long)row * slices);
    const int k0 = sl * 64;
    uint32_t packed[8];
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 64 / VS; ++b) {
      const int kb = k0 + b * VS;
      uint32_t w[WB];
      if (row < M && kb + VS <= K) {
        // (K is a multiple of 16 and x 16-byte aligned: whole vectors)
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)row * K + kb);
#pragma unroll
        for (int q = 0; q < WB / 4; ++q) {
          const uint4 u = src[q];
          w[4 * q] = u.x;
          w[4 * q + 1] = u.y;
          w[4 * q + 2] = u.z;
          w[4 * q + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < WB; ++e) w[e] = 0u;
      }
      // block amax: the largest bf16 magnitude (as bits; x holds no NaN)
      uint32_t am = 0;
#pragma unroll
      for (int e = 0; e < WB; ++e) am = max(am, max(w[e] & 0x7FFFu, (w[e] >> 16) & 0x7FFFu));
      const float amax = __uint_as_float(am << 16);
      uint32_t sc = 0;
      float f = 0.f;
      bool live = amax > 0.f;
      if constexpr (MX) {
        if (live) {
          int e = ilog2f(amax) - 2;
          e = e < -127 ? -127 : e;   // (amax < 2^128: e <= 125, and 2^-e is an fp32 normal)
          sc = (uint32_t)(e + 127);
          f = pow2f(-e);
        }
      } else {
        sc = e4m3_encode_sat(fdiv(fdiv(amax, 6.f), g));
        f = fmul(e4m3_decode((uint8_t)sc), g);
        live = f > 0.f;
      }
      word |= sc << (8 * b);
      uint32_t* pb = packed + b * (WB / 4);
      if (!live) {
#pragma unroll
        for (int q = 0; q < WB / 4; ++q) pb[q] = 0u;
      } else if constexpr (MX) {
        e2m1_block<0>(w, f, 0.f, pb);
      } else {
        const float r = __frcp_rn(f);
        if (e4m3_quotient_ok(r))
          e2m1_block<1>(w, f, r, pb);
        else
          e2m1_block<2>(w, f, r, pb);
      }
      if (!sfw && row < M && kb < K) scales[(size_t)row * (K / VS) + kb / VS] = (uint8_t)sc;
    }
    if (sfw) {
      uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)row * (kp / 2) + k0 / 2);
      dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
      const int mt = row / bn, r = row - mt * bn, ks = k0 >> 8, t = (k0 >> 6) & 3;
      sfw[(((size_t)mt * (kp >> 8) + ks) * 4 + t) * bn + r] = word;
    } else if (row < M) {
      for (int b = 0; b < 32 && k0 + 2 * b < K; ++b)
        codes[(size_t)row * (K / 2) + k0 / 2 + b] = (uint8_t)(packed[b >> 2] >> (8 * (b & 3)));
    }
  }
}

// NVFP4 activations: g_x = amax(x) / 2688 (1 for an all-zero x), written to
// *gx by the last block to finish (the blocks leave their maxima in
// partials[]; `ticket` counts them and is reset to 0 for the next call).
constexpr int kActAmaxBlocks = 1024;
__global__ void __launch_bounds__(256) act_amax_kernel(const __nv_bfloat16* __restrict__ x, long long count,
                                                       float* partials, unsigned int* ticket, float* gx) {
  pdl_launch_dependents();   // (the kernels after it wait for its completion before reading what it writes)
  pdl_wait();
  float a = 0.f;
  const long long vecs = count / 8;
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < vecs;
       i += (long long)gridDim.x * blockDim.x) {
    const uint4 u = xv[i];
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
      a = fmaxf(a, fmaxf(fabsf(__uint_as_float(w4[e] << 16)), fabsf(__uint_as_float(w4[e] & 0xFFFF0000u))));
  }
  for (long long i = vecs * 8 + blockIdx.x * (long long)blockDim.x + threadIdx.x; i < count;
       i += (long long)gridDim.x * blockDim.x)
    a = fmaxf(a, fabsf(__bfloat162float(x[i])));
  __shared__ float wmax[8];
  __shared__ int last;
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) a = fmaxf(a, wmax[w]);
    partials[blockIdx.x] = a;
    __threadfence();
    last = atomicAdd(ticket, 1u) == gridDim.x - 1 ? 1 : 0;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  float m = 0.f;
  for (int i = threadIdx.x; i < (int)gridDim.x; i += blockDim.x)
    m = fmaxf(m, *reinterpret_cast<const volatile float*>(partials + i));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
    *gx = nvfp4_global_scale(m);
    *ticket = 0u;
  }
}

// ---------------------------------------------------------------------------
// bounded-wait self test: waits on a barrier nothing will ever arrive at
// ---------------------------------------------------------------------------
__global__ void selftest_timeout_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, status, timeout_ns};
    if (mbar_wait(&bar, 0, ctl)) atomicExch(status, DEV_OK);
  }
}

}  // namespace dq
