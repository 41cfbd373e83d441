// dq_gemm.cuh -- the dequantize-in-prologue GEMM kernel for sm_100a.
//
// y[M, N] = x[M, K] . deq(W)^T + b, computed as y^T = deq(W) . x^T so that
// the 128 weight rows of a tile are the tcgen05 MMA's M and the activation
// rows are its N (BN = 16..128): the skinny decode shapes the quantized-Linear
// pages run (x of 32 rows) keep the tensor core busy on the weight side.
//
// CTA = 10 warps, warp-specialized:
//   warp 0      producer: one 1-D bulk copy of the stage's pre-tiled weight
//               chunk + two TMA box loads of the bf16 x tile, per stage
//   warp 1      MMA issuer: one thread issues tcgen05.mma into a TMEM
//               accumulator and commits stage / accumulator barriers
//   warps 2..9  the prologue: unpack + scale the packed codes of one weight
//               row per thread (two threads per row, one per k-half) into
//               bf16 operands written straight to TMEM (the MMA reads A from
//               TMEM), or, for static FP8, quantize the x tile to e4m3 into
//               shared memory; then the epilogue (tcgen05.ld, scale, bias,
//               bf16 cast, store).
// Work split: stream-K over (output tile, k-stage) units, one CTA per SM;
// a tile cut between CTAs is summed by its last-arriving CTA in a fixed
// order (deterministic), with no spin on other CTAs.
// Every wait is bounded (WaitCtl): on expiry the CTA drains its own copies
// and MMAs, frees TMEM, records DEV_TIMEOUT and returns.
#pragma once

#include "dq_common.cuh"

namespace dq {

struct GemmParams {
  const uint8_t* wchunks;        // handle's pre-tiled weight
  const float* col_scale;        // per output channel factor (FP8 formats) or null
  const __nv_bfloat16* bias;     // [N] or null
  __nv_bfloat16* y;              // [M, N]
  float* ws;                     // split-K partials: [grid][2][BN][128] fp32
  int* counters;                 // [tiles] arrival counters, self-resetting
  int* status;                   // device status word
  float sigma;                   // epilogue factor common to all channels
  float s_x;                     // static FP8 activation scale
  int mx_bias;                   // MXFP4: 126 - J
  int M, N, k_stages, m_tiles;
  long long units;               // tiles * k_stages
  unsigned long long timeout_ns;
};

__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }
__host__ __device__ constexpr int pow2_at_least(int v) {
  return v <= 32 ? 32 : v <= 64 ? 64 : v <= 128 ? 128 : v <= 256 ? 256 : 512;
}

template <int FMT, int BN>
struct GemmCfg {
  static constexpr bool STATIC = (FMT == FMT_FP8S);
  static constexpr int CHUNK = chunk_bytes(FMT);
  static constexpr int X_BYTES = BN * 256;                 // two 64-k boxes of BN rows x 128 B
  static constexpr int Q_BYTES = STATIC ? BN * 128 : 0;    // e4m3 x tile (static FP8)
  static constexpr int X_OFF = 0;
  static constexpr int Q_OFF = align_up(X_BYTES, 1024);
  static constexpr int W_OFF = Q_OFF + align_up(Q_BYTES, 1024);
  static constexpr int STAGE_BYTES = W_OFF + align_up(CHUNK, 1024);
  static constexpr int STAGES_RAW = (200 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 6 ? 6 : STAGES_RAW);
  static constexpr int A_COLS = STATIC ? 0 : STAGES * (STAGE_K / 2);   // bf16 A ring in TMEM
  static constexpr int ACC_COL = A_COLS;
  static constexpr int TMEM_COLS = pow2_at_least(A_COLS + BN);
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = STAGES * STAGE_BYTES + BAR_BYTES + 1024;   // + alignment slack
  static constexpr uint32_t IDESC = STATIC ? idesc_e4m3(BN) : idesc_bf16(BN);
  static constexpr uint32_t TX_BYTES = CHUNK + X_BYTES;
  static constexpr int THREADS = 320;
  static_assert(A_COLS + BN <= 512, "TMEM budget");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// CTA that owns stream-K unit u when U units are cut into G contiguous ranges
// [floor(c U / G), floor((c+1) U / G)).
__host__ __device__ inline int cta_of_unit(long long u, long long U, int G) {
  return (int)(((u + 1) * (long long)G - 1) / U);
}
__host__ __device__ inline long long cta_start(int c, long long U, int G) { return (long long)c * U / G; }

template <int FMT, int BN>
__device__ __forceinline__ void prologue_stage(const uint8_t* chunk, int r, int h, int mx_bias, uint32_t (&o)[32]) {
  if constexpr (FMT == FMT_FP8) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = lds128(chunk + ((h * 4 + j) * TILE_N + r) * 16);
      unpack_e4m3(v.x, o + j * 8 + 0);
      unpack_e4m3(v.y, o + j * 8 + 2);
      unpack_e4m3(v.z, o + j * 8 + 4);
      unpack_e4m3(v.w, o + j * 8 + 6);
    }
  } else {
    const uint4 v0 = lds128(chunk + ((h * 2 + 0) * TILE_N + r) * 16);
    const uint4 v1 = lds128(chunk + ((h * 2 + 1) * TILE_N + r) * 16);
    const uint8_t* sc = chunk + PACKED4_BYTES;
    if constexpr (FMT == FMT_INT4) {
      const uint32_t s = *reinterpret_cast<const uint16_t*>(sc + r * 2);
      const uint32_t s2 = s | (s << 16);
      unpack_int4(v0.x, s2, o + 0);
      unpack_int4(v0.y, s2, o + 4);
      unpack_int4(v0.z, s2, o + 8);
      unpack_int4(v0.w, s2, o + 12);
      unpack_int4(v1.x, s2, o + 16);
      unpack_int4(v1.y, s2, o + 20);
      unpack_int4(v1.z, s2, o + 24);
      unpack_int4(v1.w, s2, o + 28);
    } else if constexpr (FMT == FMT_NVFP4) {
      const uint32_t c4 = *reinterpret_cast<const uint32_t*>(sc + (h * TILE_N + r) * 4);
      uint32_t s2[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint32_t s = nvfp4_scale_bf16((c4 >> (8 * b)) & 0xFFu);
        s2[b] = s | (s << 16);
      }
      unpack_e2m1(v0.x, s2[0], o + 0);
      unpack_e2m1(v0.y, s2[0], o + 4);
      unpack_e2m1(v0.z, s2[1], o + 8);
      unpack_e2m1(v0.w, s2[1], o + 12);
      unpack_e2m1(v1.x, s2[2], o + 16);
      unpack_e2m1(v1.y, s2[2], o + 20);
      unpack_e2m1(v1.z, s2[3], o + 24);
      unpack_e2m1(v1.w, s2[3], o + 28);
    } else {  // MXFP4
      const uint32_t c2 = *reinterpret_cast<const uint16_t*>(sc + (h * TILE_N + r) * 2);
      const uint32_t sa = mxfp4_scale_bf16(c2 & 0xFFu, mx_bias), sb = mxfp4_scale_bf16(c2 >> 8, mx_bias);
      const uint32_t s2a = sa | (sa << 16), s2b = sb | (sb << 16);
      unpack_e2m1(v0.x, s2a, o + 0);
      unpack_e2m1(v0.y, s2a, o + 4);
      unpack_e2m1(v0.z, s2a, o + 8);
      unpack_e2m1(v0.w, s2a, o + 12);
      unpack_e2m1(v1.x, s2b, o + 16);
      unpack_e2m1(v1.y, s2b, o + 20);
      unpack_e2m1(v1.z, s2b, o + 24);
      unpack_e2m1(v1.w, s2b, o + 28);
    }
  }
}

// Static FP8: quantize the bf16 x tile (two SW128 boxes) into the e4m3 SW128
// B operand: q = e4m3(f32(x / s_x)), IEEE division, RNE, saturating.
template <int BN>
__device__ __forceinline__ void quantize_x_tile(const uint8_t* xs, uint8_t* qs, float s_x, int tid) {
  for (int c = tid; c < BN * 8; c += 256) {
    const int row = c >> 3, cc = c & 7;
    const uint8_t* box = xs + (cc >> 2) * BN * 128 + row * 128;
    const uint4 a = lds128(box + (((2 * (cc & 3)) ^ (row & 7)) << 4));
    const uint4 b = lds128(box + (((2 * (cc & 3) + 1) ^ (row & 7)) << 4));
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lohi[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t w = in[2 * i + k];
        const float f0 = __uint_as_float(w << 16), f1 = __uint_as_float(w & 0xFFFF0000u);
        const float2 qv = make_float2(__fdiv_rn(f0, s_x), __fdiv_rn(f1, s_x));
        lohi[k] = (uint32_t)__nv_cvt_float2_to_fp8x2(qv, __NV_SATFINITE, __NV_E4M3);
      }
      out[i] = lohi[0] | (lohi[1] << 16);
    }
    sts128(qs + row * 128 + ((cc ^ (row & 7)) << 4), make_uint4(out[0], out[1], out[2], out[3]));
  }
}

template <int FMT, int BN>
__global__ void __launch_bounds__(320, 1) dq_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                          const GemmParams p) {
  using C = GemmCfg<FMT, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* aready = full + C::STAGES;
  uint64_t* empty = aready + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* epi_a = acc_empty + 1;
  uint64_t* epi_b = epi_a + 1;
  uint64_t* drain = epi_b + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* bcast = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&aready[s], 8);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(epi_a, 256);
    mbar_init(epi_b, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    *bcast = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::TMEM_COLS);
  if (warp == 1 && lane == 0) prefetch_tmap(&tmap_x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const long long U = p.units;
  const int G = gridDim.x;
  const int KS = p.k_stages;
  const long long u0 = cta_start(blockIdx.x, U, G), u1 = cta_start(blockIdx.x + 1, U, G);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (long long u = u0; ok && u < u1;) {
        const int tile = (int)(u / KS), kb = (int)(u % KS);
        const int ke = (int)((long long)kb + (u1 - u) < KS ? kb + (u1 - u) : KS);
        const int n_tile = tile / p.m_tiles, m_tile = tile % p.m_tiles;
        for (int ks = kb; ks < ke; ++ks, ++it) {
          const int slot = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(&empty[slot], ph ^ 1, ctl)) { ok = false; break; }
          uint8_t* st = smem + slot * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[slot], C::TX_BYTES);
          bulk_g2s(st + C::W_OFF, p.wchunks + ((size_t)n_tile * KS + ks) * C::CHUNK, C::CHUNK, &full[slot]);
          tma_load_2d(st + C::X_OFF, &tmap_x, ks * STAGE_K, m_tile * BN, &full[slot]);
          tma_load_2d(st + C::X_OFF + BN * 128, &tmap_x, ks * STAGE_K + 64, m_tile * BN, &full[slot]);
        }
        u += ke - kb;
      }
      // Never leave with copies in flight: wait for the last issued stages
      // (their full barriers complete on data arrival alone).
      volatile int no_abort = 0;
      const WaitCtl drain_ctl{&no_abort, p.status, p.timeout_ns};
      const uint32_t first = it > (uint32_t)C::STAGES ? it - C::STAGES : 0;
      for (uint32_t i = first; i < it; ++i) mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1, drain_ctl);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0;
      int seg = 0;
      bool ok = true;
      for (long long u = u0; ok && u < u1; ++seg) {
        const int kb = (int)(u % KS);
        const int ke = (int)((long long)kb + (u1 - u) < KS ? kb + (u1 - u) : KS);
        if (!mbar_wait(acc_empty, (seg & 1) ^ 1, ctl)) break;
        tc_fence_after();
        for (int ks = kb; ks < ke; ++ks, ++it) {
          const int slot = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1;
          if (!mbar_wait(&full[slot], ph, ctl) || !mbar_wait(&aready[slot], ph, ctl)) { ok = false; break; }
          tc_fence_after();
          uint8_t* st = smem + slot * C::STAGE_BYTES;
          if constexpr (!C::STATIC) {
            const uint32_t xb = smem_u32(st + C::X_OFF);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = sdesc_sw128(xb + (kk >> 2) * BN * 128 + (kk & 3) * 32);
              mma_bf16_ts(tmem + C::ACC_COL, tmem + slot * (STAGE_K / 2) + kk * 8, bd, C::IDESC,
                          (ks > kb || kk > 0) ? 1u : 0u);
            }
          } else {
            const uint32_t wb = smem_u32(st + C::W_OFF), qb = smem_u32(st + C::Q_OFF);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_f8_ss(tmem + C::ACC_COL, sdesc_sw128(wb + kk * 32), sdesc_sw128(qb + kk * 32), C::IDESC,
                        (ks > kb || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(&empty[slot]);
        }
        if (!ok) break;
        tc_commit(acc_full);
        u += ke - kb;
      }
      // all MMAs this thread issued must finish before TMEM is released
      volatile int no_abort = 0;
      const WaitCtl drain_ctl{&no_abort, p.status, p.timeout_ns};
      tc_commit(drain);
      mbar_wait(drain, 0, drain_ctl);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ prologue + epilogue
    const int dw = warp - 2;            // 0..7
    const int qd = warp & 3;            // TMEM lane quadrant this warp may access
    const int h = dw >> 2;              // k-half of the stage / column half of the tile
    const int r = qd * 32 + lane;       // weight row in the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    uint32_t it = 0;
    int seg = 0, pseg = 0;
    bool ok = true;
    for (long long u = u0; ok && u < u1; ++seg) {
      const int tile = (int)(u / KS), kb = (int)(u % KS);
      const int ke = (int)((long long)kb + (u1 - u) < KS ? kb + (u1 - u) : KS);
      const int n_tile = tile / p.m_tiles, m_tile = tile % p.m_tiles;
      for (int ks = kb; ks < ke; ++ks, ++it) {
        const int slot = it % C::STAGES;
        const uint32_t ph = (it / C::STAGES) & 1;
        if (!mbar_wait(&full[slot], ph, ctl)) { ok = false; break; }
        uint8_t* st = smem + slot * C::STAGE_BYTES;
        if constexpr (!C::STATIC) {
          // the TMEM A slot is free once the MMAs of its previous use completed
          if (!mbar_wait(&empty[slot], ph ^ 1, ctl)) { ok = false; break; }
          tc_fence_after();
          uint32_t o[32];
          prologue_stage<FMT, BN>(st + C::W_OFF, r, h, p.mx_bias, o);
          tmem_st32(tmem + lane_base + slot * (STAGE_K / 2) + h * 32, o);
          tmem_wait_st();
          tc_fence_before();
        } else {
          quantize_x_tile<BN>(st + C::X_OFF, st + C::Q_OFF, p.s_x, threadIdx.x - 64);
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[slot]);
      }
      if (!ok) break;

      // ---- epilogue of this segment
      if (!mbar_wait(acc_full, seg & 1, ctl)) break;
      tc_fence_after();
      constexpr int HALF = BN / 2;
      float acc[HALF];
#pragma unroll
      for (int c8 = 0; c8 < HALF / 8; ++c8) {
        float v[8];
        tmem_ld8(tmem + lane_base + C::ACC_COL + h * HALF + c8 * 8, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[c8 * 8 + i] = v[i];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);

      const long long tu = (long long)tile * KS;
      const int c_first = cta_of_unit(tu, U, G), c_last = cta_of_unit(tu + KS - 1, U, G);
      const int nseg = c_last - c_first + 1;
      bool store = true;
      if (nseg > 1) {
        // write this CTA's partial, then let the last arriver of the tile sum
        const int which = (seg == 0) ? 0 : 1;
        float* mine = p.ws + ((size_t)(blockIdx.x * 2 + which) * BN) * TILE_N;
#pragma unroll
        for (int i = 0; i < HALF; ++i) mine[(h * HALF + i) * TILE_N + r] = acc[i];
        __threadfence();
        mbar_arrive(epi_a);
        if (dw == 0 && lane == 0) {
          int last = 0;
          if (mbar_wait(epi_a, pseg & 1, ctl)) {
            const int old = atomicAdd(&p.counters[tile], 1);
            last = (old == nseg - 1);
            if (last) p.counters[tile] = 0;   // every contributor has arrived: reset for the next call
          }
          *bcast = last;
          mbar_arrive(epi_b);
        }
        if (!mbar_wait(epi_b, pseg & 1, ctl)) break;
        ++pseg;
        store = (*bcast != 0);
        if (store) {
          // sum every contributor's partial (this CTA's included, re-read from
          // the workspace) in CTA order: the result does not depend on which
          // CTA arrived last
          __threadfence();
          for (int c = c_first; c <= c_last; ++c) {
            const int w = ((cta_start(c, U, G) / KS) == tile) ? 0 : 1;
            const float* src = p.ws + ((size_t)(c * 2 + w) * BN) * TILE_N + r;
#pragma unroll
            for (int i = 0; i < HALF; ++i) {
              const float v = __ldcg(src + (h * HALF + i) * TILE_N);
              acc[i] = (c == c_first) ? v : acc[i] + v;
            }
          }
        }
      }
      if (store) {
        const int n = n_tile * TILE_N + r;
        if (n < p.N) {
          const float sig = p.col_scale ? p.sigma * p.col_scale[n] : p.sigma;
          const float b = p.bias ? __bfloat162float(p.bias[n]) : 0.f;
#pragma unroll
          for (int i = 0; i < HALF; ++i) {
            const int m = m_tile * BN + h * HALF + i;
            if (m < p.M) p.y[(size_t)m * p.N + n] = __float2bfloat16_rn(fmaf(acc[i], sig, b));
          }
        }
      }
      u += ke - kb;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace dq
