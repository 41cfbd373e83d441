// dq_gemm.cuh -- the dequantize-in-prologue GEMM kernel for sm_100a.
//
// y[M, N] = x[M, K] . deq(W)^T + b, computed as y^T = deq(W) . x^T so that
// the 128 weight rows of a tile are the tcgen05 MMA's M and the activation
// rows are its N (BN = 16..256): the skinny decode shapes the quantized-Linear
// pages run (x of 32 rows) keep the tensor core busy on the weight side.
//
// CTA = 12 warps, warp-specialized:
//   warp 0      weight producer: one 1-D bulk copy of the stage's pre-tiled
//               weight chunk per stage into a ring of up to 8 slots, from
//               CTA entry on (weights never depend on the previous grid)
//   warp 11     x producer: after the grid-dependency wait, the TMA box
//               load(s) of the stage's x tile (bf16, or codes quantized
//               beforehand, plus W4A4's scale words) into the x ring (a
//               single-tile CTA's first ring issued by one lane per stage)
//   warps 1, 10 MMA issuers: one thread each issues tcgen05.mma for half of
//               every stage's k-steps into its own TMEM accumulator (one
//               issuer at 256-row tiles) and commits the slot / operand /
//               accumulator barriers
//   warps 2..9  the prologue, then the epilogue:
//               - weight-only formats: unpack + scale the packed codes of one
//                 weight row per thread (two threads per row, one per
//                 k-half) into bf16 operands written straight to TMEM (the
//                 MMA reads A from TMEM), taking turns with the CTA of the
//                 neighbouring call on the same SM (g_sm_turn);
//               - fused static FP8: warps 2..5 copy the e4m3 weight rows into
//                 TMEM (the FP8 MMA reads A there) and warps 6..9 quantize
//                 the bf16 x tile to e4m3 operands in shared memory;
//               - W4A4: write each stage's block scales of both operands into
//                 TMEM (the MMA reads both operands from shared memory);
//               - static FP8 on codes: nothing (both operands in shared
//                 memory; its 256-row tiles double-buffer the accumulator,
//                 so these warps' epilogue overlaps the next tile);
//               then tcgen05.ld of the accumulator(s), scale, bias, cast,
//               store.
// Work split: a tile of 128 output channels x BN activation rows is either
// computed whole by one CTA (persistent loop over tiles), or its K range is
// split over the S CTAs of a thread-block cluster: each sends every peer its
// partial of the peer's columns into the peer's shared memory (st.async),
// and each adds the S partials of its own columns in rank order
// (deterministic, no global scratch).
// Back-to-back calls overlap through programmatic dependent launch: a CTA
// sets up and starts streaming its (read-only) weights before waiting for the
// previous grid; it reads x and writes y only after that wait.
// Every mbarrier wait is bounded (WaitCtl): on expiry the CTA drains its own
// copies and MMAs, frees TMEM, records DEV_TIMEOUT and returns.
#pragma once

#include "dq_common.cuh"

namespace dq {

struct GemmParams {
  const uint8_t* wchunks;        // handle's pre-tiled weight
  const float* col_scale;        // per output channel factor (FP8 formats) or null
  const __nv_bfloat16* bias;     // [N] or null
  __nv_bfloat16* y;              // [M, N]
  int* status;                   // device status word
  float sigma;                   // epilogue factor common to all channels
  float s_x;                     // static FP8 activation scale
  float r_x, r_out;              // f32(1 / s_x) and f32(1 / s_out), correctly rounded (host division)
  int mx_bias;                   // MXFP4: 126 - J
  int M, N, k_stages, m_tiles;
  int tiles;                     // n_tiles * m_tiles
  int split;                     // CTAs per tile (cluster size); 1 = whole tiles
  int x3d;                       // x map is 3-D {64, M, K/64}: one box per stage
  unsigned long long timeout_ns;  // limit of the pipeline's waits
  unsigned long long drain_ns;    // limit of the waits for this CTA's own copies, MMAs and received
                                  // partials (never shorter than the default: leaving early would
                                  // free shared or tensor memory that is still being written)
  uint8_t* yq;                   // if set: y goes out as e4m3 codes of bf16(y) / s_out
  float s_out;                   //   (the next static-FP8 layer's activation codes)
  // two-layer static MLP (FMT_MLP): layer 1 is (wchunks, col_scale, bias,
  // sigma = s_x) with N = hidden; its output is quantized with s_out and
  // multiplied by layer 2 (w2chunks, col_scale2, bias2), N2 outputs
  const uint8_t* w2chunks;
  const float* col_scale2;
  const __nv_bfloat16* bias2;
  __nv_bfloat16* h_out;          // optional: layer 1's bf16 output [M, N]
  int N2;
  // FP4 x FP4: the activation's block-scale words, [m_tile][k_stage][4][BN]
  // (the layout of the weight's, per tile of BN rows), and for NVFP4 the
  // activation's per-call global scale (device, written by the quantizer)
  const uint32_t* xsf;
  const float* gx;
};

// the e4m3 code of an output for the next static-FP8 layer,
// q = e4m3(f32(bf16(v)) / s_out): the code dqgemm_quantize_act_fp8 gives
// for the bf16 output y = bf16(v)
__device__ __forceinline__ uint8_t out_code(const GemmParams& p, float v) {
  return act_code_r(__bfloat162float(__float2bfloat16_rn(v)), p.s_out, p.r_out);
}

__host__ __device__ constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }
__host__ __device__ constexpr int pow2_at_least(int v) {
  return v <= 32 ? 32 : v <= 64 ? 64 : v <= 128 ? 128 : v <= 256 ? 256 : 512;
}

template <int FMT, int BN>
struct GemmCfg {
  // FP4 x FP4 (W4A4): both operands packed E2M1 in shared memory, x
  // quantized beforehand (codes through a 2-D u8 map, its block-scale words
  // by a 1-D bulk copy), the block scales of both in tensor memory
  static constexpr bool W4A4 = is_w4a4(FMT);
  static constexpr bool MXS = (FMT == FMT_W4A4MX);   // E8M0 scales per 32 (else E4M3 per 16)
  // x quantized beforehand: x arrives as codes (e4m3 [M, K] for static FP8,
  // packed E2M1 for W4A4) through a 2-D u8 map (box 128 bytes x BN rows),
  // straight into the operand buffer
  static constexpr bool XQ = (FMT == FMT_FP8SQ) || W4A4;
  static constexpr bool MLP = (FMT == FMT_MLP);
  static constexpr bool STATIC = (FMT == FMT_FP8S) || (FMT == FMT_FP8SQ) || MLP;
  // fused static FP8: the e4m3 weight stage is copied from shared memory into
  // a ring of TMEM slots (32 columns each) and the MMA reads A there, so the
  // weight slots are free again at once and many stages stream in before the
  // grid-dependency wait (A from shared memory would hold every stage's slot
  // until its MMAs complete)
  static constexpr bool TSA = (FMT == FMT_FP8S);
  static constexpr bool SS = (STATIC && !TSA) || W4A4;   // A (weight) from shared memory as well
  static constexpr int CHUNK = chunk_bytes(MLP ? FMT_FP8S : FMT);
  static constexpr int X_BYTES = XQ ? 0 : BN * 256;        // two 64-k blocks of BN rows x 128 B
  static constexpr int Q_BYTES = (STATIC || W4A4) ? BN * 128 : 0;   // e4m3 / packed E2M1 x tile
  static constexpr int XSF_BYTES = W4A4 ? 4 * BN * 4 : 0;  // W4A4: x block-scale words [4][BN]
  // Two rings: packed weight chunks (streamed from the start of the kernel;
  // a slot is free once the prologue has read it, or for static FP8 and
  // W4A4 once the MMAs have) and x tiles (loaded only after the
  // grid-dependency wait; a slot is free once the MMAs have read it).
  // (fused static FP8 with A in TMEM keeps the bf16 x tiles and their e4m3
  // operands in separate rings: a bf16 slot is free as soon as its tile is
  // quantized, an operand slot once the MMAs have read it)
  static constexpr int X_SLOT = TSA ? align_up(X_BYTES, 1024) : align_up(X_BYTES, 1024) + align_up(Q_BYTES + XSF_BYTES, 1024);
  static constexpr int Q_SLOT = align_up(Q_BYTES, 1024);
  static constexpr int Q_OFF = align_up(X_BYTES, 1024);    // within an x slot
  static constexpr int XSF_OFF = Q_OFF + Q_BYTES;
  static constexpr int W_SLOT = align_up(CHUNK, 1024);
  // skinny tiles keep a CTA under half an SM's shared memory so that the next
  // call's CTA can be resident alongside (programmatic dependent launch)
  static constexpr int SMEM_BUDGET = TSA ? (BN <= 32 ? 108 * 1024 : 216 * 1024)
                                         : BN <= 64 ? 108 * 1024 : (BN <= 128 ? 200 * 1024 : 216 * 1024);
  // split-K receive area: the S partials (its own included) of the columns
  // this CTA owns, [rank][row][BN / S] fp32 = one 128 x BN fp32 tile, then
  // one validity word per (rank, 32 rows) (256-row x tiles run whole tiles
  // only: none)
  static constexpr int RECV_BYTES = BN >= 256 ? 0 : TILE_N * BN * 4;
  static constexpr int RFLAG_BYTES = 128;   // [8 ranks][4 row quadrants]
  // MLP: layer 2's weight chunk (its k-slice of this CTA's hidden columns)
  // and layer 2's B operand, this CTA's hidden activations as e4m3 codes
  static constexpr int W2_BYTES = MLP ? TILE_N * STAGE_K : 0;
  static constexpr int B2_BYTES = MLP ? align_up(BN * STAGE_K, 1024) : 0;
  static constexpr int AVAIL = SMEM_BUDGET - RECV_BYTES - RFLAG_BYTES - W2_BYTES - B2_BYTES - 3072;   // barriers, EPI, slack
  // The x ring is as deep as the budget allows while keeping three weight
  // slots: a skinny split CTA (six 128-k stages at 32 x 3072 x 4096) then
  // issues every x load of its k-range right after the grid-dependency wait.
  // (TSA: the weights drain into TMEM at once, so two or three weight slots
  // do; the bf16 landing ring gets as many slots as leave the operand ring
  // 4 (2 from 64 rows on), up to 8, so that most x loads of a CTA's k-range
  // are issued together after the grid-dependency wait; the operand ring
  // takes the rest, up to 8)
  static constexpr int TSA_WST = BN <= 16 ? 3 : 2;
  static constexpr int TSA_XST = (AVAIL - TSA_WST * W_SLOT - (BN <= 32 ? 4 : 2) * Q_SLOT) / (X_SLOT > 0 ? X_SLOT : 1);
  // (W4A4 at 256-row tiles: 3 x and 5 weight slots, the fastest of the
  // splits 5/2, 4/3, 3/5 and 2/8 measured at 4096 x 4096 x 4096)
  static constexpr bool W4WIDE = W4A4 && BN == 256;
  static constexpr int XST = W4WIDE ? 3
                             : TSA ? (TSA_XST > 8 ? 8 : TSA_XST < 2 ? 2 : TSA_XST)
                             : (AVAIL - 6 * X_SLOT >= 3 * W_SLOT) ? 6
                             : (AVAIL - 4 * X_SLOT >= 3 * W_SLOT) ? 4
                             : (AVAIL - 3 * X_SLOT >= 3 * W_SLOT) ? 3
                                                                  : 2;
  static constexpr int WST_RAW = W4WIDE ? 5 : TSA ? TSA_WST : (AVAIL - XST * X_SLOT) / W_SLOT;
  static constexpr int WST = WST_RAW < 2 ? 2 : (WST_RAW > 8 ? 8 : WST_RAW);
  static constexpr int QST_RAW = TSA ? (AVAIL - XST * X_SLOT - WST * W_SLOT) / Q_SLOT : 0;
  static constexpr int QST = QST_RAW > 8 ? 8 : QST_RAW;
  static constexpr int STAGES = WST;   // weight stages in flight (reported by the plan)
  static constexpr int X_RING_OFF = 0;
  static constexpr int Q_RING_OFF = XST * X_SLOT;
  static constexpr int W_RING_OFF = Q_RING_OFF + QST * Q_SLOT;
  static constexpr int RECV_OFF = W_RING_OFF + WST * W_SLOT;
  static constexpr int RFLAG_OFF = RECV_OFF + RECV_BYTES;
  static constexpr int W2_OFF = align_up(RFLAG_OFF + RFLAG_BYTES, 1024);
  static constexpr int B2_OFF = W2_OFF + W2_BYTES;
  // TMEM: a ring of bf16 A operands (weights, one 128 x 128 stage each) and
  // the fp32 accumulators.  Two MMA-issuing threads (in different warps) each
  // own half of every stage's k-steps and an accumulator of their own: one
  // thread issues an MMA only every ~80 cycles, two issue in parallel.  The
  // epilogue adds the two accumulators in a fixed order.
  // (a 256-row x tile needs one issuer only: an N = 256 MMA keeps the tensor
  // pipe busy for longer than a thread takes to issue the next)
  static constexpr int ISSUERS = BN >= 256 ? 1 : 2;
  // k-steps (of 16 bf16 / 32 e4m3 / 64 E2M1) per stage each issuer takes
  static constexpr int KK = (SS || TSA ? 4 : 8) / ISSUERS;
  // W4A4: the TMEM slots are the stage's block scales instead of operands:
  // per k-step t, 4 columns for the 128 weight rows (row m at lane m % 32 of
  // every quadrant, column m / 32) and SFB_COLS for the BN x rows likewise
  static constexpr int SFB_COLS = BN / 32 < 4 ? 4 : BN / 32;
  static constexpr int SF_SLOT = 4 * 4 + 4 * SFB_COLS;
  static constexpr int SFB_OFF = 16;   // within a scale slot
  // (TSA: every TMEM column the accumulators leave, at most 8 slots)
  static constexpr int TSA_STAGES = ((BN <= 64 ? 256 : 512) - 2 * BN) / 32 > 8 ? 8 : ((BN <= 64 ? 256 : 512) - 2 * BN) / 32;
  // (W4A4: as many scale slots as the accumulators leave, at most 8; the
  // scales of a stage pass through the prologue warps, and a deeper ring
  // keeps more stages of that hand-over in flight)
  static constexpr int W4_STAGES = ((BN <= 64 ? 256 : 512) - ISSUERS * BN) / SF_SLOT > 8
                                       ? 8 : ((BN <= 64 ? 256 : 512) - ISSUERS * BN) / SF_SLOT;
  static constexpr int A_STAGES = W4A4 ? W4_STAGES : TSA ? TSA_STAGES : STATIC ? 0 : (BN == 64 ? 2 : 3);
  static constexpr int A_COLS = A_STAGES * (W4A4 ? SF_SLOT : TSA ? STAGE_K / 4 : STAGE_K / 2);
  // stages of a persistent CTA's next tile the prologue warps may prepare
  // before this tile's epilogue: at most its TMEM slots, and for W4A4 (whose
  // weight and x slots only the MMAs free, which wait for that epilogue) at
  // most the weight and x slots too, else the preparation would wait on
  // itself
  static constexpr int PREFILL_RAW = W4A4 ? (XST < WST ? XST : WST) : A_STAGES;
  static constexpr int PREFILL = PREFILL_RAW < A_STAGES ? PREFILL_RAW : A_STAGES;
  static constexpr int ACC_COL = A_COLS;
  static constexpr int ACC2_COL = ACC_COL + ISSUERS * BN;   // MLP: layer 2's accumulators
  // two accumulators where TMEM has room (static FP8 on e4m3 codes at 256-row
  // tiles: no A operand or scale slots in TMEM): the MMAs of a CTA's next
  // tile run while the epilogue reads the last one
  static constexpr int ACC_BUFS = (XQ && STATIC && BN == 256) ? 2 : 1;
  static constexpr int TMEM_COLS = pow2_at_least(A_COLS + (MLP ? 2 : ACC_BUFS) * ISSUERS * BN);
  static constexpr int BAR_OFF = B2_OFF + B2_BYTES;
  static constexpr int BAR_BYTES = 8 * 80;
  // each epilogue thread's row factor and bias, parked in shared memory over
  // the main loop instead of holding registers: [2][256] fp32
  static constexpr int EPI_OFF = BAR_OFF + BAR_BYTES;
  static constexpr int EPI_BYTES = 2 * 256 * 4;
  static constexpr int SMEM = EPI_OFF + EPI_BYTES + 1024;   // + alignment slack
  static constexpr uint32_t IDESC = W4A4 ? idesc_fp4(BN, MXS) : STATIC ? idesc_e4m3(BN) : idesc_bf16(BN);
  // warp 0 weight producer, 1 and 10 MMA issuers, 2..9 prologue/epilogue,
  // 11 x producer
  static constexpr int THREADS = 384;
  static_assert(A_COLS + (MLP ? 2 : ACC_BUFS) * ISSUERS * BN <= (BN <= 64 ? 256 : 512), "TMEM budget");
  static_assert(!(MLP && BN > 64), "the MLP runs x tiles of at most 64 rows");
  static_assert(!(STATIC && !XQ && BN > 128), "the fused static-FP8 tile holds at most 128 x rows");
  static_assert(!(W4A4 && BN < 32), "W4A4 x tiles hold 32 rows or more (one scale column per 32 rows)");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");   // (two CTAs per SM need <= 113 KB)
  static_assert(A_STAGES <= 8 && XST <= 8 && WST <= 8, "barrier arrays");
  static_assert(!TSA || QST >= 2, "operand ring");
  static_assert(RECV_BYTES % 16 == 0 && RECV_OFF % 16 == 0, "16-byte st.async targets");
};

// The work of one CTA: a list of (tile, k_begin, k_end) segments.
struct Work {
  int first_tile, tile_step, ntiles;  // tiles first_tile + i * tile_step, i < ntiles
  int kb, ke;                         // k-stage range within every tile
  __device__ int stages() const { return ntiles * (ke - kb); }
};

template <bool MLP>
__device__ __forceinline__ Work cta_work(const GemmParams& p) {
  Work w;
  if (MLP) {
    // rank q of the cluster computes layer 1's output tile q (all of K) for
    // the cluster's m-tile; that tile is layer 2's k-slice q
    w.first_tile = (int)cluster_rank() * p.m_tiles + (int)blockIdx.x / p.split;
    w.tile_step = 1;
    w.ntiles = 1;
    w.kb = 0;
    w.ke = p.k_stages;
  } else if (p.split > 1) {
    const int q = (int)cluster_rank();
    w.first_tile = blockIdx.x / p.split;
    w.tile_step = 1;
    w.ntiles = 1;
    w.kb = (int)((unsigned)(q * p.k_stages) / (unsigned)p.split);
    w.ke = (int)((unsigned)((q + 1) * p.k_stages) / (unsigned)p.split);
  } else {
    w.first_tile = blockIdx.x;
    w.tile_step = gridDim.x;
    w.ntiles = (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    w.kb = 0;
    w.ke = p.k_stages;
  }
  return w;
}

// One half (hp = 0: k-steps 0..3, hp = 1: 4..7 of this thread's k-half) of
// the operand a prologue thread produces per stage: 16 words of bf16x2 for
// weight row r, in TMEM column order.  Working in halves keeps the live
// registers of the unpack low.
template <int FMT>
__device__ __forceinline__ void prologue_half(const uint8_t* chunk, int r, int h, int hp, int mx_bias, uint32_t (&o)[16]) {
  if constexpr (FMT == FMT_FP8) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint4 v = lds128(chunk + ((h * 4 + hp * 2 + j) * TILE_N + r) * 16);
      unpack_e4m3(v.x, o + j * 8 + 0);
      unpack_e4m3(v.y, o + j * 8 + 2);
      unpack_e4m3(v.z, o + j * 8 + 4);
      unpack_e4m3(v.w, o + j * 8 + 6);
    }
  } else {
    const uint4 v = lds128(chunk + ((h * 2 + hp) * TILE_N + r) * 16);
    const uint8_t* sc = chunk + PACKED4_BYTES;
    uint32_t sa, sb;   // bf16x2 scale words of the two 8-word halves of v
    uint32_t zs2 = 0;   // asymmetric INT4: bf16(128 + z) twice
    if constexpr (FMT == FMT_INT4 || FMT == FMT_INT4A) {
      const uint32_t s = *reinterpret_cast<const uint16_t*>(sc + r * 2);
      sa = sb = s | (s << 16);
      if constexpr (FMT == FMT_INT4A) {
        const uint32_t zs = 0x4300u | sc[TILE_N * 2 + r];
        zs2 = zs | (zs << 16);
      }
    } else if constexpr (FMT == FMT_NVFP4) {
      const uint32_t c2 = *reinterpret_cast<const uint16_t*>(sc + (h * TILE_N + r) * 4 + hp * 2);
      const uint32_t a = nvfp4_scale_bf16(c2 & 0xFFu), b = nvfp4_scale_bf16(c2 >> 8);
      sa = a | (a << 16);
      sb = b | (b << 16);
    } else {  // MXFP4: one scale per 32 = per half
      const uint32_t c = *(sc + (h * TILE_N + r) * 2 + hp);
      const uint32_t a = mxfp4_scale_bf16(c, mx_bias);
      sa = sb = a | (a << 16);
    }
    if constexpr (FMT == FMT_INT4) {
      unpack_int4(v.x, sa, o + 0);
      unpack_int4(v.y, sa, o + 4);
      unpack_int4(v.z, sb, o + 8);
      unpack_int4(v.w, sb, o + 12);
    } else if constexpr (FMT == FMT_INT4A) {
      unpack_int4u(v.x, zs2, sa, o + 0);
      unpack_int4u(v.y, zs2, sa, o + 4);
      unpack_int4u(v.z, zs2, sb, o + 8);
      unpack_int4u(v.w, zs2, sb, o + 12);
    } else {
      unpack_e2m1(v.x, sa, o + 0);
      unpack_e2m1(v.y, sa, o + 4);
      unpack_e2m1(v.z, sb, o + 8);
      unpack_e2m1(v.w, sb, o + 12);
    }
  }
}

template <int FMT, int BN>
__device__ __forceinline__ void prologue_stage(const uint8_t* chunk, int r, int h, int mx_bias, uint32_t (&o)[32]) {
  prologue_half<FMT>(chunk, r, h, 0, mx_bias, *reinterpret_cast<uint32_t(*)[16]>(o));
  prologue_half<FMT>(chunk, r, h, 1, mx_bias, *reinterpret_cast<uint32_t(*)[16]>(o + 16));
}

// Static FP8: quantize the bf16 x tile (two SW128 boxes) into the e4m3 SW128
// B operand: q = e4m3(f32(x / s_x)), the IEEE quotient, RNE, saturating.
// (FAST: the quotient by e4m3_quotient; a separate loop, so the division is
// not evaluated alongside)
template <int BN, int NT, bool FAST>
__device__ __forceinline__ void quantize_x_tile_loop(const uint8_t* xs, uint8_t* qs, float s_x, float r_x, int tid) {
  // BN * 8 chunks of 16 codes; a compile-time count per thread, unrolled so
  // that a thread's chunks interleave (a few quantizing warps per SM
  // sub-partition leave issue slots to fill)
  constexpr int PER = (BN * 8 + NT - 1) / NT;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = tid + i * NT;
    if (BN * 8 % NT != 0 && c >= BN * 8) break;
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
        const float2 qv = FAST ? make_float2(e4m3_quotient(f0, s_x, r_x), e4m3_quotient(f1, s_x, r_x))
                               : make_float2(__fdiv_rn(f0, s_x), __fdiv_rn(f1, s_x));
        lohi[k] = (uint32_t)__nv_cvt_float2_to_fp8x2(qv, __NV_SATFINITE, __NV_E4M3);
      }
      out[i] = lohi[0] | (lohi[1] << 16);
    }
    sts128(qs + row * 128 + ((cc ^ (row & 7)) << 4), make_uint4(out[0], out[1], out[2], out[3]));
  }
}

template <int BN, int NT = 256>
__device__ __forceinline__ void quantize_x_tile(const uint8_t* xs, uint8_t* qs, float s_x, float r_x, int tid) {
  if (e4m3_quotient_ok(r_x))
    quantize_x_tile_loop<BN, NT, true>(xs, qs, s_x, r_x, tid);
  else
    quantize_x_tile_loop<BN, NT, false>(xs, qs, s_x, r_x, tid);
}

// QOUT: the output leaves as the next static-FP8 layer's e4m3 codes (a
// separate instantiation, so the common bf16 epilogue stays as compact as
// it can be)
// Back-to-back skinny calls share each SM: the next call's CTA lands while
// this call's CTA is still waiting for the previous grid, and after that wait
// this CTA still has to unpack the stages that did not fit in TMEM before
// it; two CTAs unpacking at once run at half speed each.  So a single-tile
// CTA with such stages marks its SM (its grid's tag) from the end of its
// early unpacks to the end of its late ones, and a CTA of another grid that
// lands on a marked SM holds its early unpacks (which only have to be done by
// the time its own wait returns) until the mark clears, or for at most
// kTurnWaitNs.  The table is a scheduling hint only: a stale or torn entry
// costs at most that bounded delay, never a result.
__device__ uint32_t g_sm_turn[256];
constexpr uint64_t kTurnWaitNs = 6000;

__device__ __forceinline__ uint32_t sm_id() {
  uint32_t s;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(s));
  return s & 255u;
}
// an odd (so nonzero) tag of this launch
__device__ __forceinline__ uint32_t grid_tag() {
  uint64_t g;
  asm volatile("mov.u64 %0, %%gridid;" : "=l"(g));
  return (uint32_t)g * 2u + 1u;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
// wait (bounded) until no other grid's CTA holds this SM's mark; false if
// the wait gave up, after clearing the mark it gave up on (so that a mark
// left behind delays one CTA, not every later one)
__device__ __forceinline__ bool sm_turn_wait(uint32_t sm, uint32_t tag) {
  uint32_t v = ld_relaxed_gpu(&g_sm_turn[sm]);
  if (v == 0u || v == tag) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(128);
    const uint32_t w = ld_relaxed_gpu(&g_sm_turn[sm]);
    if (w == 0u || w == tag) return true;
    if (w != v) {
      v = w;   // another CTA took the mark: its own turn starts now
      continue;
    }
    if (globaltimer_ns() - t0 >= kTurnWaitNs) {
      atomicCAS(&g_sm_turn[sm], v, 0u);
      return false;
    }
  }
}

template <int FMT, int BN, bool QOUT>
__global__ void __launch_bounds__(384, BN <= 64 ? 2 : 1) dq_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                                                         const GemmParams p) {
  using C = GemmCfg<FMT, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* x_ring = smem + C::X_RING_OFF;
  uint8_t* w_ring = smem + C::W_RING_OFF;
  uint64_t* full_w = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);   // [8] weight chunk landed
  uint64_t* wempty = full_w + 8;          // [8] weight slot read (prologue, or MMAs for static FP8)
  uint64_t* full_x = wempty + 8;          // [8] x tile landed
  uint64_t* xempty = full_x + 8;          // [8] x slot read by the MMAs
  uint64_t* aready = xempty + 8;          // [8] operand written: TMEM A slot (bf16) / e4m3 x (static, per x slot)
  uint64_t* aempty = aready + 8;          // [8] TMEM A slot read by the MMAs
  uint64_t* acc_full = aempty + 8;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;        // [2], one per MMA issuer
  uint64_t* recv_bar = drain + 2;         // split-K: the peers' partials and flags have landed
  uint64_t* full_w2 = recv_bar + 1;       // MLP: layer 2's weight chunk landed
  uint64_t* b2ready = full_w2 + 1;        // MLP: layer 2's B operand (hidden codes) written
  uint64_t* acc2_full = b2ready + 1;      // MLP: layer 2's accumulators complete
  uint64_t* xready = acc2_full + 1;       // [8] fused static with A in TMEM: operand slot written
  uint64_t* qempty = xready + 8;          // [8]   ... and read by the MMAs
  uint64_t* acc_full_b[2] = {acc_full, qempty + 8};        // the second accumulator's, if any
  uint64_t* acc_empty_b[2] = {acc_empty, qempty + 9};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* recv = reinterpret_cast<float*>(smem + C::RECV_OFF);             // [S][128][BN/S]
  uint32_t* rflag = reinterpret_cast<uint32_t*>(smem + C::RFLAG_OFF);     // [S][4]: sender rank, row quadrant

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool arrived = false;   // split-K: this thread has arrived at the closing cluster barrier (warp-uniform)
  // wait control, rebuilt from kernel parameters at each wait so that it
  // holds no registers across the long loops
  const auto ctl = [&] { return WaitCtl{abort_flag, p.status, p.timeout_ns}; };
  const auto ctl_no_abort = [&] { return WaitCtl{nullptr, p.status, p.drain_ns}; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&full_w[s], 1);
      mbar_init(&wempty[s], C::SS ? C::ISSUERS : C::TSA ? 4 : 8);
      mbar_init(&full_x[s], 1);
      mbar_init(&xempty[s], C::TSA ? 4 : C::ISSUERS);   // (TSA: the quantizing warps free the bf16 slot)
      mbar_init(&aready[s], C::TSA ? 4 : 8);
      mbar_init(&xready[s], 4);
      mbar_init(&qempty[s], C::ISSUERS);
      mbar_init(&aempty[s], C::ISSUERS);
    }
    mbar_init(acc_full, C::ISSUERS);
    mbar_init(acc_empty, 8);
    mbar_init(acc_full_b[1], C::ISSUERS);
    mbar_init(acc_empty_b[1], 8);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(recv_bar, 1);
    mbar_init(full_w2, 1);
    mbar_init(b2ready, 8);
    mbar_init(acc2_full, C::ISSUERS);
    if (p.split > 1) {
      // every peer sends this CTA its partial of the columns this CTA owns
      // plus one validity word per 32 rows, whether or not its own work
      // succeeded
      const int cmax = BN / p.split;
      mbar_arrive_expect_tx(recv_bar, (uint32_t)((p.split - 1) * (TILE_N * cmax * 4 + 4 * 4)));
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::TMEM_COLS);
  if (warp == 11 && lane == 0) prefetch_tmap(&tmap_x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // split-K: no CTA sends into a peer before the peer's receive barrier is
  // initialized (this barrier runs before the grid-dependency wait)
  if (p.split > 1) cluster_sync();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();   // the next call may start its own prologue now

  const Work wk = cta_work<C::MLP>(p);
  const int KS = p.k_stages;
  const int nst = wk.ke - wk.kb;   // stages per tile
  // (all ring positions are kept in counters: an integer division by a
  // runtime value costs a long dependent chain on the single-thread roles)

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    // Weights do not depend on earlier grids: they stream from the start, as
    // far ahead as the ring allows.
    if (lane == 0) {
      if constexpr (C::MLP) {
        // layer 2's weight chunk for this CTA's k-slice: its single output
        // tile (N2 <= 128), stage q = the cluster rank
        mbar_arrive_expect_tx(full_w2, C::CHUNK);
        bulk_g2s(smem + C::W2_OFF, p.w2chunks + (size_t)cluster_rank() * C::CHUNK, C::CHUNK, full_w2);
      }
      const int total = wk.stages();
      int ks = wk.kb, tile = wk.first_tile, ws = 0, it = 0;
      uint32_t wph = 0;
      const uint8_t* wsrc = p.wchunks + (size_t)(tile / p.m_tiles) * KS * C::CHUNK;
      for (; it < total; ++it) {
        if (it >= C::WST && !mbar_wait(&wempty[ws], wph ^ 1, ctl())) break;
        mbar_arrive_expect_tx(&full_w[ws], C::CHUNK);
        bulk_g2s(w_ring + ws * C::W_SLOT, wsrc + (size_t)ks * C::CHUNK, C::CHUNK, &full_w[ws]);
        if (++ks == wk.ke) {
          ks = wk.kb;
          tile += wk.tile_step;
          wsrc = p.wchunks + (size_t)(tile / p.m_tiles) * KS * C::CHUNK;
        }
        if (++ws == C::WST) {
          ws = 0;
          wph ^= 1;
        }
      }
      // never leave with copies in flight: wait for the chunks issued last
      for (int i = it > C::WST ? it - C::WST : 0; i < it; ++i)
        mbar_wait(&full_w[i % C::WST], (i / C::WST) & 1, ctl_no_abort());
      if constexpr (C::MLP) mbar_wait(full_w2, 0, ctl_no_abort());
    }
    __syncwarp();
  } else if (warp == 11) {
    // ------------------------------------------------------------ x producer
    // one stage's x copy into slot xs (bf16 boxes, or codes and W4A4's
    // scale words)
    const auto issue_x = [&](int xs, int ks, int m_tile) {
      uint8_t* xd = x_ring + xs * C::X_SLOT;
      if constexpr (C::XQ) {
        // codes straight into the operand buffer of the slot (128 bytes
        // of each row per stage), and for W4A4 the stage's scale words
        mbar_arrive_expect_tx(&full_x[xs], C::Q_BYTES + C::XSF_BYTES);
        tma_load_2d(xd + C::Q_OFF, &tmap_x, ks * 128, m_tile * BN, &full_x[xs]);
        if constexpr (C::W4A4)
          bulk_g2s(xd + C::XSF_OFF, p.xsf + ((size_t)m_tile * KS + ks) * 4 * BN, C::XSF_BYTES, &full_x[xs]);
      } else {
        mbar_arrive_expect_tx(&full_x[xs], C::X_BYTES);
        if (p.x3d) {
          tma_load_3d(xd, &tmap_x, 0, m_tile * BN, ks * 2, &full_x[xs]);
        } else {
          tma_load_2d(xd, &tmap_x, ks * STAGE_K, m_tile * BN, &full_x[xs]);
          tma_load_2d(xd + BN * 128, &tmap_x, ks * STAGE_K + 64, m_tile * BN, &full_x[xs]);
        }
      }
    };
    // A single-tile CTA's first ring of x copies is issued by that many
    // lanes at once (one stage each): on the critical path after the wait,
    // one thread issuing them in turn took ~0.3 us a copy.  The rest, and
    // every copy of a persistent CTA, come from lane 0 in ring order.
    const int nfirst = wk.ntiles == 1 ? (nst < C::XST ? nst : C::XST) : 0;
    if (lane < nfirst) {
      pdl_wait();   // x may be the previous grid's output
      const int m_tile = wk.first_tile - (wk.first_tile / p.m_tiles) * p.m_tiles;
      issue_x(lane, wk.kb + lane, m_tile);
    }
    __syncwarp();
    if (lane == 0) {
      if (nfirst == 0) pdl_wait();
      int it = nfirst, xs = nfirst == C::XST ? 0 : nfirst;
      uint32_t xph = nfirst == C::XST ? 1u : 0u;
      bool ok = true;
      for (int t = 0; ok && t < wk.ntiles; ++t) {
        const int tile = wk.first_tile + t * wk.tile_step;
        const int m_tile = tile - (tile / p.m_tiles) * p.m_tiles;
        for (int ks = wk.kb + (t == 0 ? nfirst : 0); ks < wk.ke; ++ks, ++it) {
          if (it >= C::XST && !mbar_wait(&xempty[xs], xph ^ 1, ctl())) { ok = false; break; }
          issue_x(xs, ks, m_tile);
          if (++xs == C::XST) {
            xs = 0;
            xph ^= 1;
          }
        }
      }
      for (int i = it > C::XST ? it - C::XST : 0; i < it; ++i)
        mbar_wait(&full_x[i % C::XST], (i / C::XST) & 1, ctl_no_abort());
    }
    __syncwarp();
  } else if (warp == 1 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0 && (warp == 1 || C::ISSUERS == 2)) {
      const int which = warp == 1 ? 0 : 1;   // k-steps [which*KK, (which+1)*KK) of each stage
      constexpr int KK = C::KK;
      int ws = 0, xs = 0, as = 0;
      uint32_t wph = 0, xph = 0, aph = 0;
      bool ok = true, issued = false;
      for (int t = 0; ok && t < wk.ntiles; ++t) {
        const int ab = C::ACC_BUFS == 2 ? (t & 1) : 0;              // this tile's accumulator
        const uint32_t acc_ph = (uint32_t)(C::ACC_BUFS == 2 ? (t >> 1) : t) & 1u;
        const uint32_t d_tmem = tmem + C::ACC_COL + ab * (C::ISSUERS * BN) + which * BN;
        if (!mbar_wait(acc_empty_b[ab], acc_ph ^ 1, ctl())) break;
        tc_fence_after();
        for (int j = 0; j < nst; ++j) {
          const uint32_t xb = smem_u32(x_ring + xs * C::X_SLOT);
          if constexpr (C::W4A4) {
            // both operands in shared memory (k-step t = 32 bytes into each
            // 128-byte row), the stage's block scales in TMEM slot `as`
            if (!mbar_wait(&full_w[ws], wph, ctl()) || !mbar_wait(&full_x[xs], xph, ctl()) ||
                !mbar_wait(&aready[as], aph, ctl())) { ok = false; break; }
            tc_fence_after();
            const uint32_t wb = smem_u32(w_ring + ws * C::W_SLOT) + which * KK * 32;
            const uint32_t qb = xb + C::Q_OFF + which * KK * 32;
            const uint32_t sf = tmem + as * C::SF_SLOT;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
              const int t = which * KK + kk;
              mma_fp4_ss<C::MXS>(d_tmem, sdesc_sw128(wb + kk * 32), sdesc_sw128(qb + kk * 32), C::IDESC, sf + 4 * t,
                                 sf + C::SFB_OFF + C::SFB_COLS * t, (j > 0 || kk > 0) ? 1u : 0u);
            }
            issued = true;
            tc_commit(&wempty[ws]);
            tc_commit(&aempty[as]);
            if (++ws == C::WST) {
              ws = 0;
              wph ^= 1;
            }
            if (++as == C::A_STAGES) {
              as = 0;
              aph ^= 1;
            }
          } else if constexpr (!C::STATIC) {
            if (!mbar_wait(&full_x[xs], xph, ctl()) || !mbar_wait(&aready[as], aph, ctl())) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_tmem = tmem + as * (STAGE_K / 2) + which * KK * 8;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
              // k-step ks of the stage: 64-k box ks / 4 of the x slot, 32 bytes per k-step in its rows
              const int ks = which * KK + kk;
              const uint32_t bx = xb + (ks >> 2) * BN * 128 + (ks & 3) * 32;
              mma_bf16_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(bx), C::IDESC, (j > 0 || kk > 0) ? 1u : 0u);
            }
            issued = true;
            tc_commit(&aempty[as]);
            if (++as == C::A_STAGES) {
              as = 0;
              aph ^= 1;
            }
          } else if constexpr (C::TSA) {
            // A: the e4m3 weight stage in TMEM slot `as` (8 columns per
            // k-step of 32); B: the e4m3 operand in slot xs of the operand
            // ring (xs / xph count that ring here)
            if (!mbar_wait(&aready[as], aph, ctl()) || !mbar_wait(&xready[xs], xph, ctl())) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_tmem = tmem + as * (STAGE_K / 4) + which * KK * 8;
            const uint32_t qb = smem_u32(smem + C::Q_RING_OFF + xs * C::Q_SLOT) + which * KK * 32;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk)
              mma_f8_ts(d_tmem, a_tmem + kk * 8, sdesc_sw128(qb + kk * 32), C::IDESC, (j > 0 || kk > 0) ? 1u : 0u);
            issued = true;
            tc_commit(&aempty[as]);
            if (++as == C::A_STAGES) {
              as = 0;
              aph ^= 1;
            }
          } else {
            // (x quantized in the kernel: the prologue warps signal each x
            // slot's e4m3 operand; quantized beforehand: the x copy itself)
            if (!mbar_wait(&full_w[ws], wph, ctl()) ||
                !mbar_wait(C::XQ ? &full_x[xs] : &aready[xs], xph, ctl())) { ok = false; break; }
            tc_fence_after();
            const uint32_t wb = smem_u32(w_ring + ws * C::W_SLOT) + which * KK * 32;
            const uint32_t qb = xb + C::Q_OFF + which * KK * 32;
#pragma unroll
            for (int kk = 0; kk < KK; ++kk)
              mma_f8_ss(d_tmem, sdesc_sw128(wb + kk * 32), sdesc_sw128(qb + kk * 32), C::IDESC,
                        (j > 0 || kk > 0) ? 1u : 0u);
            issued = true;
            tc_commit(&wempty[ws]);
            if (++ws == C::WST) {
              ws = 0;
              wph ^= 1;
            }
          }
          if constexpr (C::TSA) {
            tc_commit(&qempty[xs]);
            if (++xs == C::QST) {
              xs = 0;
              xph ^= 1;
            }
          } else {
            tc_commit(&xempty[xs]);
            if (++xs == C::XST) {
              xs = 0;
              xph ^= 1;
            }
          }
        }
        if (!ok) break;
        tc_commit(acc_full_b[ab]);
      }
      if constexpr (C::MLP) {
        // layer 2 on this CTA's k-slice: A = layer 2's weight chunk, B = the
        // hidden activations' e4m3 codes the epilogue warps wrote
        if (ok && mbar_wait(full_w2, 0, ctl()) && mbar_wait(b2ready, 0, ctl())) {
          tc_fence_after();
          const uint32_t wb = smem_u32(smem + C::W2_OFF) + which * KK * 32;
          const uint32_t bb = smem_u32(smem + C::B2_OFF) + which * KK * 32;
          const uint32_t d2 = tmem + C::ACC2_COL + which * BN;
#pragma unroll
          for (int kk = 0; kk < KK; ++kk)
            mma_f8_ss(d2, sdesc_sw128(wb + kk * 32), sdesc_sw128(bb + kk * 32), C::IDESC, kk > 0 ? 1u : 0u);
          issued = true;
          tc_commit(acc2_full);
        }
      }
      // all MMAs this thread issued must finish before TMEM is released (a
      // commit with no MMA before it would never arrive: an issuer that gave
      // up before its first MMA has nothing to drain)
      if (issued) {
        tc_commit(&drain[which]);
        mbar_wait(&drain[which], 0, ctl_no_abort());
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ prologue + epilogue
    const int dw = warp - 2;            // 0..7
    const int qd = warp & 3;            // TMEM lane quadrant this warp may access
    const int h = dw >> 2;              // k-half of the stage / column half of the tile
    const int r = qd * 32 + lane;       // weight row in the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    constexpr int HALF = BN / 2;
    // 256-row x tiles stream the accumulator out in chunks (its 128 columns
    // per thread would not fit in registers); smaller tiles hold it whole
    constexpr bool CHUNKED = BN > 128;
    float acc[CHUNKED ? 1 : HALF];
#pragma unroll
    for (int i = 0; i < (CHUNKED ? 1 : HALF); ++i) acc[i] = 0.f;
    float* epi = reinterpret_cast<float*>(smem + C::EPI_OFF);   // [2][256]: this thread's slots only
    const int et = threadIdx.x - 64;
    int tile = 0;
    int ws = 0, xs = 0, as = 0, qs = 0;     // ring positions, kept across the tiles of a persistent CTA
    uint32_t wph = 0, xph = 0, aph = 0, qph = 0;
    int pre = 0;                            // stages of this tile already handled (prefilled during the last)
    bool ok = true, have_acc = false;
    bool marked = false;                    // this CTA's mark in g_sm_turn is set (one thread)
    for (int t = 0; ok && t < wk.ntiles; ++t) {
      tile = wk.first_tile + t * wk.tile_step;
      // this row's epilogue factor and bias: read-only, fetched now so the
      // loads are long done when the epilogue needs them
      {
        const int n_row = (tile / p.m_tiles) * TILE_N + r;
        float e_sig = p.sigma, e_bias = 0.f;
        if (n_row < p.N) {
          if (p.col_scale) e_sig = p.sigma * ld_nc_f32(p.col_scale + n_row);
          if (p.bias) e_bias = ld_nc_bf16(p.bias + n_row);
        }
        if constexpr (FMT == FMT_W4A4NV) {
          // the activation's global scale is this call's quantizer output:
          // read only once that grid has completed (and past any cache)
          pdl_wait();
          e_sig *= *reinterpret_cast<const volatile float*>(p.gx);
        }
        epi[et] = e_sig;
        epi[256 + et] = e_bias;
      }
      if constexpr (C::W4A4) {
        // the stage's block scales into TMEM slot `as`: every lane quadrant
        // holds all rows (lane i, column c = row 32c + i); this warp writes
        // the k-steps t = 2h, 2h + 1 into its own quadrant, from the weight
        // chunk's and the x slot's scale words ([t][row] each)
        constexpr int NB = BN / 32;
        const auto sf_stage = [&]() -> bool {
          if (!mbar_wait_warp(&full_w[ws], wph, ctl()) || !mbar_wait_warp(&full_x[xs], xph, ctl())) return false;
          const uint32_t* wsf = reinterpret_cast<const uint32_t*>(w_ring + ws * C::W_SLOT + W4_SF_OFF);
          const uint32_t* xsf = reinterpret_cast<const uint32_t*>(x_ring + xs * C::X_SLOT + C::XSF_OFF);
          uint32_t va[8], vb[2 * NB];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int t = 2 * h + u;
#pragma unroll
            for (int c = 0; c < 4; ++c) va[u * 4 + c] = wsf[t * TILE_N + c * 32 + lane];
#pragma unroll
            for (int c = 0; c < NB; ++c) vb[u * NB + c] = xsf[t * BN + c * 32 + lane];
          }
          if (!mbar_wait_warp(&aempty[as], aph ^ 1, ctl())) return false;
          tc_fence_after();
          const uint32_t ts = tmem + lane_base + as * C::SF_SLOT;
          tmem_st_cols<8>(ts + 8 * h, va);
#pragma unroll
          for (int u = 0; u < 2; ++u) tmem_st_cols<NB>(ts + C::SFB_OFF + C::SFB_COLS * (2 * h + u), vb + u * NB);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&aready[as]);
          if (++ws == C::WST) {
            ws = 0;
            wph ^= 1;
          }
          if (++xs == C::XST) {
            xs = 0;
            xph ^= 1;
          }
          if (++as == C::A_STAGES) {
            as = 0;
            aph ^= 1;
          }
          return true;
        };
        // this tile's stages not handled yet, then the next tile's first
        // ones (their TMEM slots free up as this tile's MMAs complete), so
        // that its MMAs can start as soon as the accumulator is read
        for (int j = pre; j < nst; ++j)
          if (!sf_stage()) { ok = false; break; }
        pre = 0;
        if (ok && t + 1 < wk.ntiles) {
          for (int j = 0; j < (nst < C::PREFILL ? nst : C::PREFILL); ++j, ++pre)
            if (!sf_stage()) { ok = false; break; }
        }
      } else if constexpr (C::TSA) {
        if (h == 0) {
          // warps 2..5, one per lane quadrant: weight row r's 128 e4m3 codes
          // from the swizzled image into TMEM slot `as` (the weights need no
          // x: these run ahead of the grid-dependency wait, A_STAGES deep)
          for (int j = 0; j < nst; ++j) {
            if (!mbar_wait_warp(&full_w[ws], wph, ctl())) { ok = false; break; }
            // (in two halves of 64 codes, as the unpack does, to keep the
            // live registers low; the slot is free once the second is read)
            const uint8_t* row = w_ring + ws * C::W_SLOT + r * 128;
            const uint32_t ta = tmem + lane_base + as * (STAGE_K / 4);
            uint32_t o[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = lds128(row + ((c ^ (r & 7)) << 4));
              o[4 * c] = v.x;
              o[4 * c + 1] = v.y;
              o[4 * c + 2] = v.z;
              o[4 * c + 3] = v.w;
            }
            if (!mbar_wait_warp(&aempty[as], aph ^ 1, ctl())) { ok = false; break; }
            tc_fence_after();
            tmem_st16(ta, o);
#pragma unroll
            for (int c = 4; c < 8; ++c) {
              const uint4 v = lds128(row + ((c ^ (r & 7)) << 4));
              o[4 * c - 16] = v.x;
              o[4 * c - 15] = v.y;
              o[4 * c - 14] = v.z;
              o[4 * c - 13] = v.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[ws]);
            tmem_st16(ta + 16, o);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&aready[as]);
            if (++ws == C::WST) {
              ws = 0;
              wph ^= 1;
            }
            if (++as == C::A_STAGES) {
              as = 0;
              aph ^= 1;
            }
          }
        } else {
          // warps 6..9: quantize each bf16 x tile into a slot of the operand
          // ring (qs), then free the bf16 slot for the next load
          for (int j = 0; j < nst; ++j) {
            if (!mbar_wait_warp(&full_x[xs], xph, ctl())) { ok = false; break; }
            if (!mbar_wait_warp(&qempty[qs], qph ^ 1, ctl())) { ok = false; break; }
            quantize_x_tile<BN, 128>(x_ring + xs * C::X_SLOT, smem + C::Q_RING_OFF + qs * C::Q_SLOT, p.s_x, p.r_x, et - 128);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&xready[qs]);
              mbar_arrive(&xempty[xs]);
            }
            if (++xs == C::XST) {
              xs = 0;
              xph ^= 1;
            }
            if (++qs == C::QST) {
              qs = 0;
              qph ^= 1;
            }
          }
        }
      } else if constexpr (!C::STATIC) {
        // the weight operand needs no x: the first A_STAGES stages are
        // unpacked before the grid-dependency wait has even returned
        const auto unpack_stage = [&]() -> bool {
          if (!mbar_wait_warp(&full_w[ws], wph, ctl())) return false;
          // unpack the first half while the TMEM slot may still be read by
          // the MMAs of an earlier stage, then store it, unpack the second
          // half (after which the weight slot is free) and store it
          const uint8_t* chunk = w_ring + ws * C::W_SLOT;
          const uint32_t ta = tmem + lane_base + as * (STAGE_K / 2) + h * 32;
          uint32_t o[16];
          prologue_half<FMT>(chunk, r, h, 0, p.mx_bias, o);
          if (!mbar_wait_warp(&aempty[as], aph ^ 1, ctl())) return false;
          tc_fence_after();
          tmem_st16(ta, o);
          prologue_half<FMT>(chunk, r, h, 1, p.mx_bias, o);
          __syncwarp();
          if (lane == 0) mbar_arrive(&wempty[ws]);
          tmem_st16(ta + 16, o);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&aready[as]);
          if (++ws == C::WST) {
            ws = 0;
            wph ^= 1;
          }
          if (++as == C::A_STAGES) {
            as = 0;
            aph ^= 1;
          }
          return true;
        };
        // this tile's stages not unpacked yet, then the next tile's first
        // ones (their TMEM slots free up as this tile's MMAs complete), so
        // that its MMAs can start as soon as the accumulator is read.
        // A single-tile CTA takes turns with the other grid's CTA on its SM
        // (g_sm_turn): its early unpacks wait for that CTA's late ones, and
        // it marks the SM while its own late unpacks are pending.
        const bool turns = wk.ntiles == 1 && nst > C::A_STAGES;
        if (turns && lane == 0) sm_turn_wait(sm_id(), grid_tag());
        __syncwarp();
        for (int j = pre; j < nst; ++j) {
          if (!unpack_stage()) { ok = false; break; }
          if (turns && j == C::A_STAGES - 1 && warp == 2 && lane == 0) {
            atomicExch(&g_sm_turn[sm_id()], grid_tag());
            marked = true;
          }
        }
        if (marked) {
          atomicCAS(&g_sm_turn[sm_id()], grid_tag(), 0u);
          marked = false;
        }
        pre = 0;
        if (ok && t + 1 < wk.ntiles) {
          for (int j = 0; j < (nst < C::PREFILL ? nst : C::PREFILL); ++j, ++pre)
            if (!unpack_stage()) { ok = false; break; }
        }
      } else {
        // static FP8: quantize each x tile into the e4m3 half of its slot
        // (the slot was refilled only after its previous MMAs completed);
        // pre-quantized x needs nothing here (the MMAs wait for its copy)
        if constexpr (!C::XQ) {
          for (int j = 0; j < nst; ++j) {
            if (!mbar_wait_warp(&full_x[xs], xph, ctl())) { ok = false; break; }
            uint8_t* xd = x_ring + xs * C::X_SLOT;
            quantize_x_tile<BN>(xd, xd + C::Q_OFF, p.s_x, p.r_x, et);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&aready[xs]);
            if (++xs == C::XST) {
              xs = 0;
              xph ^= 1;
            }
          }
        }
      }
      if (!ok) break;
      // ---- epilogue of this tile
      const int ab = C::ACC_BUFS == 2 ? (t & 1) : 0;                  // its accumulator
      const uint32_t acc_ph = (uint32_t)(C::ACC_BUFS == 2 ? (t >> 1) : t) & 1u;
      if (!mbar_wait_warp(acc_full_b[ab], acc_ph, ctl())) { ok = false; break; }
      tc_fence_after();
      if constexpr (CHUNKED) {
        // one accumulator (one issuer): the thread's 128 columns read 32 at
        // a time and kept as finished outputs (bf16 pairs, or e4m3 quads),
        // the accumulator released after the last read, then everything
        // stored (so the stores overlap the next tile's MMAs)
        const int n_row = (tile / p.m_tiles) * TILE_N + r, m_tile = tile % p.m_tiles;
        const float e_sig = epi[et], e_bias = epi[256 + et];
        constexpr int PW = QOUT ? HALF / 4 : HALF / 2;   // packed words of outputs
        uint32_t pk[PW];
#pragma unroll
        for (int c32 = 0; c32 < HALF / 32; ++c32) {
          float a[32];
          tmem_ld32(tmem + lane_base + C::ACC_COL + ab * BN + h * HALF + c32 * 32, a);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += (QOUT ? 4 : 2)) {
            if constexpr (!QOUT) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(fmaf(a[i], e_sig, e_bias), fmaf(a[i + 1], e_sig, e_bias));
              pk[(c32 * 32 + i) / 2] = *reinterpret_cast<const uint32_t*>(&v2);
            } else {
              uint32_t w = 0;
#pragma unroll
              for (int k = 0; k < 4; ++k) w |= (uint32_t)out_code(p, fmaf(a[i + k], e_sig, e_bias)) << (8 * k);
              pk[(c32 * 32 + i) / 4] = w;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty_b[ab]);
        if (n_row < p.N) {
#pragma unroll
          for (int i = 0; i < HALF; ++i) {
            const int m = m_tile * BN + h * HALF + i;
            if (m < p.M) {
              if constexpr (!QOUT)
                p.y[(size_t)m * p.N + n_row] = __ushort_as_bfloat16((unsigned short)(pk[i / 2] >> (16 * (i & 1))));
              else
                p.yq[(size_t)m * p.N + n_row] = (uint8_t)(pk[i / 4] >> (8 * (i & 3)));
            }
          }
        }
        have_acc = true;
        continue;
      } else {
#pragma unroll
      for (int c8 = 0; c8 < HALF / 8; ++c8) {
        float a1[8];
        tmem_ld8(tmem + lane_base + C::ACC_COL + h * HALF + c8 * 8, *reinterpret_cast<float(*)[8]>(acc + c8 * 8));
        tmem_ld8(tmem + lane_base + C::ACC_COL + BN + h * HALF + c8 * 8, a1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[c8 * 8 + i] += a1[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      have_acc = true;
      if constexpr (C::MLP) {
        // layer 1's epilogue: h = bf16(acc * s_x1 * s_w1[n] + b1[n]) for this
        // thread's hidden unit n (tile q, row r) and the rows m of its half;
        // the code e4m3(h / s_x2) is layer 2's B operand at (row m, k = r)
        // (128-byte swizzled K-major rows), and h goes out if asked for
        have_acc = false;
        const int n1 = (tile / p.m_tiles) * TILE_N + r, m_tile = tile % p.m_tiles;
        const float e_sig = epi[et], e_bias = epi[256 + et];
        uint8_t* b2 = smem + C::B2_OFF;
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const int mm = h * HALF + i;
          const float v = fmaf(acc[i], e_sig, e_bias);
          const int m = m_tile * BN + mm;
          if (p.h_out && m < p.M) p.h_out[(size_t)m * p.N + n1] = __float2bfloat16_rn(v);
          b2[mm * 128 + (((r >> 4) ^ (mm & 7)) << 4) + (r & 15)] = out_code(p, v);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(b2ready);
        // layer 2's factors for its output row n2 = r (one tile of <= 128)
        {
          float e_sig2 = p.s_out, e_bias2 = 0.f;
          if (r < p.N2) {
            e_sig2 = p.s_out * ld_nc_f32(p.col_scale2 + r);
            if (p.bias2) e_bias2 = ld_nc_bf16(p.bias2 + r);
          }
          epi[et] = e_sig2;
          epi[256 + et] = e_bias2;
        }
        if (!mbar_wait_warp(acc2_full, 0, ctl())) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c8 = 0; c8 < HALF / 8; ++c8) {
          float a1[8];
          tmem_ld8(tmem + lane_base + C::ACC2_COL + h * HALF + c8 * 8, *reinterpret_cast<float(*)[8]>(acc + c8 * 8));
          tmem_ld8(tmem + lane_base + C::ACC2_COL + BN + h * HALF + c8 * 8, a1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[c8 * 8 + i] += a1[i];
        }
        have_acc = true;
      }
      // (no grid-dependency wait here: the producer's wait precedes the x
      // loads this accumulator depends on, so every earlier grid is done)
      if (p.split == 1) {
        const int n_row = (tile / p.m_tiles) * TILE_N + r, m_tile = tile % p.m_tiles;
        const float e_sig = epi[et], e_bias = epi[256 + et];
        if (n_row < p.N) {
          if constexpr (!QOUT) {
#pragma unroll
            for (int i = 0; i < HALF; ++i) {
              const int m = m_tile * BN + h * HALF + i;
              if (m < p.M) p.y[(size_t)m * p.N + n_row] = __float2bfloat16_rn(fmaf(acc[i], e_sig, e_bias));
            }
          } else {
#pragma unroll
            for (int i = 0; i < HALF; ++i) {
              const int m = m_tile * BN + h * HALF + i;
              if (m < p.M) p.yq[(size_t)m * p.N + n_row] = out_code(p, fmaf(acc[i], e_sig, e_bias));
            }
          }
        }
      }
      }   // !CHUNKED
    }
    if (!ok) *abort_flag = 1;

    if constexpr (!CHUNKED) if (p.split > 1) {
      // ---- cluster split-K by push.  Rank q owns the tile's columns
      // [q*BN/S, (q+1)*BN/S).  Every CTA sends each peer d its partial of
      // d's columns with st.async straight into d's receive area (whose
      // barrier counts the bytes).  Each sending warp adds one word saying
      // whether its 32 rows are valid (it held its accumulator); it sends
      // even after an abort, so that every receive completes.  The threads
      // holding this CTA's own columns then add the S partials in rank order
      // (deterministic) and store y where every partial of their rows was
      // valid.  No CTA leaves before every CTA of the cluster has received
      // everything sent to it (the closing cluster barrier below).
      const int S = p.split;
      const int q = (int)cluster_rank();
      const int cmax = BN / S;
      const uint32_t good = (ok && have_acc) ? 1u : 0u;   // warp-uniform
      const int lg_cmax = __ffs(cmax) - 1;                 // cmax is a power of two
      // (compact code: this part runs once per call, its instructions are
      // fetched cold, and each one costs more than its work)
      if (cmax >= 4) {
#pragma unroll
        for (int i = 0; i < HALF; i += 4) {
          const int c = h * HALF + i;                  // this thread's columns c .. c+3 lie in one owner's range
          const int d = c >> lg_cmax;
          float* slot = recv + (q * TILE_N + r) * cmax + (c & (cmax - 1));
          if (d == q)
            *reinterpret_cast<float4*>(slot) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
          else
            st_async_v4(dsmem_addr(slot, (uint32_t)d), acc[i], acc[i + 1], acc[i + 2], acc[i + 3],
                        dsmem_addr(recv_bar, (uint32_t)d));
        }
      } else {
#pragma unroll
        for (int i = 0; i < HALF; i += 2) {
          const int c = h * HALF + i;
          const int d = c >> lg_cmax;
          float* slot = recv + (q * TILE_N + r) * cmax + (c & (cmax - 1));
          if (d == q)
            *reinterpret_cast<float2*>(slot) = make_float2(acc[i], acc[i + 1]);
          else
            st_async_v2(dsmem_addr(slot, (uint32_t)d), acc[i], acc[i + 1], dsmem_addr(recv_bar, (uint32_t)d));
        }
      }
      // this warp's validity word, to every peer it sent rows to: the owners
      // of the columns in half h, rflag[sender rank][row quadrant]
      if (lane == 0) {
        for (int d = (h * HALF) >> lg_cmax; d < ((h + 1) * HALF) >> lg_cmax; ++d)
          if (d != q) st_async_u32(dsmem_addr(rflag + q * 4 + qd, (uint32_t)d), good, dsmem_addr(recv_bar, (uint32_t)d));
      }
      // the threads that hold this CTA's own columns reduce them: row r,
      // columns [q*cmax, (q+1)*cmax), the S partials in rank order (this
      // thread wrote its own partial into slot q above)
      if (h == (q * cmax) / HALF) {
        const WaitCtl rx_ctl{nullptr, p.status, 2 * p.drain_ns};
        int rx = 1;
        if (lane == 0) rx = mbar_wait_cluster(recv_bar, 0, rx_ctl) ? 1 : 0;
        rx = __shfl_sync(0xFFFFFFFFu, rx, 0);
        if (rx) mbar_try_wait_cluster(recv_bar, 0);
        // nothing more lands in this CTA: arrive at the closing barrier now,
        // so that it never waits on this CTA's stores
        cluster_arrive_relaxed();
        arrived = true;
        bool all_good = good && rx;
        for (int pr = 0; pr < S; ++pr) all_good = all_good && (pr == q || rflag[pr * 4 + qd] != 0u);
        // (MLP: layer 2's single output tile, N2 columns of y)
        const int n_row = C::MLP ? r : (tile / p.m_tiles) * TILE_N + r;
        const int n_out = C::MLP ? p.N2 : p.N;
        const int m0 = (tile % p.m_tiles) * BN + q * cmax;
        if (all_good && n_row < n_out) {
          const float e_sig = epi[et], e_bias = epi[256 + et];
          const float* row = recv + r * cmax;          // partial of rank pr at row[pr * TILE_N * cmax]
          const int rstride = TILE_N * cmax;
          // columns in chunks of (at most) 8: the S partials of a chunk are
          // vector loads, added in rank order
          const int cw = cmax < 8 ? cmax : 8;
#pragma unroll 1
          for (int c0 = 0; c0 < cmax && m0 + c0 < p.M; c0 += cw) {
            float v[8];
            const float* src = row + c0;
            if (cw >= 4) {
              const float4 a = *reinterpret_cast<const float4*>(src);
              v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
              if (cw == 8) {
                const float4 b = *reinterpret_cast<const float4*>(src + 4);
                v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
              }
            } else {
              const float2 a = *reinterpret_cast<const float2*>(src);
              v[0] = a.x; v[1] = a.y;
            }
#pragma unroll 1
            for (int pr = 1; pr < S; ++pr) {
              src += rstride;
              if (cw >= 4) {
                const float4 a = *reinterpret_cast<const float4*>(src);
                v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
                if (cw == 8) {
                  const float4 b = *reinterpret_cast<const float4*>(src + 4);
                  v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
                }
              } else {
                const float2 a = *reinterpret_cast<const float2*>(src);
                v[0] += a.x; v[1] += a.y;
              }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int m = m0 + c0 + i;
              if (i < cw && m < p.M) {
                const size_t o = (size_t)m * n_out + n_row;
                if constexpr (!QOUT)
                  p.y[o] = __float2bfloat16_rn(fmaf(v[i], e_sig, e_bias));
                else
                  p.yq[o] = out_code(p, fmaf(v[i], e_sig, e_bias));
              }
            }
          }
        }
      }
    }
  }

  __syncwarp();
  // split-K: every thread of the cluster arrives once (the reducing threads
  // as soon as their receive completed, every other thread when its part is
  // done), so past this barrier no st.async into any CTA of the cluster is
  // still in flight and no sender leaves with one outstanding
  if (p.split > 1) {
    if (!arrived) cluster_arrive_relaxed();
    cluster_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace dq
