// dq_layout.h -- the handle-internal weight layout ("kernel tile order").
//
// dqgemm_create re-lays the canonical weight (nn.Linear [N, K], groups along
// K) into chunks, one per (tile of 128 output channels, stage of 128 k):
//
//   chunk(t, s) at byte offset (t * k_stages + s) * chunk_bytes(fmt)
//
// so that one CTA streaming consecutive stages of a tile reads contiguous
// memory with a single 1-D bulk copy per stage.  Rows n >= N and columns
// k >= K are zero codes with zero scales.
//
// Inside a chunk, row r (0..127) of the tile is dequantized by one thread per
// half-stage h (k 64h..64h+63).  Its bytes sit in 16-byte vectors
//   4-bit formats: vector (h, j in 0..1, r) at ((h*2 + j)*128 + r)*16,
//                  word w of it covers k = 64h + 32j + 8w + [0, 8)
//   FP8 weight-only: vector (h, j in 0..3, r) at ((h*4 + j)*128 + r)*16,
//                  word w of it covers k = 64h + 16j + 4w + [0, 4)
// so a warp (32 consecutive r) reads 512 contiguous bytes per vector.
// Within a 32-bit word the codes of consecutive k are bit-permuted so that
// each bf16x2 operand pair comes out with one shift and one mask (see
// dq_common.cuh for the extraction):
//   INT4 nibbles n0..n7:  n_{2j} at bits 4j..4j+3, n_{2j+1} at 16+4j..16+4j+3
//                         (the same for the unsigned codes of asymmetric INT4)
//   E2M1 (NVFP4/MXFP4) magnitude c = n & 7 and sign s = n >> 3:
//        c0@0  c1@16 s0@14 s1@30 | c2@3 c3@19 s2@12 s3@28 |
//        c4@6  c5@22 s4@15 s5@31 | c6@9 c7@25 s6@13 s7@29
//   E4M3 bytes b0..b3, magnitude m = b & 0x7F, sign s = b >> 7:
//        m0@0 m1@16 s0@15 s1@31 | m2@7 m3@23 s2@14 s3@30
// Scales follow the 8192 packed bytes of a 4-bit chunk:
//   INT4   bf16 s[r] for the group of this stage        (128 x 2 B)
//   INT4 asymmetric  bf16 s[r] as INT4, then the zero point z[r] (128 x 1 B)
//   NVFP4  E4M3 codes of blocks 4h..4h+3 at (h*128 + r)*4 (2 x 128 x 4 B)
//   MXFP4  E8M0 codes of blocks 2h..2h+1 at (h*128 + r)*2 (2 x 128 x 2 B)
// FP8 weight-only chunks hold codes only (the per-channel scale is applied
// in the epilogue).  Static-FP8 chunks are the tensor core's K-major,
// 128-byte-swizzled shared-memory image of the 128 x 128 e4m3 tile:
//   byte (r, k) at r*128 + (((k >> 4) ^ (r & 7)) << 4) + (k & 15).
// FP4 x FP4 (W4A4) chunks cover 256 k per stage: the 128 x 128-byte image of
// the packed E2M1 codes in the same swizzled layout (byte b of a row holds
// k = 2b in its low nibble and k = 2b + 1 in its high nibble), then the block
// scales as tensor-memory words, one per (k-step t of 64, row r) at
// 16384 + (t * 128 + r) * 4:
//   MXFP4 (E8M0 per 32)  byte 0 = block 2t, byte 1 = block 2t + 1, bytes 2-3 zero
//   NVFP4 (E4M3 per 16)  byte j = block 4t + j
#pragma once

#include <stdint.h>

namespace dq {

enum Fmt { FMT_INT4 = 0, FMT_NVFP4 = 1, FMT_MXFP4 = 2, FMT_FP8 = 3, FMT_FP8S = 4,
           FMT_INT4A = 5,   // asymmetric INT4, per-group zero point
           // FP4 x FP4 with dynamic activation quantization (native
           // block-scaled MMA): MXFP4 and NVFP4 weights
           FMT_W4A4MX = 6, FMT_W4A4NV = 7,
           // static FP8 GEMM fed with activations quantized beforehand (same
           // weight chunks as FMT_FP8S; a kernel variant, not a storage format)
           FMT_FP8SQ = 8,
           // the static-FP8 two-layer MLP in one launch (layer 1 in FP8S
           // chunks, layer 2 likewise; a kernel variant)
           FMT_MLP = 9 };

constexpr int TILE_N = 128;      // output channels per tile (MMA M)
constexpr int STAGE_K = 128;     // k per pipeline stage (= one INT4 group)
constexpr int PACKED4_BYTES = TILE_N * STAGE_K / 2;   // 8192
constexpr int W4_STAGE_K = 256;  // k per pipeline stage of the FP4 x FP4 GEMM (128 bytes of codes a row)
constexpr int W4_SF_OFF = TILE_N * W4_STAGE_K / 2;    // 16384: the scale words of a W4A4 chunk

__host__ __device__ constexpr bool is_w4a4(int fmt) { return fmt == FMT_W4A4MX || fmt == FMT_W4A4NV; }

__host__ __device__ constexpr int chunk_bytes(int fmt) {
  return is_w4a4(fmt) ? W4_SF_OFF + 4 * TILE_N * 4
       : fmt == FMT_INT4 ? PACKED4_BYTES + TILE_N * 2
       : fmt == FMT_INT4A ? PACKED4_BYTES + TILE_N * 3
       : fmt == FMT_NVFP4 ? PACKED4_BYTES + TILE_N * 8
       : fmt == FMT_MXFP4 ? PACKED4_BYTES + TILE_N * 4
       : TILE_N * STAGE_K;
}

__host__ __device__ constexpr bool is_4bit(int fmt) {
  return fmt == FMT_INT4 || fmt == FMT_INT4A || fmt == FMT_NVFP4 || fmt == FMT_MXFP4;
}

}  // namespace dq
