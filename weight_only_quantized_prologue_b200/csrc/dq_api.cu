// dq_api.cu -- the C ABI declared in include/dqgemm.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "dq_aux.cuh"
#include "dq_codec.h"
#include "dq_gemm.cuh"
#include "dqgemm.h"

using namespace dq;

struct dqgemm_s {
  int fmt = 0, K = 0, N = 0;
  int k_stages = 0, n_tiles = 0;
  int device = 0, num_sms = 0;
  uint8_t* wchunks = nullptr;       // pre-tiled weight
  size_t wchunk_bytes = 0;
  float* col_scale = nullptr;       // [N] for FP8 formats
  __nv_bfloat16* bias = nullptr;    // [N] or null
  int* status = nullptr;            // status word as the device addresses it
  int* status_host = nullptr;       //   ... and as the host reads it (mapped pinned memory)
  float sigma = 1.f, s_x = 1.f;
  int mx_bias = 126;
  long long weight_bytes = 0;       // canonical packed + scale bytes
  int max_clusters[4][9] = {};      // co-resident clusters per (BN index, cluster size), 0 = unknown
  // FP4 x FP4: the activation workspace (codes, scale words, the NVFP4 amax
  // partials, ticket and g_x), grown on demand and reused by every call
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  unsigned long long timeout_ns = 0;  // limit of the kernels' pipeline waits
  // activation tensor maps already encoded, by (x, M, tile rows, e4m3 input):
  // encoding one costs host time on every call, and layers see the same
  // few activation buffers again and again
  struct MapEntry {
    const void* x = nullptr;
    int M = 0, bn = 0;
    bool xq = false, x3d = false;
    CUtensorMap map;
  };
  static constexpr int kMaps = 8;
  MapEntry maps[kMaps];
  int next_map = 0;
  std::mutex maps_mu;               // run entry points may be called from several threads
};

namespace {

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;   // 2 s

unsigned long long timeout_ns() {
  static unsigned long long t = [] {
    const char* e = std::getenv("DQGEMM_TIMEOUT_MS");
    return e ? (unsigned long long)std::strtoull(e, nullptr, 10) * 1000000ull : kDefaultTimeoutNs;
  }();
  return t;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

// canonical storage sizes of dqgemm.h
// the canonical storage of a W4A4 handle is that of its weight format
int storage_fmt(int fmt) { return fmt == FMT_W4A4MX ? FMT_MXFP4 : fmt == FMT_W4A4NV ? FMT_NVFP4 : fmt; }

size_t packed_bytes(int fmt, int K, int N) {
  fmt = storage_fmt(fmt);
  return is_4bit(fmt) ? (size_t)N * K / 2 : (size_t)N * K;
}
size_t scale_bytes(int fmt, int K, int N) {
  fmt = storage_fmt(fmt);
  switch (fmt) {
    case FMT_INT4: return (size_t)N * (K / 128) * 2;
    case FMT_INT4A: return (size_t)N * (K / 128) * 3;   // bf16 scales, then u8 zero points
    case FMT_NVFP4: return (size_t)N * (K / 16);
    case FMT_MXFP4: return (size_t)N * (K / 32);
    default: return (size_t)N * 4;
  }
}

dqgemm_status check_shape(int fmt, int K, int N) {
  if (fmt < 0 || fmt > FMT_W4A4NV || K <= 0 || N <= 0) return DQ_ERR_INVALID_ARG;
  switch (storage_fmt(fmt)) {
    case FMT_INT4:
    case FMT_INT4A: return K % 128 ? DQ_ERR_INVALID_ARG : DQ_OK;
    case FMT_NVFP4: return (K % 16 || N % 16) ? DQ_ERR_INVALID_ARG : DQ_OK;
    case FMT_MXFP4: return (K % 32 || N % 32) ? DQ_ERR_INVALID_ARG : DQ_OK;
    default: return K % 16 ? DQ_ERR_INVALID_ARG : DQ_OK;
  }
}

// ---------------------------------------------------------------------------
// host re-layout: canonical -> kernel tile order (see dq_layout.h)
// ---------------------------------------------------------------------------
void relayout(int fmt, int K, int N, int KS, int NT, const std::vector<uint8_t>& packed,
              const std::vector<uint8_t>& scales, std::vector<uint8_t>& out) {
  const int CH = chunk_bytes(fmt);
  out.assign((size_t)NT * KS * CH, 0);
  auto nib = [&](int n, int k) -> uint32_t {
    if (n >= N || k >= K) return 0;
    return (packed[(size_t)n * (K / 2) + k / 2] >> ((k & 1) * 4)) & 0xFu;
  };
  auto code8 = [&](int n, int k) -> uint32_t {
    if (n >= N || k >= K) return 0;
    return packed[(size_t)n * K + k];
  };
  auto put32 = [](uint8_t* p, uint32_t v) { std::memcpy(p, &v, 4); };
  for (int t = 0; t < NT; ++t) {
    for (int s = 0; s < KS; ++s) {
      uint8_t* ch = out.data() + ((size_t)t * KS + s) * CH;
      for (int r = 0; r < TILE_N; ++r) {
        const int n = t * TILE_N + r;
        if (is_w4a4(fmt)) {
          // swizzled K-major image of the packed codes (256 k = 128 bytes a
          // row), then the scale words [k-step t4][row]
          for (int b = 0; b < 128; ++b) {
            const int k = s * W4_STAGE_K + 2 * b;
            ch[r * 128 + (((b >> 4) ^ (r & 7)) << 4) + (b & 15)] = (uint8_t)(nib(n, k) | (nib(n, k + 1) << 4));
          }
          const bool mx = fmt == FMT_W4A4MX;
          const int vs = mx ? 32 : 16, blocks = K / vs, per_step = 64 / vs;
          for (int t4 = 0; t4 < 4; ++t4) {
            uint32_t word = 0;
            for (int j = 0; j < per_step; ++j) {
              const int blk = (s * W4_STAGE_K + t4 * 64) / vs + j;
              if (n < N && blk < blocks) word |= (uint32_t)scales[(size_t)n * blocks + blk] << (8 * j);
            }
            put32(ch + W4_SF_OFF + (t4 * TILE_N + r) * 4, word);
          }
        } else if (is_4bit(fmt)) {
          for (int h = 0; h < 2; ++h)
            for (int j = 0; j < 2; ++j)
              for (int w = 0; w < 4; ++w) {
                const int k0 = s * STAGE_K + 64 * h + 32 * j + 8 * w;
                uint32_t c[8], word = 0;
                for (int i = 0; i < 8; ++i) c[i] = nib(n, k0 + i);
                if (fmt == FMT_INT4 || fmt == FMT_INT4A) {
                  for (int jj = 0; jj < 4; ++jj) word |= (c[2 * jj] << (4 * jj)) | (c[2 * jj + 1] << (16 + 4 * jj));
                } else {
                  uint32_t m[8], sg[8];
                  for (int i = 0; i < 8; ++i) { m[i] = c[i] & 7u; sg[i] = c[i] >> 3; }
                  word = m[0] | (m[1] << 16) | (sg[0] << 14) | (sg[1] << 30) |
                         (m[2] << 3) | (m[3] << 19) | (sg[2] << 12) | (sg[3] << 28) |
                         (m[4] << 6) | (m[5] << 22) | (sg[4] << 15) | (sg[5] << 31) |
                         (m[6] << 9) | (m[7] << 25) | (sg[6] << 13) | (sg[7] << 29);
                }
                put32(ch + ((h * 2 + j) * TILE_N + r) * 16 + w * 4, word);
              }
          uint8_t* sc = ch + PACKED4_BYTES;
          if (fmt == FMT_INT4 || fmt == FMT_INT4A) {
            const int groups = K / 128;
            uint16_t v = 0;
            if (n < N && s < groups) std::memcpy(&v, &scales[((size_t)n * groups + s) * 2], 2);
            std::memcpy(sc + r * 2, &v, 2);
            if (fmt == FMT_INT4A)
              sc[TILE_N * 2 + r] = (n < N && s < groups) ? scales[(size_t)2 * N * groups + (size_t)n * groups + s] : 0;
          } else if (fmt == FMT_NVFP4) {
            const int blocks = K / 16;
            for (int h = 0; h < 2; ++h)
              for (int b = 0; b < 4; ++b) {
                const int blk = s * 8 + 4 * h + b;
                sc[(h * TILE_N + r) * 4 + b] = (n < N && blk < blocks) ? scales[(size_t)n * blocks + blk] : 0;
              }
          } else {
            const int blocks = K / 32;
            for (int h = 0; h < 2; ++h)
              for (int b = 0; b < 2; ++b) {
                const int blk = s * 4 + 2 * h + b;
                sc[(h * TILE_N + r) * 2 + b] = (n < N && blk < blocks) ? scales[(size_t)n * blocks + blk] : 0;
              }
          }
        } else if (fmt == FMT_FP8) {
          for (int h = 0; h < 2; ++h)
            for (int j = 0; j < 4; ++j)
              for (int w = 0; w < 4; ++w) {
                const int k0 = s * STAGE_K + 64 * h + 16 * j + 4 * w;
                uint32_t b[4], m[4], sg[4];
                for (int i = 0; i < 4; ++i) { b[i] = code8(n, k0 + i); m[i] = b[i] & 0x7Fu; sg[i] = b[i] >> 7; }
                const uint32_t word = m[0] | (m[1] << 16) | (sg[0] << 15) | (sg[1] << 31) |
                                      (m[2] << 7) | (m[3] << 23) | (sg[2] << 14) | (sg[3] << 30);
                put32(ch + ((h * 4 + j) * TILE_N + r) * 16 + w * 4, word);
              }
        } else {  // static FP8: swizzled K-major shared-memory image
          for (int kl = 0; kl < STAGE_K; ++kl)
            ch[r * 128 + (((kl >> 4) ^ (r & 7)) << 4) + (kl & 15)] = (uint8_t)code8(n, s * STAGE_K + kl);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// tensor map for the bf16 activation x [M, K]: boxes of 64 k x BN rows, 128B swizzle
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// With K a multiple of 64 the map is 3-D {64, M, K/64} (the k-blocks are
// 128 bytes apart) so one box {64, bn, 2} brings a whole 128-k stage.
bool make_x_map(CUtensorMap* map, const void* x, int M, int K, int bn, bool* is3d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  *is3d = (K % 64) == 0;
  if (*is3d) {
    const cuuint64_t dims[3] = {64, (cuuint64_t)M, (cuuint64_t)(K / 64)};
    const cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)bn, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)bn};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// e4m3 activations [M, K] (u8, K % 16 == 0): box of 128 k x bn rows, the
// tensor core's 128-byte-swizzled K-major image
bool make_q_map(CUtensorMap* map, const void* q, int M, int K, int bn) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  const cuuint64_t strides[1] = {(cuuint64_t)K};
  const cuuint32_t box[2] = {128, (cuuint32_t)bn};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// launch dispatch
// ---------------------------------------------------------------------------
bool pdl_enabled() {
  static bool on = [] {
    const char* e = std::getenv("DQGEMM_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <int FMT, int BN>
struct GemmLauncher {
  using C = GemmCfg<FMT, BN>;
  static cudaError_t set_attr() {
    cudaError_t e = set_attr_q<false>();
    if constexpr (FMT != FMT_MLP && !is_w4a4(FMT)) {
      if (e == cudaSuccess) e = set_attr_q<true>();
    }
    return e;
  }
  template <bool QOUT>
  static cudaError_t set_attr_q() {
    cudaError_t e =
        cudaFuncSetAttribute(dq_gemm_kernel<FMT, BN, QOUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    // every GEMM kernel asks for the same (largest) shared-memory carveout, so
    // back-to-back calls never reconfigure the SM's L1 / shared split
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(dq_gemm_kernel<FMT, BN, QOUT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    return e;
  }
  static void config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attrs, int grid, int split, cudaStream_t st) {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    int na = 0;
    if (pdl_enabled()) {
      attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attrs[na].val.programmaticStreamSerializationAllowed = 1;
      ++na;
    }
    if (split > 1) {
      attrs[na].id = cudaLaunchAttributeClusterDimension;
      attrs[na].val.clusterDim.x = split;
      attrs[na].val.clusterDim.y = 1;
      attrs[na].val.clusterDim.z = 1;
      ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
  }
  static cudaError_t launch(const CUtensorMap& tm, const GemmParams& p, int grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attrs[2];
    config(cfg, attrs, grid, p.split, st);
    if constexpr (FMT == FMT_MLP || is_w4a4(FMT)) {
      return cudaLaunchKernelEx(&cfg, dq_gemm_kernel<FMT, BN, false>, tm, p);
    } else {
      return p.yq ? cudaLaunchKernelEx(&cfg, dq_gemm_kernel<FMT, BN, true>, tm, p)
                  : cudaLaunchKernelEx(&cfg, dq_gemm_kernel<FMT, BN, false>, tm, p);
    }
  }
  static int max_active_clusters(int split) {
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attrs[2];
    config(cfg, attrs, split, split, nullptr);
    int n = 0;
    if (split > 1) {
      if (cudaOccupancyMaxActiveClusters(&n, dq_gemm_kernel<FMT, BN, false>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
    }
    return n;
  }
};

template <int FMT>
int stages_for(int bn) {
  switch (bn) {
    case 16: return GemmCfg<FMT, is_w4a4(FMT) ? 32 : 16>::STAGES;
    case 32: return GemmCfg<FMT, 32>::STAGES;
    case 64: return GemmCfg<FMT, 64>::STAGES;
    case 128: return GemmCfg<FMT, 128>::STAGES;
    default:
      if constexpr (FMT == FMT_FP8S) return GemmCfg<FMT, 128>::STAGES;
      else return GemmCfg<FMT, 256>::STAGES;
  }
}
template <int FMT>
int xstages_for(int bn) {
  switch (bn) {
    case 16: return GemmCfg<FMT, is_w4a4(FMT) ? 32 : 16>::XST;
    case 32: return GemmCfg<FMT, 32>::XST;
    case 64: return GemmCfg<FMT, 64>::XST;
    case 128: return GemmCfg<FMT, 128>::XST;
    default:
      if constexpr (FMT == FMT_FP8S) return GemmCfg<FMT, 128>::XST;
      else return GemmCfg<FMT, 256>::XST;
  }
}
template <int FMT>
int smem_for(int bn) {
  switch (bn) {
    case 16: return GemmCfg<FMT, is_w4a4(FMT) ? 32 : 16>::SMEM;
    case 32: return GemmCfg<FMT, 32>::SMEM;
    case 64: return GemmCfg<FMT, 64>::SMEM;
    case 128: return GemmCfg<FMT, 128>::SMEM;
    default:
      if constexpr (FMT == FMT_FP8S) return GemmCfg<FMT, 128>::SMEM;
      else return GemmCfg<FMT, 256>::SMEM;
  }
}
template <int FMT>
cudaError_t set_attrs() {
  // (W4A4 x tiles hold 32 rows or more: there is no 16-row instance)
  cudaError_t e = GemmLauncher<FMT, is_w4a4(FMT) ? 32 : 16>::set_attr();
  if (e == cudaSuccess) e = GemmLauncher<FMT, 32>::set_attr();
  if (e == cudaSuccess) e = GemmLauncher<FMT, 64>::set_attr();
  if (e == cudaSuccess) e = GemmLauncher<FMT, 128>::set_attr();
  if constexpr (FMT != FMT_FP8S) {
    if (e == cudaSuccess) e = GemmLauncher<FMT, 256>::set_attr();
  }
  return e;
}
template <int FMT>
cudaError_t launch_fmt(int bn, const CUtensorMap& tm, const GemmParams& p, int grid, cudaStream_t st) {
  switch (bn) {
    case 16:
      if constexpr (is_w4a4(FMT)) return cudaErrorInvalidValue;   // never planned
      else return GemmLauncher<FMT, 16>::launch(tm, p, grid, st);
    case 32: return GemmLauncher<FMT, 32>::launch(tm, p, grid, st);
    case 64: return GemmLauncher<FMT, 64>::launch(tm, p, grid, st);
    case 128: return GemmLauncher<FMT, 128>::launch(tm, p, grid, st);
    default:
      if constexpr (FMT != FMT_FP8S) return GemmLauncher<FMT, 256>::launch(tm, p, grid, st);
      return cudaErrorInvalidValue;   // never planned: the fused static-FP8 tile holds at most 128 x rows
  }
}

template <int FMT>
int max_clusters_fmt(int bn, int split) {
  switch (bn) {
    case 16: return GemmLauncher<FMT, is_w4a4(FMT) ? 32 : 16>::max_active_clusters(split);
    case 32: return GemmLauncher<FMT, 32>::max_active_clusters(split);
    case 64: return GemmLauncher<FMT, 64>::max_active_clusters(split);
    default: return GemmLauncher<FMT, 128>::max_active_clusters(split);
  }
}

#define DQ_FMT_SWITCH(fmt, CALL)                  \
  switch (fmt) {                                  \
    case FMT_INT4: { constexpr int F = FMT_INT4; CALL; } break;   \
    case FMT_INT4A: { constexpr int F = FMT_INT4A; CALL; } break; \
    case FMT_NVFP4: { constexpr int F = FMT_NVFP4; CALL; } break; \
    case FMT_MXFP4: { constexpr int F = FMT_MXFP4; CALL; } break; \
    case FMT_FP8: { constexpr int F = FMT_FP8; CALL; } break;     \
    case FMT_W4A4MX: { constexpr int F = FMT_W4A4MX; CALL; } break; \
    case FMT_W4A4NV: { constexpr int F = FMT_W4A4NV; CALL; } break; \
    default: { constexpr int F = FMT_FP8S; CALL; } break;         \
  }

int bn_index(int bn) { return bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : 3; }

// How many clusters of `split` CTAs can be resident at once (cached per handle).
int cluster_capacity(dqgemm_s* h, int bn, int split) {
  int& c = h->max_clusters[bn_index(bn)][split];
  if (c == 0) {
    int n = 0;
    DQ_FMT_SWITCH(h->fmt, n = max_clusters_fmt<F>(bn, split));
    c = n > 0 ? n : -1;
  }
  return c;
}

// Tiles of 128 output channels x bn activation rows.  With at least one tile
// per SM, each CTA computes whole tiles (persistent loop).  With fewer tiles
// than SMs, the K range of each tile is split over the S CTAs of a cluster,
// S the largest power of two (<= 8, <= k_stages) whose T * S CTAs are all
// resident.
// From 129 rows on, an x tile of 256 rows halves the weight dequantization
// per FLOP (one N = 256 MMA per k-step); it is taken when it keeps at least
// half the SMs busy and its waves of tiles cost no more than 5/4 of the
// 128-row tiling's (the 128-row tile is bound by the unpack, about 5/4 of
// its MMA time).  The fused static-FP8 kernel stays at 128 rows.
int pick_bn(const dqgemm_s* h, int M, bool xq) {
  int bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  if (is_w4a4(h->fmt) && bn < 32) bn = 32;   // one block-scale column per 32 x rows
  // From 16 to 64 rows, when the output tiles fill more than half the SMs
  // (so the K range cannot be split) and fit one wave, every CTA streams a
  // whole tile alone on its SM: the 128-row tile's larger rings serve it
  // better than the skinny tiles' two-CTAs-per-SM budget (measured at
  // 4096 x 14336: INT4 24.0 against 29.6 us, FP8-WO 21.7 against 27.0).
  // Not below 16 rows, where x boxes of 128 rows with 8 or fewer rows in the
  // tensor ran twice as slow (W4A4 is exempt: its quantized x is padded to
  // the tile), and not for fused static FP8, whose 128-row tile keeps few
  // x slots (54 against 23 us).
  if (bn <= 64 && (M >= 16 || is_w4a4(h->fmt)) && !(h->fmt == FMT_FP8S && !xq) &&
      2 * (long long)h->n_tiles > h->num_sms && h->n_tiles <= h->num_sms)
    bn = 128;
  if (M > 128 && !(h->fmt == FMT_FP8S && !xq)) {
    const long long sms = h->num_sms, nt = h->n_tiles;
    const long long t256 = (M + 255) / 256 * nt, t128 = (M + 127) / 128 * nt;
    const long long w256 = (t256 + sms - 1) / sms, w128 = (t128 + sms - 1) / sms;
    if (2 * t256 >= sms && w256 * 256 * 4 <= w128 * 128 * 5) bn = 256;
  }
  return bn;
}

// The FP4 x FP4 activation workspace for M rows in x tiles of bn rows: the
// NVFP4 amax partials, the amax ticket and g_x at fixed offsets (the ticket
// is zeroed once, when the workspace is allocated, and left at zero by every
// call), then codes [rows][kp / 2] and scale words [m_tiles][k_stages][4][bn].
struct W4Workspace {
  static constexpr size_t partials = 0, ticket = (size_t)kActAmaxBlocks * 4, gx = ticket + 16, codes = 8192;
  int rows = 0, kp = 0;
  size_t sfw = 0, total = 0;
};
W4Workspace w4a4_workspace(const dqgemm_s* h, int M, int bn) {
  W4Workspace w;
  w.rows = (M + bn - 1) / bn * bn;
  w.kp = h->k_stages * W4_STAGE_K;
  w.sfw = W4Workspace::codes + (size_t)w.rows * (w.kp / 2);
  w.total = w.sfw + (size_t)w.rows * h->k_stages * 16;
  return w;
}
static_assert(W4Workspace::gx + 16 <= W4Workspace::codes, "workspace header");

void fill_plan(dqgemm_s* h, int M, dqgemm_plan* pl, bool xq = false) {
  std::memset(pl, 0, sizeof(*pl));
  const int bn = pick_bn(h, M, xq);
  pl->bn = bn;
  pl->m_tiles = (M + bn - 1) / bn;
  pl->n_tiles = h->n_tiles;
  pl->k_stages = h->k_stages;
  const long long T = (long long)pl->m_tiles * pl->n_tiles;
  // CTAs per SM the split may assume (skinny tiles fit two per SM)
  static const int occ = [] {
    const char* e = std::getenv("DQGEMM_CTAS_PER_SM");
    const int v = e ? std::atoi(e) : 1;
    return v >= 2 ? 2 : 1;
  }();
  const int slots = h->num_sms * (bn <= 64 ? occ : 1);
  static const int force_split = [] {
    const char* e = std::getenv("DQGEMM_SPLIT");
    return e ? std::atoi(e) : 0;
  }();
  // the split is a power of two (<= 8, so it divides every bn): each rank
  // then owns bn / S whole columns of the tile in the reduction
  int split = 1;
  if (bn > 128) {
    // whole tiles only
  } else if (force_split >= 1 && force_split <= 8) {
    while (split * 2 <= std::min(force_split, h->k_stages)) split *= 2;
    if (split > 1 && cluster_capacity(h, bn, split) < T) split = 1;
  } else if (T < slots) {
    for (int s = 8; s >= 2; s /= 2) {
      if (s > h->k_stages || T * s > slots) continue;
      const int cap = cluster_capacity(h, bn, s);
      if (cap > 0 && cap >= T) { split = s; break; }
    }
  }
  pl->max_segments = split;
  pl->grid = split > 1 ? (int)(T * split) : (int)std::min<long long>(T, h->num_sms);
  int st = 0, sm = 0, xs = 0;
  if (xq) {
    st = stages_for<FMT_FP8SQ>(bn);
    sm = smem_for<FMT_FP8SQ>(bn);
    xs = xstages_for<FMT_FP8SQ>(bn);
  } else {
    DQ_FMT_SWITCH(h->fmt, st = stages_for<F>(bn); sm = smem_for<F>(bn); xs = xstages_for<F>(bn));
  }
  pl->stages = st;
  pl->smem_bytes = sm;
  pl->workspace_bytes = is_w4a4(h->fmt) ? (long long)w4a4_workspace(h, M, bn).total : 0;
  pl->weight_bytes = h->weight_bytes;
  pl->x_stages = xs;
  // the split gives rank q the stages [q*KS/S, (q+1)*KS/S); whole tiles give
  // a CTA every ceil(T / grid)-th tile
  pl->max_cta_stages = split > 1 ? (h->k_stages + split - 1) / split
                                 : (int)((T + pl->grid - 1) / pl->grid) * h->k_stages;
}

// The activation tensor map for (x, M, tile rows, e4m3 input), from the
// handle's cache or freshly encoded.  A map encodes only those and K, so a
// cached one for the same key is the map this call would encode.
bool x_map(dqgemm_s* h, const void* x, int M, int bn, bool xq, CUtensorMap* tm, bool* x3d, int q_row_bytes = 0) {
  std::lock_guard<std::mutex> lock(h->maps_mu);
  for (const auto& e : h->maps) {
    if (e.x == x && e.M == M && e.bn == bn && e.xq == xq) {
      *tm = e.map;
      *x3d = e.x3d;
      return true;
    }
  }
  if (xq ? !make_q_map(tm, x, M, q_row_bytes ? q_row_bytes : h->K, bn) : !make_x_map(tm, x, M, h->K, bn, x3d))
    return false;
  auto& e = h->maps[h->next_map];
  h->next_map = (h->next_map + 1) % dqgemm_s::kMaps;
  e.x = x;
  e.M = M;
  e.bn = bn;
  e.xq = xq;
  e.x3d = *x3d;
  e.map = *tm;
  return true;
}

dqgemm_status cuda_err(cudaError_t e) { return e == cudaSuccess ? DQ_OK : DQ_ERR_CUDA; }

// f32(1 / s), correctly rounded (an IEEE fp32 division on the host): the
// reciprocal the kernels' static-FP8 quantizers multiply by
float recip_rn(float s) {
  volatile float one = 1.f;
  volatile float r = one / s;
  return r;
}

// a small kernel in the programmatic-dependent-launch chain of the GEMMs
// (its first instruction waits for the previous grid)
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kern)(KArgs...), int grid, int block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.stream = st;
  cudaLaunchAttribute a[1];
  int na = 0;
  if (pdl_enabled()) {
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    na = 1;
  }
  cfg.attrs = a;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

int act_amax_grid(long long count) {
  return (int)std::max<long long>(1, std::min<long long>((count / 8 + 255) / 256, kActAmaxBlocks));
}

// Codes the canonical storage may hold (the packers produce nothing else):
//   FP8 formats  no NaN weight code (0x7F / 0xFF)
//   NVFP4        block scales are non-negative finite E4M3 (no sign bit, no 0x7F)
//   MXFP4        no NaN exponent (0xFF); and, because the prologue's bf16
//                operand e2m1 * 2^(e - 127 - J) (J = max(0, emax - 128),
//                undone in the epilogue) must not fall below the smallest
//                bf16 subnormal, every block with a nonzero element has an
//                exponent code >= emax - 133 when emax > 128
//                (DQ_ERR_UNSUPPORTED otherwise: the span of 2^133 between a
//                handle's block scales is past what it represents exactly)
dqgemm_status check_codes(int fmt, int K, int N, const std::vector<uint8_t>& hp, const std::vector<uint8_t>& hs) {
  if (fmt == FMT_FP8 || fmt == FMT_FP8S) {
    for (uint8_t c : hp)
      if ((c & 0x7F) == 0x7F) return DQ_ERR_INVALID_ARG;
  } else if (fmt == FMT_NVFP4 || fmt == FMT_W4A4NV) {
    for (uint8_t c : hs)
      if (c >= 0x7F) return DQ_ERR_INVALID_ARG;
  } else if (fmt == FMT_W4A4MX) {
    // the tensor core takes every E8M0 exponent but the NaN code
    for (uint8_t c : hs)
      if (c == 255) return DQ_ERR_INVALID_ARG;
  } else if (fmt == FMT_MXFP4) {
    int cmax = 0;
    for (uint8_t c : hs) {
      if (c == 255) return DQ_ERR_INVALID_ARG;
      cmax = std::max<int>(cmax, c);
    }
    if (cmax > 128) {
      const int blocks = K / 32;
      for (int n = 0; n < N; ++n)
        for (int b = 0; b < blocks; ++b) {
          if (hs[(size_t)n * blocks + b] >= cmax - 133) continue;
          const uint8_t* e = &hp[(size_t)n * (K / 2) + (size_t)b * 16];
          for (int i = 0; i < 16; ++i)
            if (e[i] & 0x77) return DQ_ERR_UNSUPPORTED;   // a nonzero magnitude in either nibble
        }
    }
  }
  return DQ_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* dqgemm_status_string(dqgemm_status s) {
  switch (s) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_INVALID_ARG: return "DQ_ERR_INVALID_ARG";
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED";
    case DQ_ERR_ALIGNMENT: return "DQ_ERR_ALIGNMENT";
    case DQ_ERR_ALLOC: return "DQ_ERR_ALLOC";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA";
    case DQ_ERR_TIMEOUT: return "DQ_ERR_TIMEOUT";
  }
  return "DQ_ERR_UNKNOWN";
}

dqgemm_status dqgemm_destroy(dqgemm_handle h) {
  if (!h) return DQ_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  cudaFree(h->wchunks);
  cudaFree(h->ws);
  cudaFree(h->col_scale);
  cudaFree(h->bias);
  if (h->status_host) cudaFreeHost(h->status_host);
  delete h;
  return DQ_OK;
}

dqgemm_status dqgemm_create(dqgemm_handle* out, dqgemm_format fmt_, int K, int N, const void* packed_w,
                            const void* scales, float global_scale, const void* bias) {
  if (!out) return DQ_ERR_INVALID_ARG;
  *out = nullptr;
  const int fmt = (int)fmt_;
  dqgemm_status st = check_shape(fmt, K, N);
  if (st != DQ_OK) return st;
  if (!packed_w || !scales) return DQ_ERR_INVALID_ARG;
  if (!aligned16(packed_w) || !aligned16(scales) || (bias && !aligned16(bias))) return DQ_ERR_ALIGNMENT;
  if (!is_device_ptr(packed_w) || !is_device_ptr(scales) || (bias && !is_device_ptr(bias)))
    return DQ_ERR_INVALID_ARG;
  if ((fmt == FMT_NVFP4 || fmt == FMT_W4A4NV || fmt == FMT_FP8S) && !(std::isfinite(global_scale) && global_scale > 0.f))
    return DQ_ERR_INVALID_ARG;

  std::vector<uint8_t> hp(packed_bytes(fmt, K, N)), hs(scale_bytes(fmt, K, N));
  if (cudaMemcpy(hp.data(), packed_w, hp.size(), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(hs.data(), scales, hs.size(), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DQ_ERR_CUDA;
  st = check_codes(fmt, K, N, hp, hs);
  if (st != DQ_OK) return st;

  dqgemm_s* h = new dqgemm_s();
  h->fmt = fmt;
  h->K = K;
  h->N = N;
  const int stage_k = is_w4a4(fmt) ? W4_STAGE_K : STAGE_K;
  h->k_stages = (K + stage_k - 1) / stage_k;
  h->n_tiles = (N + TILE_N - 1) / TILE_N;
  h->weight_bytes = (long long)(hp.size() + hs.size());
  h->timeout_ns = timeout_ns();
  cudaGetDevice(&h->device);
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);

  // epilogue factors
  if (fmt == FMT_NVFP4) {
    h->sigma = global_scale * 128.f;   // operand carries dec(sb) * 2^-7
  } else if (fmt == FMT_MXFP4) {
    int cmax = 0;
    for (uint8_t c : hs) cmax = std::max<int>(cmax, c);
    const int J = std::max(0, cmax - 128);
    h->mx_bias = 126 - J;
    h->sigma = std::ldexp(1.f, J);
  } else if (fmt == FMT_FP8S) {
    h->sigma = global_scale;
    h->s_x = global_scale;
  } else if (fmt == FMT_W4A4NV) {
    h->sigma = global_scale;           // g_w; the call's g_x is applied on the device
  }

  std::vector<uint8_t> chunks;
  relayout(fmt, K, N, h->k_stages, h->n_tiles, hp, hs, chunks);
  h->wchunk_bytes = chunks.size();

  cudaError_t e = cudaMalloc(&h->wchunks, chunks.size());
  // the status word lives in mapped pinned host memory: kernels store to it,
  // the host reads it without synchronizing the device
  if (e == cudaSuccess) e = cudaHostAlloc(&h->status_host, sizeof(int), cudaHostAllocMapped | cudaHostAllocPortable);
  if (e == cudaSuccess) {
    *h->status_host = 0;
    e = cudaHostGetDevicePointer(reinterpret_cast<void**>(&h->status), h->status_host, 0);
  }
  if (e == cudaSuccess && (fmt == FMT_FP8 || fmt == FMT_FP8S)) e = cudaMalloc(&h->col_scale, (size_t)N * 4);
  if (e == cudaSuccess && bias) e = cudaMalloc(&h->bias, (size_t)N * 2);
  if (e != cudaSuccess) { dqgemm_destroy(h); return DQ_ERR_ALLOC; }
  e = cudaMemcpy(h->wchunks, chunks.data(), chunks.size(), cudaMemcpyHostToDevice);
  if (e == cudaSuccess && h->col_scale) e = cudaMemcpy(h->col_scale, hs.data(), (size_t)N * 4, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && h->bias) e = cudaMemcpy(h->bias, bias, (size_t)N * 2, cudaMemcpyDeviceToDevice);
  if (e == cudaSuccess) { DQ_FMT_SWITCH(fmt, e = set_attrs<F>()); }
  if (e == cudaSuccess && fmt == FMT_FP8S) e = set_attrs<FMT_FP8SQ>();
  if (e == cudaSuccess && fmt == FMT_FP8S) e = GemmLauncher<FMT_MLP, 16>::set_attr();
  if (e == cudaSuccess && fmt == FMT_FP8S) e = GemmLauncher<FMT_MLP, 32>::set_attr();
  if (e == cudaSuccess && fmt == FMT_FP8S) e = GemmLauncher<FMT_MLP, 64>::set_attr();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) { dqgemm_destroy(h); return DQ_ERR_CUDA; }
  *out = h;
  return DQ_OK;
}

dqgemm_status dqgemm_set_wait_limit(dqgemm_handle h, long long timeout_ns_) {
  if (!h || timeout_ns_ < 0) return DQ_ERR_INVALID_ARG;
  h->timeout_ns = timeout_ns_ == 0 ? timeout_ns() : (unsigned long long)timeout_ns_;
  return DQ_OK;
}

dqgemm_status dqgemm_get_plan(dqgemm_handle h, int M, dqgemm_plan* plan) {
  if (!h || !plan || M < 1) return DQ_ERR_INVALID_ARG;
  fill_plan(h, M, plan);
  return DQ_OK;
}

// FP4 x FP4: quantize x into the handle's workspace (NVFP4: its amax first),
// then the block-scaled GEMM on those codes; three or two launches chained by
// programmatic dependent launch.
static dqgemm_status run_w4a4(dqgemm_handle h, const void* x, int M, void* y, void* stream) {
  dqgemm_plan pl;
  fill_plan(h, M, &pl);
  const W4Workspace w = w4a4_workspace(h, M, pl.bn);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  {
    std::lock_guard<std::mutex> lock(h->maps_mu);
    if (h->ws_bytes < w.total) {
      // grow: calls already launched may still read the old workspace
      cudaError_t e = cudaDeviceSynchronize();
      cudaFree(h->ws);
      h->ws = nullptr;
      h->ws_bytes = 0;
      if (e != cudaSuccess) return DQ_ERR_CUDA;
      if (cudaMalloc(&h->ws, w.total) != cudaSuccess) {
        h->ws = nullptr;
        return DQ_ERR_ALLOC;
      }
      if (cudaMemset(h->ws, 0, w.total) != cudaSuccess) return DQ_ERR_CUDA;
      h->ws_bytes = w.total;
    }
  }
  uint8_t* codes = h->ws + W4Workspace::codes;
  uint32_t* sfw = reinterpret_cast<uint32_t*>(h->ws + w.sfw);
  float* gx = reinterpret_cast<float*>(h->ws + W4Workspace::gx);
  const bool mx = h->fmt == FMT_W4A4MX;
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  cudaError_t e = cudaSuccess;
  if (!mx) {
    const long long count = (long long)M * h->K;
    e = launch_chained(act_amax_kernel, act_amax_grid(count), 256, s, xb, count,
                       reinterpret_cast<float*>(h->ws + W4Workspace::partials),
                       reinterpret_cast<unsigned int*>(h->ws + W4Workspace::ticket), gx);
  }
  if (e == cudaSuccess) {
    const long long threads = (long long)w.rows * (w.kp / 64);
    const int grid = (int)std::min<long long>((threads + 255) / 256, 148 * 8);
    e = mx ? launch_chained(w4a4_act_quant_kernel<true>, grid, 256, s, xb, M, h->K, w.rows, w.kp, pl.bn,
                            (const float*)gx, codes, sfw, (uint8_t*)nullptr)
           : launch_chained(w4a4_act_quant_kernel<false>, grid, 256, s, xb, M, h->K, w.rows, w.kp, pl.bn,
                            (const float*)gx, codes, sfw, (uint8_t*)nullptr);
  }
  if (e != cudaSuccess) return DQ_ERR_CUDA;
  CUtensorMap tm;
  bool x3d = false;
  if (!x_map(h, codes, w.rows, pl.bn, true, &tm, &x3d, w.kp / 2)) return DQ_ERR_CUDA;
  GemmParams p{};
  p.wchunks = h->wchunks;
  p.bias = h->bias;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.status = h->status;
  p.sigma = h->sigma;
  p.s_x = 1.f;
  p.s_out = 1.f;
  p.r_x = 1.f;
  p.r_out = 1.f;
  p.M = M;
  p.N = h->N;
  p.k_stages = h->k_stages;
  p.m_tiles = pl.m_tiles;
  p.tiles = pl.m_tiles * pl.n_tiles;
  p.split = pl.max_segments;
  p.timeout_ns = h->timeout_ns;
  p.drain_ns = std::max(timeout_ns(), kDefaultTimeoutNs);
  p.xsf = sfw;
  p.gx = mx ? nullptr : gx;
  DQ_FMT_SWITCH(h->fmt, e = launch_fmt<F>(pl.bn, tm, p, pl.grid, s));
  return cuda_err(e);
}

static dqgemm_status run_gemm(dqgemm_handle h, const void* x, bool xq, int M, void* y, bool yq, float s_out,
                              void* stream) {
  if (!h || !x || !y || M < 1) return DQ_ERR_INVALID_ARG;
  if (is_w4a4(h->fmt)) {
    if (xq || yq) return DQ_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(y)) return DQ_ERR_ALIGNMENT;
    return run_w4a4(h, x, M, y, stream);
  }
  if (yq && !(std::isfinite(s_out) && s_out > 0.f)) return DQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return DQ_ERR_ALIGNMENT;
  dqgemm_plan pl;
  fill_plan(h, M, &pl, xq);
  CUtensorMap tm;
  bool x3d = false;
  if (!x_map(h, x, M, pl.bn, xq, &tm, &x3d)) return DQ_ERR_CUDA;
  GemmParams p{};
  p.wchunks = h->wchunks;
  p.col_scale = h->col_scale;
  p.bias = h->bias;
  p.y = yq ? nullptr : static_cast<__nv_bfloat16*>(y);
  p.yq = yq ? static_cast<uint8_t*>(y) : nullptr;
  p.s_out = yq ? s_out : 1.f;
  p.r_out = recip_rn(p.s_out);
  p.status = h->status;
  p.sigma = h->sigma;
  p.s_x = h->s_x;
  p.r_x = recip_rn(p.s_x);
  p.mx_bias = h->mx_bias;
  p.M = M;
  p.N = h->N;
  p.k_stages = h->k_stages;
  p.m_tiles = pl.m_tiles;
  p.tiles = pl.m_tiles * pl.n_tiles;
  p.split = pl.max_segments;
  p.x3d = x3d ? 1 : 0;
  p.timeout_ns = h->timeout_ns;
  p.drain_ns = std::max(timeout_ns(), kDefaultTimeoutNs);
  cudaError_t e = cudaSuccess;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (xq) {
    e = launch_fmt<FMT_FP8SQ>(pl.bn, tm, p, pl.grid, s);
  } else {
    DQ_FMT_SWITCH(h->fmt, e = launch_fmt<F>(pl.bn, tm, p, pl.grid, s));
  }
  return cuda_err(e);
}

dqgemm_status dqgemm_run(dqgemm_handle h, const void* x, int M, void* y, void* stream) {
  return run_gemm(h, x, false, M, y, false, 1.f, stream);
}

dqgemm_status dqgemm_run_fp8_static_quantized(dqgemm_handle h, const void* q, int M, void* y, void* stream) {
  if (!h) return DQ_ERR_INVALID_ARG;
  if (h->fmt != FMT_FP8S) return DQ_ERR_UNSUPPORTED;
  return run_gemm(h, q, true, M, y, false, 1.f, stream);
}

dqgemm_status dqgemm_run_quantized_out(dqgemm_handle h, const void* x, int M, void* q_out, float s_out,
                                       void* stream) {
  return run_gemm(h, x, false, M, q_out, true, s_out, stream);
}

dqgemm_status dqgemm_run_fp8_static_quantized_out(dqgemm_handle h, const void* q, int M, void* q_out,
                                                  float s_out, void* stream) {
  if (!h) return DQ_ERR_INVALID_ARG;
  if (h->fmt != FMT_FP8S) return DQ_ERR_UNSUPPORTED;
  return run_gemm(h, q, true, M, q_out, true, s_out, stream);
}

dqgemm_status dqgemm_run_static_mlp(dqgemm_handle l1, dqgemm_handle l2, const void* x, int M, void* h_out, void* y,
                                    void* stream) {
  if (!l1 || !l2 || !x || !y || M < 1) return DQ_ERR_INVALID_ARG;
  if (l1->fmt != FMT_FP8S || l2->fmt != FMT_FP8S) return DQ_ERR_UNSUPPORTED;
  if (l2->K != l1->N || l1->N % TILE_N != 0) return DQ_ERR_INVALID_ARG;
  const int S = l1->N / TILE_N;                 // cluster size: one hidden tile per CTA
  // (the cluster's split-K hands each rank BN / S whole columns: S a power of two)
  if ((S != 2 && S != 4 && S != 8) || l2->N > TILE_N || l1->device != l2->device) return DQ_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(y) || (h_out && !aligned16(h_out))) return DQ_ERR_ALIGNMENT;
  const int bn = M <= 16 ? 16 : M <= 32 ? 32 : 64;
  const int m_tiles = (M + bn - 1) / bn;
  CUtensorMap tm;
  bool x3d = false;
  if (!x_map(l1, x, M, bn, false, &tm, &x3d)) return DQ_ERR_CUDA;
  GemmParams p{};
  p.wchunks = l1->wchunks;
  p.col_scale = l1->col_scale;
  p.bias = l1->bias;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.status = l1->status;
  p.sigma = l1->s_x;
  p.s_x = l1->s_x;
  p.s_out = l2->s_x;
  p.r_x = recip_rn(p.s_x);
  p.r_out = recip_rn(p.s_out);
  p.M = M;
  p.N = l1->N;
  p.k_stages = l1->k_stages;
  p.m_tiles = m_tiles;
  p.tiles = S * m_tiles;
  p.split = S;
  p.x3d = x3d ? 1 : 0;
  p.timeout_ns = l1->timeout_ns;
  p.drain_ns = std::max(timeout_ns(), kDefaultTimeoutNs);
  p.w2chunks = l2->wchunks;
  p.col_scale2 = l2->col_scale;
  p.bias2 = l2->bias;
  p.h_out = static_cast<__nv_bfloat16*>(h_out);
  p.N2 = l2->N;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int grid = S * m_tiles;
  cudaError_t e;
  switch (bn) {
    case 16: e = GemmLauncher<FMT_MLP, 16>::launch(tm, p, grid, s); break;
    case 32: e = GemmLauncher<FMT_MLP, 32>::launch(tm, p, grid, s); break;
    default: e = GemmLauncher<FMT_MLP, 64>::launch(tm, p, grid, s); break;
  }
  return cuda_err(e);
}

extern "C++" {
template <int FMT>
void launch_dequant(const dqgemm_s* h, float sigma, __nv_bfloat16* o, cudaStream_t s) {
  if constexpr (!is_w4a4(FMT)) {
    const dim3 grid(h->n_tiles, h->k_stages);
    dequant_kernel<FMT><<<grid, 256, 0, s>>>(h->wchunks, h->col_scale, sigma, h->mx_bias, h->N, h->K, h->k_stages, o);
  }
}
}

dqgemm_status dqgemm_dequantize(dqgemm_handle h, void* w_bf16, void* stream) {
  if (!h || !w_bf16) return DQ_ERR_INVALID_ARG;
  if (is_w4a4(h->fmt)) return DQ_ERR_UNSUPPORTED;   // no bf16 operand: the tensor core reads the codes
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(w_bf16);
  // static FP8: the weight alone is e4m3 * s_w[n] (sigma there is the activation scale)
  const float sigma = h->fmt == FMT_FP8S ? 1.f : h->sigma;
  DQ_FMT_SWITCH(h->fmt, launch_dequant<F>(h, sigma, o, s));
  return cuda_err(cudaGetLastError());
}

dqgemm_status dqgemm_quantize_act_fp8(const void* x, int M, int K, float s_x, void* q, void* stream) {
  if (!x || !q || M < 1 || K < 1 || !(std::isfinite(s_x) && s_x > 0.f)) return DQ_ERR_INVALID_ARG;
  const long long count = (long long)M * K;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  uint8_t* qb = static_cast<uint8_t*>(q);
  // 16 elements per thread where both buffers are 16-byte aligned, the
  // element-wise kernel for the tail (or for everything otherwise)
  long long done = 0;
  if (aligned16(x) && aligned16(q)) {
    const long long groups = count / 16;
    if (groups > 0) {
      const int blocks = (int)std::min<long long>((groups + 255) / 256, 148 * 8);
      act_quant16_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(xb), groups, s_x,
                                                 reinterpret_cast<uint4*>(qb));
      done = groups * 16;
    }
  }
  if (done < count) {
    const long long rest = count - done;
    const int blocks = (int)std::min<long long>((rest + 255) / 256, 148 * 8);
    act_quant_kernel<<<blocks, 256, 0, s>>>(xb + done, rest, s_x, qb + done);
  }
  return cuda_err(cudaGetLastError());
}

namespace {
// the canonical FP4 activation quantizer's NVFP4 amax scratch: partial
// maxima, then the ticket (zero-initialized, left at zero by every call)
static __device__ __align__(256) float g_act_fp4_scratch[kActAmaxBlocks + 4];
}  // namespace

dqgemm_status dqgemm_quantize_act_fp4(dqgemm_format fmt_, const void* x, int M, int K, void* codes, void* scales,
                                      float* g_x, void* stream) {
  const int fmt = storage_fmt((int)fmt_);
  if (fmt != FMT_MXFP4 && fmt != FMT_NVFP4) return DQ_ERR_UNSUPPORTED;
  const bool mx = fmt == FMT_MXFP4;
  if (!x || !codes || !scales || M < 1 || K < 1 || K % (mx ? 32 : 16) || (!mx && !g_x)) return DQ_ERR_INVALID_ARG;
  if (!aligned16(x)) return DQ_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  cudaError_t e = cudaSuccess;
  if (!mx) {
    void* scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_act_fp4_scratch) != cudaSuccess || !scratch) {
      cudaGetLastError();
      return DQ_ERR_CUDA;
    }
    float* partials = static_cast<float*>(scratch);
    const long long count = (long long)M * K;
    e = launch_chained(act_amax_kernel, act_amax_grid(count), 256, s, xb, count, partials,
                       reinterpret_cast<unsigned int*>(partials + kActAmaxBlocks), g_x);
  }
  if (e == cudaSuccess) {
    const int kp = (K + 63) / 64 * 64;
    const long long threads = (long long)M * (kp / 64);
    const int grid = (int)std::min<long long>((threads + 255) / 256, 148 * 8);
    uint8_t* c = static_cast<uint8_t*>(codes);
    uint8_t* sc = static_cast<uint8_t*>(scales);
    e = mx ? launch_chained(w4a4_act_quant_kernel<true>, grid, 256, s, xb, M, K, M, kp, 1, (const float*)g_x, c,
                            (uint32_t*)nullptr, sc)
           : launch_chained(w4a4_act_quant_kernel<false>, grid, 256, s, xb, M, K, M, kp, 1, (const float*)g_x, c,
                            (uint32_t*)nullptr, sc);
  }
  return cuda_err(e);
}

dqgemm_status dqgemm_pack_host(dqgemm_format fmt_, const float* W, int K, int N, void* packed, void* scales,
                               float* global_scale) {
  const int fmt = storage_fmt((int)fmt_);
  dqgemm_status st = check_shape(fmt, K, N);
  if (st != DQ_OK) return st;
  if (!W || !packed || !scales) return DQ_ERR_INVALID_ARG;
  const size_t count = (size_t)N * K;
  float amax = 0.f;
  for (size_t i = 0; i < count; ++i) {
    if (!std::isfinite(W[i])) return DQ_ERR_INVALID_ARG;
    amax = std::max(amax, std::fabs(W[i]));
  }
  uint8_t* P = static_cast<uint8_t*>(packed);
  float g = 1.f;
  std::vector<int8_t> c8(128);
  std::vector<uint8_t> cu(128);
  for (int n = 0; n < N; ++n) {
    const float* w = W + (size_t)n * K;
    if (fmt == FMT_INT4) {
      uint16_t* S = static_cast<uint16_t*>(scales);
      for (int gi = 0; gi < K / 128; ++gi) {
        S[(size_t)n * (K / 128) + gi] = quant_int4_group(w + gi * 128, 128, c8.data());
        for (int i = 0; i < 64; ++i)
          P[(size_t)n * (K / 2) + gi * 64 + i] = (uint8_t)((c8[2 * i] & 0xF) | ((c8[2 * i + 1] & 0xF) << 4));
      }
    } else if (fmt == FMT_INT4A) {
      uint8_t* S = static_cast<uint8_t*>(scales);
      const size_t G = (size_t)N * (K / 128);
      for (int gi = 0; gi < K / 128; ++gi) {
        const size_t idx = (size_t)n * (K / 128) + gi;
        uint8_t z = 0;
        const uint16_t sb = quant_int4_asym_group(w + gi * 128, 128, cu.data(), &z);
        S[idx * 2] = (uint8_t)(sb & 0xFF);
        S[idx * 2 + 1] = (uint8_t)(sb >> 8);
        S[2 * G + idx] = z;
        for (int i = 0; i < 64; ++i)
          P[(size_t)n * (K / 2) + gi * 64 + i] = (uint8_t)(cu[2 * i] | (cu[2 * i + 1] << 4));
      }
    } else if (fmt == FMT_NVFP4) {
      g = nvfp4_global_scale(amax);
      uint8_t* S = static_cast<uint8_t*>(scales);
      for (int b = 0; b < K / 16; ++b) {
        S[(size_t)n * (K / 16) + b] = quant_nvfp4_block(w + b * 16, 16, g, cu.data());
        for (int i = 0; i < 8; ++i) P[(size_t)n * (K / 2) + b * 8 + i] = (uint8_t)(cu[2 * i] | (cu[2 * i + 1] << 4));
      }
    } else if (fmt == FMT_MXFP4) {
      uint8_t* S = static_cast<uint8_t*>(scales);
      for (int b = 0; b < K / 32; ++b) {
        S[(size_t)n * (K / 32) + b] = quant_mxfp4_block(w + b * 32, 32, cu.data());
        for (int i = 0; i < 16; ++i)
          P[(size_t)n * (K / 2) + b * 16 + i] = (uint8_t)(cu[2 * i] | (cu[2 * i + 1] << 4));
      }
    } else {
      float* S = static_cast<float*>(scales);
      S[n] = quant_fp8_row(w, K, P + (size_t)n * K);
    }
  }
  if (global_scale) *global_scale = (fmt == FMT_NVFP4) ? nvfp4_global_scale(amax) : 1.f;
  return DQ_OK;
}

dqgemm_status dqgemm_pack_device(dqgemm_format fmt_, const float* W, int K, int N, void* packed, void* scales,
                                 float* global_scale, void* stream) {
  const int fmt = storage_fmt((int)fmt_);
  dqgemm_status st = check_shape(fmt, K, N);
  if (st != DQ_OK) return st;
  if (!W || !packed || !scales) return DQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scales)) return DQ_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* P = static_cast<uint8_t*>(packed);
  const long long count = (long long)N * K;
  unsigned int* amax = nullptr;
  float* gdev = nullptr;
  if (cudaMalloc(&amax, 8) != cudaSuccess) return DQ_ERR_ALLOC;
  gdev = reinterpret_cast<float*>(amax + 1);
  cudaError_t e = cudaMemsetAsync(amax, 0, 8, s);
  const int T = 256;
  if (fmt == FMT_INT4) {
    const long long n = (long long)N * (K / 128);
    pack_int4_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, P, static_cast<uint16_t*>(scales));
  } else if (fmt == FMT_INT4A) {
    const long long n = (long long)N * (K / 128);
    pack_int4a_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, P, static_cast<uint8_t*>(scales));
  } else if (fmt == FMT_NVFP4) {
    amax_kernel<<<(unsigned)std::min<long long>((count + T - 1) / T, 4096), T, 0, s>>>(W, count, amax);
    const long long n = (long long)N * (K / 16);
    pack_nvfp4_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, amax, P, static_cast<uint8_t*>(scales),
                                                                gdev);
  } else if (fmt == FMT_MXFP4) {
    const long long n = (long long)N * (K / 32);
    pack_mxfp4_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, P, static_cast<uint8_t*>(scales));
  } else {
    pack_fp8_kernel<<<(unsigned)((N + 7) / 8), T, 0, s>>>(W, N, K, P, static_cast<float*>(scales));
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess && global_scale) {
    float g = 1.f;
    if (fmt == FMT_NVFP4) e = cudaMemcpyAsync(&g, gdev, 4, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    *global_scale = g;
  }
  cudaStreamSynchronize(s);
  cudaFree(amax);
  return cuda_err(e);
}

// ---------------------------------------------------------------------------
// allocation-free GPU packer: the NVFP4 tensor-amax scratch lives in a
// file-scope device array instead of cudaMalloc'd memory
// ---------------------------------------------------------------------------
namespace {
constexpr int kNoAllocMaxPartials = 4096;          // partial maxima the scratch holds
constexpr long long kNoAllocChunk = 65536;         // weights reduced per partial
// [0, 4096): partial maxima; [4096]: amax bits; [4097]: global scale g
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxPartials + 2];

// Device address of the scratch on the current device.  The symbol's
// host-side name is not a device address, so it is looked up on every call:
// a cached address would go stale if the device's primary context were torn
// down and the library's device code loaded again.
float* noalloc_scratch(dqgemm_status* st) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    *st = DQ_ERR_CUDA;
    return nullptr;
  }
  *st = DQ_OK;
  return static_cast<float*>(p);
}
}  // namespace

dqgemm_status dqgemm_pack_device_noalloc(dqgemm_format fmt_, const float* W, int K, int N, void* packed,
                                         void* scales, float* global_scale, void* stream) {
  const int fmt = storage_fmt((int)fmt_);
  dqgemm_status st = check_shape(fmt, K, N);
  if (st != DQ_OK) return st;
  if (!W || !packed || !scales) return DQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scales)) return DQ_ERR_ALIGNMENT;
  const long long count = (long long)N * K;
  const long long nparts = (count + kNoAllocChunk - 1) / kNoAllocChunk;
  if (fmt == FMT_NVFP4 && nparts > kNoAllocMaxPartials) return DQ_ERR_UNSUPPORTED;   // N*K > 2^28
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* P = static_cast<uint8_t*>(packed);
  const int T = 256;
  cudaError_t e = cudaSuccess;
  float g = 1.f;
  if (fmt == FMT_INT4) {
    const long long n = (long long)N * (K / 128);
    pack_int4_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, P, static_cast<uint16_t*>(scales));
  } else if (fmt == FMT_INT4A) {
    const long long n = (long long)N * (K / 128);
    pack_int4a_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, P, static_cast<uint8_t*>(scales));
  } else if (fmt == FMT_NVFP4) {
    float* scratch = noalloc_scratch(&st);
    if (!scratch) return st;
    unsigned int* amax = reinterpret_cast<unsigned int*>(scratch + kNoAllocMaxPartials);
    float* gdev = scratch + kNoAllocMaxPartials + 1;
    // every scratch word read below is written earlier in the same call
    amax_partials_kernel<<<(unsigned)nparts, T, 0, s>>>(W, count, kNoAllocChunk, scratch);
    amax_final_kernel<<<1, T, 0, s>>>(scratch, (int)nparts, amax);
    const long long n = (long long)N * (K / 16);
    pack_nvfp4_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, amax, P, static_cast<uint8_t*>(scales),
                                                                gdev);
    e = cudaGetLastError();
    if (e == cudaSuccess && global_scale) e = cudaMemcpyAsync(&g, gdev, 4, cudaMemcpyDeviceToHost, s);
  } else if (fmt == FMT_MXFP4) {
    const long long n = (long long)N * (K / 32);
    pack_mxfp4_kernel<<<(unsigned)((n + T - 1) / T), T, 0, s>>>(W, N, K, P, static_cast<uint8_t*>(scales));
  } else {
    pack_fp8_kernel<<<(unsigned)((N + 7) / 8), T, 0, s>>>(W, N, K, P, static_cast<float*>(scales));
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess && global_scale) {
    e = cudaStreamSynchronize(s);
    *global_scale = g;
  }
  return cuda_err(e);
}

dqgemm_status dqgemm_last_error(dqgemm_handle h) {
  if (!h) return DQ_ERR_INVALID_ARG;
  volatile int* w = h->status_host;
  const int v = *w;
  if (v != 0) *w = 0;
  return v == 0 ? DQ_OK : (dqgemm_status)v;
}

dqgemm_status dqgemm_selftest_timeout(int timeout_us, void* stream) {
  if (timeout_us < 1) return DQ_ERR_INVALID_ARG;
  int* status = nullptr;
  if (cudaMalloc(&status, sizeof(int)) != cudaSuccess) return DQ_ERR_ALLOC;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(status, 0xFF, sizeof(int), s);
  selftest_timeout_kernel<<<1, 32, 0, s>>>(status, (unsigned long long)timeout_us * 1000ull);
  if (e == cudaSuccess) e = cudaGetLastError();
  int v = -1;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&v, status, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFree(status);
  if (e != cudaSuccess) return DQ_ERR_CUDA;
  return v == DEV_TIMEOUT ? DQ_ERR_TIMEOUT : (v == DEV_OK ? DQ_OK : DQ_ERR_CUDA);
}

}  // extern "C"
