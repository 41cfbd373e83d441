/*
 * dqgemm.h -- C ABI of libdqgemm: a quantized nn.Linear for NVIDIA B200
 * (sm_100a) whose low-bit weight stays packed in HBM and is dequantized in
 * the prologue of a tcgen05 tensor-core GEMM:
 *
 *     y[M, N] = x[M, K] . deq(W)[N, K]^T + b[N]        (x, y, b in bf16)
 *
 * The operation is the one the Torch-TensorRT / TorchAO tutorial pages build
 * as "weight constant + DQ prologue into GEMM":
 *   - "TorchAO INT4 Weight-Only Quantization (Linear)", intro: symmetric
 *     group-wise INT4 (zero-point 0, group_size=128), DQ prologue into GEMM.
 *   - "TorchAO NVFP4 Weight-Only Quantization (Linear)", intro: packed FP4
 *     E2M1 weights, FP8 E4M3 block scales, FP32 global scale, two-level DQ
 *     prologue into a high-precision GEMM; activations stay bf16.
 *   - "TorchAO MXFP4 Dynamic Activation + MX Weight (Linear)", intro: packed
 *     E2M1 weights, E8M0 block scales, block size 32, weight DQ prologue.
 *   - "TorchAO FP8 Weight-Only Quantization (Linear)", intro: FP8 weight
 *     constant plus a DQ prologue fused into the matmul on Blackwell.
 *   - "TorchAO Static FP8 Quantization (Linear)", intro and "Graph after
 *     export": activations quantized to e4m3 with a calibrated per-tensor
 *     scale, weights e4m3 per channel, GEMM in FP8 on the tensor cores.
 *
 * Conventions for every entry point
 *   - All pointers are plain pointers.  "device" means memory the CUDA device
 *     can address (cudaMalloc / torch CUDA tensors); "host" means CPU memory.
 *   - Matrices are row-major and densely packed.  W is [N, K] as in
 *     nn.Linear (out_features x in_features); groups / blocks run along K.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls that take a stream are asynchronous on it.
 *   - Every entry point returns a dqgemm_status.  Argument checks are
 *     synchronous.  Nothing aborts, throws or traps across this boundary.
 *   - Device pointers must be 16-byte aligned (DQ_ERR_ALIGNMENT otherwise),
 *     except where an entry point says so.
 *   - The library never frees or retains caller memory.
 *   - A handle belongs to the device that was current at dqgemm_create.  Every
 *     later call on it must be made with that device current, with x, y and
 *     the stream on that device (not checked: the launch goes to the current
 *     device).
 *   - The run entry points keep no host state between calls apart from a
 *     small cache of the activation tensor maps they encode (a map depends
 *     only on x, M and the tile; the cache is locked), so one handle may be
 *     run from several host threads and streams at once.
 *     dqgemm_destroy must not overlap any other call on the same handle, nor
 *     any of its kernels still in flight.
 *
 * Environment variables, each read once per process, for tuning and tests
 * only (results do not depend on them except through the split, which only
 * changes the fp32 summation order):
 *   DQGEMM_TIMEOUT_MS   limit of every device-side wait (default 2000 ms).
 *   DQGEMM_PDL=0        launch without programmatic dependent launch.
 *   DQGEMM_SPLIT=S      force the split-K depth to the largest power of two
 *                       <= min(S, 8, K/128) that fits the cluster limits.
 *   DQGEMM_CTAS_PER_SM  2 lets the split plan count two resident CTAs per SM
 *                       for the skinny tiles (default 1).
 */
#ifndef DQGEMM_H
#define DQGEMM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Weight formats and the canonical storage each takes at dqgemm_create.
 *   DQ_INT4_G128   packed  u8 [N, K/2]: two's-complement nibbles, low nibble = even k
 *                  scales  bf16 [N, K/128] (one per group of 128 along K)
 *                  K % 128 == 0
 *   DQ_NVFP4       packed  u8 [N, K/2]: E2M1 nibbles, low nibble = even k
 *                  scales  u8 [N, K/16]: E4M3 block scales (one per 16 along K)
 *                  global_scale: the FP32 global scale g;  K % 16 == 0, N % 16 == 0
 *   DQ_MXFP4       packed  u8 [N, K/2]: E2M1 nibbles, low nibble = even k
 *                  scales  u8 [N, K/32]: E8M0 block exponents 2^(e-127)
 *                  K % 32 == 0, N % 32 == 0
 *   DQ_FP8_WO      packed  u8 [N, K]: E4M3 codes;  scales fp32 [N] per channel
 *                  K % 16 == 0
 *   DQ_FP8_STATIC  as DQ_FP8_WO, plus global_scale = the calibrated fp32
 *                  per-tensor activation scale s_x; the GEMM runs FP8 x FP8
 *                  on e4m3(x / s_x) and rescales by s_x * s_w[n].
 *   DQ_INT4_ASYM_G128  asymmetric INT4 with a zero point per group of 128
 *                  (the zero-point counterpart of the INT4 page's symmetric
 *                  format): packed u8 [N, K/2] unsigned nibbles 0..15, low
 *                  nibble = even k; scales u8 [3 * N * K/128]: the bf16
 *                  scales [N, K/128] followed by the u8 zero points
 *                  [N, K/128] in [0, 15]; weight = (code - z) * s;
 *                  K % 128 == 0
 *   DQ_W4A4_MXFP4  FP4 x FP4 ("TorchAO MXFP4 Dynamic Activation + MX Weight
 *                  (Linear)", intro: MX dynamic activation + MX weight, native
 *                  MXFP4 x MXFP4 on B200): the weight in DQ_MXFP4 storage;
 *                  each call quantizes x to MXFP4 (E8M0 per 32 along K, the
 *                  weight's recipe) and runs the tensor core's block-scaled
 *                  FP4 MMA, y = sum_k deq(Q(x)) deq(W) + b.
 *                  K % 32 == 0, N % 32 == 0
 *   DQ_W4A4_NVFP4  the same with NVFP4: the weight in DQ_NVFP4 storage
 *                  (global_scale = g_w); x quantized per call with its own
 *                  global scale g_x = amax(x) / 2688 and E4M3 scales per 16.
 *                  K % 16 == 0, N % 16 == 0
 */
typedef enum {
  DQ_INT4_G128 = 0,
  DQ_NVFP4 = 1,
  DQ_MXFP4 = 2,
  DQ_FP8_WO = 3,
  DQ_FP8_STATIC = 4,
  DQ_INT4_ASYM_G128 = 5,
  DQ_W4A4_MXFP4 = 6,
  DQ_W4A4_NVFP4 = 7
} dqgemm_format;

typedef enum {
  DQ_OK = 0,
  DQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size or divisibility, unknown format */
  DQ_ERR_UNSUPPORTED = 2,  /* valid request this build cannot serve (e.g. scale range) */
  DQ_ERR_ALIGNMENT = 3,    /* a device pointer is not 16-byte aligned */
  DQ_ERR_ALLOC = 4,        /* device or host allocation failed */
  DQ_ERR_CUDA = 5,         /* a CUDA runtime/driver call or a launch failed */
  DQ_ERR_TIMEOUT = 6       /* a bounded device-side wait expired (see dqgemm_last_error) */
} dqgemm_status;

typedef struct dqgemm_s* dqgemm_handle;

/* Create a quantized Linear.  Reads `packed_w`, `scales` and `bias` (device
 * pointers in the canonical layout above; `bias` is bf16 [N] or NULL), copies
 * them, and re-lays the weight out into the kernel's tile order in device
 * memory owned by the handle (the analogue of the INT4 page's "re-packs ...
 * into an INT4 constant at build time", "Export and compile").  The caller may
 * free its buffers afterwards; the weights are immutable for the handle's
 * life.  Synchronizes the device.  On error *out is set to NULL.
 * Stored codes outside what the formats define are refused with
 * DQ_ERR_INVALID_ARG: a NaN weight code (0x7F / 0xFF) of the FP8 formats, an
 * NVFP4 block scale that is negative or NaN (the block scales are
 * non-negative E4M3), an MXFP4 exponent 0xFF.  An MXFP4 handle whose largest
 * block exponent code emax exceeds 128 needs every block holding a nonzero
 * element to have a code >= emax - 133 (the bf16 operand of the prologue
 * covers a span of 2^133 exactly); DQ_ERR_UNSUPPORTED otherwise.  (The W4A4
 * formats take every non-NaN exponent: their scales go to the tensor core
 * unchanged.) */
dqgemm_status dqgemm_create(dqgemm_handle* out, dqgemm_format fmt, int K, int N,
                            const void* packed_w, const void* scales,
                            float global_scale, const void* bias);

/* y = x . deq(W)^T + b.  x: device bf16 [M, K]; y: device bf16 [M, N]; M >= 1.
 * One kernel launch on `stream` (no allocation, no synchronization).  For
 * DQ_FP8_STATIC the activation is quantized to e4m3 inside the same kernel.
 * When there are fewer output tiles than SMs the K range of a tile is split
 * over a thread-block cluster whose partial sums meet in distributed shared
 * memory (deterministic).  Launched with programmatic dependent launch: the
 * kernel streams its weights before waiting for the previous kernel in the
 * stream, and reads x / writes y only after that wait.  Device-side wait
 * timeouts are reported through dqgemm_last_error after the stream has been
 * synchronized.
 * W4A4 handles launch two kernels (MXFP4: quantize x, GEMM) or three (NVFP4:
 * amax of x, quantize, GEMM), chained the same way.  The quantized x lives
 * in a workspace the handle owns (dqgemm_plan.workspace_bytes for M): a call
 * that needs more than the handle holds allocates it, after synchronizing the
 * device, so make the first call of the largest M before any stream capture.
 * Calls on one W4A4 handle share that workspace and must be stream-ordered
 * (not concurrent on different streams). */
dqgemm_status dqgemm_run(dqgemm_handle h, const void* x, int M, void* y, void* stream);

/* DQ_FP8_STATIC only: the GEMM on activations already quantized by
 * dqgemm_quantize_act_fp8 with the handle's s_x (the static page's "Graph
 * after export": the Q node's e4m3 output feeds the FP8 GEMM).  q: device u8
 * [M, K] e4m3 codes, row-major, 16-byte aligned; y as in dqgemm_run.  The
 * result is bit-identical to dqgemm_run on the x that q was quantized from;
 * the in-kernel quantization of dqgemm_run is repeated for every 128-channel
 * tile, so for larger M (about 128 rows and up) quantizing once and calling
 * this is faster.  DQ_ERR_UNSUPPORTED for other formats. */
dqgemm_status dqgemm_run_fp8_static_quantized(dqgemm_handle h, const void* q, int M, void* y, void* stream);

/* Chained static FP8 (the static page's two-layer "Graph after export", where
 * the next layer's Q node reads this layer's output): as dqgemm_run, but the
 * result leaves the kernel as the next layer's e4m3 activation codes,
 * q_out[m, n] = e4m3(f32(y[m, n]) / s_out) with y the bf16 result, IEEE
 * division, round to nearest even, saturating -- the codes
 * dqgemm_quantize_act_fp8(y, s_out) would give.  q_out: device u8 [M, N],
 * 16-byte aligned; s_out > 0 (DQ_ERR_INVALID_ARG otherwise).  Any format. */
dqgemm_status dqgemm_run_quantized_out(dqgemm_handle h, const void* x, int M, void* q_out, float s_out,
                                       void* stream);

/* DQ_FP8_STATIC only: both ends quantized -- the input as for
 * dqgemm_run_fp8_static_quantized, the output as for
 * dqgemm_run_quantized_out (a middle layer of a static-FP8 chain). */
dqgemm_status dqgemm_run_fp8_static_quantized_out(dqgemm_handle h, const void* q, int M, void* q_out,
                                                  float s_out, void* stream);

/* The static page's two-layer model in one launch ("TorchAO Static FP8
 * Quantization (Linear)", "Define a small two-layer Linear model" and the
 * Q -> DQ -> GEMM -> Q -> DQ -> GEMM chain of its "Graph after export"):
 *     h = bf16(layer1(x)),  y = bf16(layer2(e4m3(h / s_x2)))
 * with l1, l2 DQ_FP8_STATIC handles (s_x2 is l2's activation scale, each
 * layer's bias added if its handle has one).  Layer 1's output never leaves
 * the chip: CTA q of a thread-block cluster computes hidden units
 * [128q, 128q+128) over all of K, quantizes them into layer 2's operand in
 * shared memory, multiplies them by layer 2's matching k-slice, and the
 * cluster adds the slices in rank order (deterministic).
 * x: device bf16 [M, K1]; y: device bf16 [M, N2]; h_out: NULL or device bf16
 * [M, N1] receiving layer 1's output (for checks; y does not depend on it).
 * Requirements: l2's K equals l1's N; N1 = 128 * S with S = 2, 4 or 8
 * (256, 512 or 1024 hidden units); N2 <= 128; both handles on the current device (DQ_ERR_INVALID_ARG or
 * DQ_ERR_UNSUPPORTED otherwise); 16-byte aligned buffers.  Layer 1 sums
 * over K in one CTA, so h can differ in the last bit from a separate
 * dqgemm_run of l1 (which may split K); everything else is the same
 * arithmetic as two dqgemm_run calls.  Device-side timeouts are reported
 * through dqgemm_last_error(l1). */
dqgemm_status dqgemm_run_static_mlp(dqgemm_handle l1, dqgemm_handle l2, const void* x, int M,
                                    void* h_out, void* y, void* stream);

/* Release the handle and its device memory.  Synchronizes the device (the
 * CUDA runtime's cudaFree does so in any case); no kernel of the handle may
 * still be queued or running. */
dqgemm_status dqgemm_destroy(dqgemm_handle h);

/* Debug: write the dequantized weight as bf16 [N, K] (device) from the
 * handle's re-laid-out storage, through the same unpack code the GEMM
 * prologue uses:  INT4 bf16(c*s);  NVFP4 bf16(f32(e2m1*dec(sb)*g));
 * MXFP4 bf16(e2m1*2^(e-127));  FP8 bf16(f32(e4m3*s[n])).  -0.0 is kept. */
dqgemm_status dqgemm_dequantize(dqgemm_handle h, void* w_bf16, void* stream);

/* Static-FP8 activation quantization (the Q node of the static FP8 page's
 * "Graph after export"): q[m,k] = e4m3(f32(x[m,k] / s_x)), IEEE division,
 * round to nearest even, saturating to +-448.  x: device bf16 [M, K];
 * q: device u8 [M, K]; s_x finite and > 0, M >= 1, K >= 1, else
 * DQ_ERR_INVALID_ARG.  Element-wise, so x and q need only their natural
 * alignment (the one exception to the 16-byte rule above). */
dqgemm_status dqgemm_quantize_act_fp8(const void* x, int M, int K, float s_x,
                                      void* q, void* stream);

/* FP4 activation quantization, the first step of a W4A4 call, into the
 * canonical storage of the weight formats (the same recipe as the packers
 * below, applied per call to each row of x).  fmt DQ_MXFP4 or DQ_W4A4_MXFP4:
 * codes u8 [M, K/2] (E2M1 nibbles, low nibble = even k), scales u8 [M, K/32]
 * E8M0; K % 32 == 0.  fmt DQ_NVFP4 or DQ_W4A4_NVFP4: g_x = amax(x) / 2688
 * (1 for a zero x) written to the device float *g_x, then scales u8
 * [M, K/16] E4M3 under g_x and the codes; K % 16 == 0.  x: device bf16
 * [M, K], 16-byte aligned; codes, scales: device.  The NVFP4 form reduces
 * the amax in a static device scratch shared by all calls: calls that
 * overlap on the GPU race.  DQ_ERR_UNSUPPORTED for other formats. */
dqgemm_status dqgemm_quantize_act_fp4(dqgemm_format fmt, const void* x, int M, int K,
                                      void* codes, void* scales, float* g_x, void* stream);

/* Quantize and pack a host fp32 weight [N, K] into the canonical layout of
 * `fmt` (host outputs `packed` and `scales`, sized as listed above).  The
 * recipes (fp32 operations, round to nearest even):
 *   INT4   s = bf16(amax_group/7); c = clamp(rne(W/s), -8, 7); s == 0 -> c = 0
 *   NVFP4  g = amax/2688 (1 if amax == 0); sb = e4m3((amax_blk16/6)/g);
 *          c = e2m1(W/(dec(sb)*g)), saturating; 0 where the divisor is 0
 *   MXFP4  e = floor(log2 amax_blk32) - 2 in [-127,127]; code e+127 (0 for a
 *          zero block); c = e2m1(W * 2^-e), saturating
 *   FP8    s[n] = max|W[n,:]|/448; c = e4m3(W/s[n]) (0 for a zero row)
 *   INT4 asymmetric  lo = min(0, min W), hi = max(0, max W) per group;
 *          s = bf16(f32(hi - lo)/15); z = clamp(rne(-lo/s), 0, 15);
 *          c = clamp(rne(W/s) + z, 0, 15); s == 0 -> c = 0, z = 0; a group
 *          whose range hi - lo exceeds the fp32 maximum (weights of both
 *          signs near +-3.4e38) gets an infinite scale: it is not rejected
 * `global_scale` (host, may be NULL) receives g for NVFP4 and 1 otherwise.
 * DQ_ERR_INVALID_ARG if W holds a non-finite value. */
dqgemm_status dqgemm_pack_host(dqgemm_format fmt, const float* W, int K, int N,
                               void* packed, void* scales, float* global_scale);

/* Same as dqgemm_pack_host on the GPU: W, packed and scales are device
 * pointers; results are bit-identical to dqgemm_pack_host.  If
 * `global_scale` (host pointer) is not NULL the call synchronizes `stream`
 * and stores g there.  Allocates and frees 8 bytes of device memory. */
dqgemm_status dqgemm_pack_device(dqgemm_format fmt, const float* W, int K, int N,
                                 void* packed, void* scales, float* global_scale,
                                 void* stream);

/* dqgemm_pack_device without any device allocation, for callers that cannot
 * call cudaMalloc: a serving process that reserved all device memory up
 * front, or code that must not trigger the device-wide synchronization that
 * cudaMalloc / cudaFree may cause while other streams run.  The tutorial
 * pages have no counterpart; this is a deployment variant of the packer.
 * Results are bit-identical to dqgemm_pack_device.  NVFP4 needs a tensor-wide
 * amax: its two-pass reduction keeps up to 4096 partial maxima (one per
 * 65536 weights) in a static device array that every GPU loading the library
 * holds (16 KB) until exit, so NVFP4 requires N*K <= 4096*65536 and returns
 * DQ_ERR_UNSUPPORTED beyond that; the other formats need no scratch.  Each
 * NVFP4 call looks up the array's device address on the current device
 * (cudaGetSymbolAddress); the first such call on a device may load the
 * library's device code, so make it before any stream capture.  All calls
 * share the array: calls whose kernels overlap on the GPU race with each
 * other.  If `global_scale` (host) is not
 * NULL the call synchronizes `stream` and stores g there. */
dqgemm_status dqgemm_pack_device_noalloc(dqgemm_format fmt, const float* W, int K, int N,
                                         void* packed, void* scales, float* global_scale,
                                         void* stream);

/* Status of the device-side checks of the handle's completed kernels (DQ_OK,
 * or DQ_ERR_TIMEOUT if a bounded wait of any of them gave up), then clears
 * it.  The status word is host memory the kernels write into: this call does
 * not synchronize anything, so synchronize the streams the handle's kernels
 * ran on first (a kernel still running may report later). */
dqgemm_status dqgemm_last_error(dqgemm_handle h);

/* Test and diagnostic use: the limit, in nanoseconds, of the device-side
 * waits of this handle's GEMM pipeline (0 restores the default, which is
 * DQGEMM_TIMEOUT_MS or 2 s).  A wait that does not complete at once gives up
 * when its limit has passed: the kernel then records DQ_ERR_TIMEOUT (read by
 * dqgemm_last_error) and writes no output of the tiles it gave up on.  The
 * waits for a CTA's own copies, tensor-core operations and received split-K
 * partials keep a limit of at least the default, so that no kernel leaves
 * memory that is still being written.  Calls already launched keep the limit
 * they were launched with.  DQ_ERR_INVALID_ARG for a null handle or a
 * negative limit. */
dqgemm_status dqgemm_set_wait_limit(dqgemm_handle h, long long timeout_ns);

/* Diagnostic: launch a kernel whose only wait can never complete and which
 * must give up after `timeout_us` microseconds; returns DQ_ERR_TIMEOUT when
 * the bounded wait worked (the context stays usable), DQ_OK never.
 * Synchronizes `stream`. */
dqgemm_status dqgemm_selftest_timeout(int timeout_us, void* stream);

/* Launch plan that dqgemm_run uses for a given M (for benchmarks and tests). */
typedef struct {
  int bn;               /* MMA N (activation rows per tile): 16, 32, 64 or 128 */
  int m_tiles;          /* ceil(M / bn) */
  int n_tiles;          /* ceil(N / 128) */
  int k_stages;         /* ceil(K / 128) */
  int grid;             /* CTAs launched (<= number of SMs) */
  int max_segments;     /* most CTAs sharing one output tile (split-K depth) */
  int stages;           /* shared-memory pipeline depth */
  int smem_bytes;       /* dynamic shared memory per CTA */
  long long workspace_bytes; /* global split-K scratch the plan needs (0: partials stay on chip) */
  long long weight_bytes;    /* packed weight + scale bytes streamed per call */
  int x_stages;         /* activation-tile ring depth (128-k stages) */
  int max_cta_stages;   /* most 128-k weight stages one CTA streams */
} dqgemm_plan;

dqgemm_status dqgemm_get_plan(dqgemm_handle h, int M, dqgemm_plan* plan);

/* Human-readable name of a status code (static storage). */
const char* dqgemm_status_string(dqgemm_status s);

#ifdef __cplusplus
}
#endif

#endif /* DQGEMM_H */
