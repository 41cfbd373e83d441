/* A plain C99 user of libdqgemm: it sees only include/dqgemm.h and the
 * shared library (plus the CUDA runtime for device memory in "gemm" mode),
 * with no Python or C++ in the loop.  tests/test_c_consumer.py builds it
 * with gcc and compares what it writes against the oracle.
 *
 *   dq_consumer pack FMT K N W.f32 OUT
 *       dqgemm_pack_host on the fp32 weight [N, K]; OUT gets the int32
 *       status, the fp32 global scale, the packed bytes, the scale bytes.
 *   dq_consumer errors
 *       prints "<case> <status>" for argument errors that every entry point
 *       must report as a status (no device needed).
 *   dq_consumer gemm FMT M K N SX W.f32 X.bf16 B.bf16 OUT      (needs a GPU)
 *       packs W on the device, creates the layer (SX = the static-FP8
 *       activation scale, ignored otherwise), runs y = x . deq(W)^T + b
 *       once on the default stream and writes y bf16 [M, N] to OUT.
 *
 * Exit status: 0 when every call that should succeed returned DQ_OK.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <math.h>
#include <string.h>

#include "dqgemm.h"

#ifdef DQ_CONSUMER_GPU
#include <cuda_runtime_api.h>
#endif

static size_t packed_bytes(int fmt, int K, int N) {
  return (fmt == DQ_FP8_WO || fmt == DQ_FP8_STATIC) ? (size_t)N * K : (size_t)N * K / 2;
}

static size_t scale_bytes(int fmt, int K, int N) {
  switch (fmt) {
    case DQ_INT4_G128: return (size_t)N * (K / 128) * 2;
    case DQ_INT4_ASYM_G128: return (size_t)N * (K / 128) * 3;
    case DQ_NVFP4: return (size_t)N * (K / 16);
    case DQ_MXFP4: return (size_t)N * (K / 32);
    default: return (size_t)N * 4;
  }
}

static void* read_exact(const char* path, size_t n) {
  FILE* f = fopen(path, "rb");
  void* p = malloc(n ? n : 1);
  if (!f || !p || fread(p, 1, n, f) != n) {
    fprintf(stderr, "cannot read %zu bytes from %s\n", n, path);
    exit(2);
  }
  fclose(f);
  return p;
}

static void write_all(FILE* f, const void* p, size_t n) {
  if (fwrite(p, 1, n, f) != n) {
    fprintf(stderr, "short write\n");
    exit(2);
  }
}

static int do_pack(int fmt, int K, int N, const char* win, const char* out) {
  float* W = (float*)read_exact(win, (size_t)N * K * sizeof(float));
  size_t pb = packed_bytes(fmt, K, N), sb = scale_bytes(fmt, K, N);
  void* packed = malloc(pb);
  void* scales = malloc(sb);
  float g = 0.f;
  int32_t st = (int32_t)dqgemm_pack_host((dqgemm_format)fmt, W, K, N, packed, scales, &g);
  FILE* f = fopen(out, "wb");
  if (!f) return 2;
  write_all(f, &st, sizeof st);
  write_all(f, &g, sizeof g);
  write_all(f, packed, pb);
  write_all(f, scales, sb);
  fclose(f);
  free(W);
  free(packed);
  free(scales);
  return st == DQ_OK ? 0 : 1;
}

static int do_errors(void) {
  /* malloc returns memory aligned for any type: 16 bytes on x86-64 */
  float* w = (float*)calloc(256, sizeof(float));
  uint8_t* packed = (uint8_t*)calloc(256, 1);
  uint8_t* scales = (uint8_t*)calloc(16, 1);
  float g;
  dqgemm_handle h = NULL;
  dqgemm_plan plan;
  if (!w || !packed || !scales) return 2;
  printf("pack_null_weight %d\n", (int)dqgemm_pack_host(DQ_INT4_G128, NULL, 128, 2, packed, scales, &g));
  printf("pack_k_not_group %d\n", (int)dqgemm_pack_host(DQ_INT4_G128, w, 100, 2, packed, scales, &g));
  printf("pack_unknown_format %d\n", (int)dqgemm_pack_host((dqgemm_format)9, w, 128, 2, packed, scales, &g));
  w[3] = INFINITY;
  printf("pack_non_finite %d\n", (int)dqgemm_pack_host(DQ_FP8_WO, w, 128, 2, packed, scales, &g));
  printf("create_null_out %d\n", (int)dqgemm_create(NULL, DQ_INT4_G128, 128, 128, packed, scales, 1.f, NULL));
  printf("create_null_weight %d %d\n",
         (int)dqgemm_create(&h, DQ_INT4_G128, 128, 128, NULL, scales, 1.f, NULL), h == NULL);
  printf("run_null_handle %d\n", (int)dqgemm_run(NULL, packed, 1, packed, NULL));
  printf("plan_null_handle %d\n", (int)dqgemm_get_plan(NULL, 1, &plan));
  printf("destroy_null %d\n", (int)dqgemm_destroy(NULL));
  printf("last_error_null %d\n", (int)dqgemm_last_error(NULL));
  /* 16-byte alignment is checked before any device access */
  printf("create_misaligned %d\n",
         (int)dqgemm_create(&h, DQ_INT4_G128, 128, 128, packed + 1, scales, 1.f, NULL));
  printf("pack_device_misaligned %d\n",
         (int)dqgemm_pack_device(DQ_INT4_G128, w + 1, 128, 2, packed, scales, NULL, NULL));
  printf("pack_device_null %d\n", (int)dqgemm_pack_device(DQ_INT4_G128, NULL, 128, 2, packed, scales, NULL, NULL));
  printf("act_quant_m0 %d\n", (int)dqgemm_quantize_act_fp8(packed, 0, 16, 1.f, packed, NULL));
  printf("act_quant_zero_scale %d\n", (int)dqgemm_quantize_act_fp8(packed, 1, 16, 0.f, packed, NULL));
  printf("act_quant_nan_scale %d\n", (int)dqgemm_quantize_act_fp8(packed, 1, 16, NAN, packed, NULL));
  printf("status_string %s\n", dqgemm_status_string(DQ_ERR_INVALID_ARG));
  free(w);
  free(packed);
  free(scales);
  return 0;
}

#ifdef DQ_CONSUMER_GPU
#define CK(call)                                                            \
  do {                                                                      \
    int s_ = (int)(call);                                                   \
    if (s_ != 0) {                                                          \
      fprintf(stderr, "%s failed: %d (%s)\n", #call, s_, dqgemm_status_string((dqgemm_status)s_)); \
      return 1;                                                             \
    }                                                                       \
  } while (0)
#define CUDA(call)                                                          \
  do {                                                                      \
    if ((call) != cudaSuccess) {                                            \
      fprintf(stderr, "%s failed\n", #call);                                \
      return 1;                                                             \
    }                                                                       \
  } while (0)

static int do_gemm(int fmt, int M, int K, int N, float s_x, const char* win, const char* xin,
                   const char* bin, const char* out) {
  size_t wb = (size_t)N * K * sizeof(float), xb = (size_t)M * K * 2, yb = (size_t)M * N * 2;
  size_t pb = packed_bytes(fmt, K, N), sb = scale_bytes(fmt, K, N);
  float* W = (float*)read_exact(win, wb);
  void* x = read_exact(xin, xb);
  void* b = read_exact(bin, (size_t)N * 2);
  void* y = malloc(yb);
  void *dW, *dp, *ds, *dx, *db, *dy;
  float g = 1.f;
  dqgemm_handle h = NULL;
  int pack_fmt = fmt == DQ_FP8_STATIC ? DQ_FP8_WO : fmt;
  CUDA(cudaMalloc(&dW, wb));
  CUDA(cudaMalloc(&dp, pb));
  CUDA(cudaMalloc(&ds, sb));
  CUDA(cudaMalloc(&dx, xb));
  CUDA(cudaMalloc(&db, (size_t)N * 2));
  CUDA(cudaMalloc(&dy, yb));
  CUDA(cudaMemcpy(dW, W, wb, cudaMemcpyHostToDevice));
  CUDA(cudaMemcpy(dx, x, xb, cudaMemcpyHostToDevice));
  CUDA(cudaMemcpy(db, b, (size_t)N * 2, cudaMemcpyHostToDevice));
  CK(dqgemm_pack_device((dqgemm_format)pack_fmt, (const float*)dW, K, N, dp, ds, &g, NULL));
  if (fmt == DQ_FP8_STATIC) g = s_x;
  CK(dqgemm_create(&h, (dqgemm_format)fmt, K, N, dp, ds, g, fmt == DQ_FP8_STATIC ? NULL : db));
  CUDA(cudaFree(dW));   /* the handle owns its own copy of the weight */
  CUDA(cudaFree(dp));
  CUDA(cudaFree(ds));
  CK(dqgemm_run(h, dx, M, dy, NULL));
  CUDA(cudaDeviceSynchronize());
  CK(dqgemm_last_error(h));
  CUDA(cudaMemcpy(y, dy, yb, cudaMemcpyDeviceToHost));
  CK(dqgemm_destroy(h));
  CUDA(cudaFree(dx));
  CUDA(cudaFree(db));
  CUDA(cudaFree(dy));
  {
    FILE* f = fopen(out, "wb");
    if (!f) return 2;
    write_all(f, y, yb);
    fclose(f);
  }
  free(W);
  free(x);
  free(b);
  free(y);
  return 0;
}
#endif

int main(int argc, char** argv) {
  if (argc >= 2 && !strcmp(argv[1], "errors")) return do_errors();
  if (argc == 7 && !strcmp(argv[1], "pack"))
    return do_pack(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), argv[5], argv[6]);
#ifdef DQ_CONSUMER_GPU
  if (argc == 11 && !strcmp(argv[1], "gemm"))
    return do_gemm(atoi(argv[2]), atoi(argv[3]), atoi(argv[4]), atoi(argv[5]), (float)atof(argv[6]),
                   argv[7], argv[8], argv[9], argv[10]);
#endif
  fprintf(stderr, "usage: see the header comment of dq_consumer.c\n");
  return 2;
}
