/* A C99 caller of libnwc's device entry points, built and run by
 * tests/test_c_abi_gpu.py on a GPU: the caller owns the device memory (here
 * from the CUDA runtime), and compress, decompress and GEMV run through the C
 * ABI alone.
 *
 * Usage: c_abi_device OUT_PREFIX
 * Matrix: 300 x 1000 BF16 patterns w[i][j] = 0x3C00 + (37 i + 11 j) % 1024,
 * x: 40 x 1000 patterns 0x3F80 + (i + 3 j) % 64 (values near 1).  Writes
 * OUT_PREFIX.w (the decompressed matrix), OUT_PREFIX.y1 (y for the first 3
 * rows of x, CUDA-core kernel) and OUT_PREFIX.y40 (all 40 rows, tensor-core
 * kernel), and prints one "key value" line per checked quantity. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "nwc.h"

/* The three CUDA runtime calls this caller needs, by their C signatures (the
 * runtime's own header is not strict C99); error codes are ints, 0 = success. */
extern int cudaMalloc(void** ptr, size_t bytes);
extern int cudaFree(void* ptr);
extern int cudaMemcpy(void* dst, const void* src, size_t bytes, int kind);
enum { cudaMemcpyHostToDevice = 1, cudaMemcpyDeviceToHost = 2 };

#define ROWS 300
#define COLS 1000
#define BATCH 40

static int fail(const char* what, nwc_status st) {
  fprintf(stderr, "%s: %s\n", what, nwc_status_string(st));
  return 1;
}

static int dump(const char* prefix, const char* ext, const void* p, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s.%s", prefix, ext);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(p, 1, bytes, f) != bytes) return 1;
  fclose(f);
  return 0;
}

int main(int argc, char** argv) {
  if (argc != 2) return 2;
  static uint16_t w[ROWS * COLS], x[BATCH * COLS], back[ROWS * COLS];
  static float y[BATCH * ROWS];
  for (int i = 0; i < ROWS; ++i)
    for (int j = 0; j < COLS; ++j) w[i * COLS + j] = (uint16_t)(0x3C00 + (37 * i + 11 * j) % 1024);
  for (int i = 0; i < BATCH; ++i)
    for (int j = 0; j < COLS; ++j) x[i * COLS + j] = (uint16_t)(0x3F80 + (i + 3 * j) % 64);

  nwc_plan_t plan = NULL;
  nwc_status st = nwc_plan(w, ROWS, COLS, NULL, &plan);
  if (st != NWC_OK) return fail("nwc_plan", st);
  uint64_t dev_bytes = 0, blob_bytes = 0;
  if ((st = nwc_plan_size(plan, &dev_bytes, &blob_bytes)) != NWC_OK) return fail("size", st);
  void *d_img = NULL, *d_w = NULL, *d_x = NULL, *d_y = NULL;
  if (cudaMalloc(&d_img, dev_bytes) || cudaMalloc(&d_w, sizeof w) || cudaMalloc(&d_x, sizeof x) ||
      cudaMalloc(&d_y, sizeof y))
    return 3;
  nwc_handle_t h = NULL;
  st = nwc_compress(plan, w, d_img, dev_bytes, NULL, &h);
  nwc_plan_destroy(plan);
  if (st != NWC_OK) return fail("nwc_compress", st);
  if (cudaMemcpy(d_x, x, sizeof x, cudaMemcpyHostToDevice)) return 3;

  if ((st = nwc_decompress(h, (uint16_t*)d_w, NULL)) != NWC_OK) return fail("decompress", st);
  if (cudaMemcpy(back, d_w, sizeof back, cudaMemcpyDeviceToHost)) return 3;
  if (dump(argv[1], "w", back, sizeof back)) return 1;

  int32_t launches = 0, tc = 0;
  nwc_gemv_path(h, (const uint16_t*)d_x, 3, &launches, &tc);
  printf("b3_launches %d\nb3_tensor_cores %d\n", launches, tc);
  if ((st = nwc_gemv(h, (const uint16_t*)d_x, (float*)d_y, 3, NULL)) != NWC_OK)
    return fail("gemv 3", st);
  if (cudaMemcpy(y, d_y, 3 * ROWS * sizeof(float), cudaMemcpyDeviceToHost)) return 3;
  if (dump(argv[1], "y1", y, 3 * ROWS * sizeof(float))) return 1;

  nwc_gemv_path(h, (const uint16_t*)d_x, BATCH, &launches, &tc);
  printf("b40_launches %d\nb40_tensor_cores %d\n", launches, tc);
  if ((st = nwc_gemv(h, (const uint16_t*)d_x, (float*)d_y, BATCH, NULL)) != NWC_OK)
    return fail("gemv 40", st);
  if (cudaMemcpy(y, d_y, sizeof y, cudaMemcpyDeviceToHost)) return 3;
  if (dump(argv[1], "y40", y, sizeof y)) return 1;

  uint32_t word = 0;
  printf("device_error %d\nword %u\n", (int)nwc_get_device_error(h, NULL, &word), word);
  printf("bad_batch %d\n", (int)nwc_gemv(h, (const uint16_t*)d_x, (float*)d_y, 65, NULL));
  nwc_handle_destroy(h);
  cudaFree(d_img);
  cudaFree(d_w);
  cudaFree(d_x);
  cudaFree(d_y);
  return 0;
}
