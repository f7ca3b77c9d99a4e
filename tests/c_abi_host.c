/* A C99 caller of libnwc's host-only entry points, built and run by
 * tests/test_c_abi.py: the header must compile as strict C, and a C program
 * must be able to plan, encode and inspect a matrix through the ABI alone.
 *
 * Usage: c_abi_host OUT_PREFIX
 * Writes OUT_PREFIX.nwb1 (prefix code), OUT_PREFIX.nwr1 (ranked unary code)
 * and OUT_PREFIX.nwe1 (verbatim runs for rare exponents) for the 24 x 200 matrix w[i][j] = 0x3C00 + (37 i + 11 j) % 1024 (BF16 bit
 * patterns), and prints one "key value" line per checked quantity. */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "nwc.h"

#define ROWS 24
#define COLS 200

static int fail(const char* what, nwc_status st) {
  fprintf(stderr, "%s: %s\n", what, nwc_status_string(st));
  return 1;
}

static int encode(const uint16_t* w, const nwc_opts* opts, const char* path,
                  uint64_t* device_bytes) {
  nwc_plan_t plan = NULL;
  nwc_status st = nwc_plan(w, ROWS, COLS, opts, &plan);
  if (st != NWC_OK) return fail("nwc_plan", st);
  uint64_t dev = 0, host = 0;
  st = nwc_plan_size(plan, &dev, &host);
  if (st != NWC_OK) return fail("nwc_plan_size", st);
  uint8_t* blob = (uint8_t*)malloc((size_t)host);
  if (!blob) return 1;
  st = nwc_compress_host(plan, w, blob, host);
  nwc_plan_destroy(plan);
  if (st != NWC_OK) return fail("nwc_compress_host", st);
  FILE* f = fopen(path, "wb");
  if (!f || fwrite(blob, 1, (size_t)host, f) != (size_t)host) return 1;
  fclose(f);
  free(blob);
  *device_bytes = dev;
  return 0;
}

int main(int argc, char** argv) {
  if (argc != 2) return 2;
  static uint16_t w[ROWS * COLS];
  for (int i = 0; i < ROWS; ++i)
    for (int j = 0; j < COLS; ++j) w[i * COLS + j] = (uint16_t)(0x3C00 + (37 * i + 11 * j) % 1024);
  char path[4096];

  /* Prefix code with the defaults (opts = NULL). */
  uint64_t dev = 0;
  snprintf(path, sizeof path, "%s.nwb1", argv[1]);
  if (encode(w, NULL, path, &dev)) return 1;
  printf("nwb1_device_bytes %llu\n", (unsigned long long)dev);

  /* Read the blob back: device bytes and the launch schedule for a B200. */
  FILE* f = fopen(path, "rb");
  if (!f) return 1;
  fseek(f, 0, SEEK_END);
  const long n = ftell(f);
  fseek(f, 0, SEEK_SET);
  uint8_t* blob = (uint8_t*)malloc((size_t)n);
  if (!blob || fread(blob, 1, (size_t)n, f) != (size_t)n) return 1;
  fclose(f);
  uint64_t dev2 = 0;
  nwc_status st = nwc_blob_device_bytes(blob, (uint64_t)n, &dev2);
  if (st != NWC_OK) return fail("nwc_blob_device_bytes", st);
  printf("blob_device_bytes %llu\n", (unsigned long long)dev2);
  nwc_schedule_info info;
  memset(&info, 0, sizeof info);
  info.struct_size = sizeof info;
  st = nwc_schedule_describe(blob, (uint64_t)n, 148, 232448, 1, &info, NULL, NULL, NULL);
  if (st != NWC_OK) return fail("nwc_schedule_describe", st);
  printf("schedule_tiles %llu\n", (unsigned long long)info.tiles);
  printf("schedule_ctas %d\n", (int)info.ctas);
  blob[0] ^= 1; /* no longer a blob */
  printf("corrupt_status %d\n", (int)nwc_blob_device_bytes(blob, (uint64_t)n, &dev2));
  free(blob);

  /* The ranked unary code through the options struct. */
  nwc_opts opts;
  memset(&opts, 0, sizeof opts);
  opts.struct_size = sizeof opts;
  opts.tile_rows = 8;
  opts.tile_cols = 64;
  opts.lmax = 3;
  opts.threads = 2;
  opts.code = NWC_CODE_RANK;
  snprintf(path, sizeof path, "%s.nwr1", argv[1]);
  if (encode(w, &opts, path, &dev)) return 1;
  printf("nwr1_device_bytes %llu\n", (unsigned long long)dev);

  /* Verbatim runs for rare exponents: 4 kept exponents, 128-column tiles. */
  memset(&opts, 0, sizeof opts);
  opts.struct_size = sizeof opts;
  opts.tile_rows = 8;
  opts.tile_cols = 128;
  opts.threads = 2;
  opts.code = NWC_CODE_ESCAPE;
  opts.keep = 4;
  snprintf(path, sizeof path, "%s.nwe1", argv[1]);
  if (encode(w, &opts, path, &dev)) return 1;
  printf("nwe1_device_bytes %llu\n", (unsigned long long)dev);

  /* Argument errors come back as status codes. */
  nwc_plan_t plan = NULL;
  printf("null_matrix_status %d\n", (int)nwc_plan(NULL, ROWS, COLS, NULL, &plan));
  for (int s = 0; s <= 8; ++s)
    if (!nwc_status_string((nwc_status)s)) return 1;
  printf("version %d\n", nwc_version());
  return 0;
}
