/*
 * A C caller of the library: the QSA layer for one prefill from host buffers through the C ABI
 * (include/qsa.h) alone, no Python.  The caller owns all memory: page-locked host buffers for the
 * inputs and the output, and one device scratch buffer of qsa_prefill_host_device_bytes().
 *
 *   prefill_host check           host-side calls only (no GPU needed): version, sizes, refusals
 *   prefill_host run DIR T SEED  a T-token prefill (16 q / 2 KV heads, D 128, 4 x 64 indexer,
 *                                k 512) on synthetic inputs; writes DIR/{q,k,v,qi,ki,out}.bin
 *
 * Build: gcc -std=c11 -I include -I $CUDA/include prefill_host.c -L <lib dir> -lqsa_b200
 *        -L $CUDA/lib64 -lcudart -Wl,-rpath,<lib dir>
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "qsa.h"

enum { HQ = 16, HKV = 2, D = 128, HI = 4, DI = 64, K = 512, BLK = 4 };

static int fail(const char* what, int code) {
  fprintf(stderr, "%s: %d\n", what, code);
  return 1;
}

/* bf16 bits of x (round to nearest even), for the synthetic inputs */
static uint16_t to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* a 64-bit LCG drawing values uniform in [-a, a) */
static uint64_t g_state;
static float draw(float a) {
  g_state = g_state * 6364136223846793005ull + 1442695040888963407ull;
  return a * ((float)(g_state >> 40) / 8388608.0f - 1.0f);
}

static int fill(uint16_t* p, size_t n, float a) {
  for (size_t i = 0; i < n; ++i) p[i] = to_bf16(draw(a));
  return 0;
}

static int save(const char* dir, const char* name, const void* p, size_t bytes) {
  char path[4096];
  snprintf(path, sizeof path, "%s/%s.bin", dir, name);
  FILE* f = fopen(path, "wb");
  if (!f) return 1;
  const size_t w = fwrite(p, 1, bytes, f);
  fclose(f);
  return w != bytes;
}

static int check(void) {
  if (qsa_abi_version() != QSA_ABI_VERSION) return fail("abi version", qsa_abi_version());
  const size_t need = qsa_prefill_host_device_bytes(1, 4096, 4096, HQ, HKV, D, HI, DI, K, BLK, 0, 0, 0, 2);
  if (need == 0) return fail("device bytes", 0);
  if (qsa_prefill_host_device_bytes(1, 4096, 100, HQ, HKV, D, HI, DI, K, BLK, 0, 0, 0, 2) != 0)
    return fail("device bytes of an invalid shape", 1);
  char dummy[16];
  /* refusals happen on the host, before anything is enqueued */
  qsa_status_t st = qsa_prefill_host(NULL, dummy, dummy, dummy, dummy, dummy, 1, 64, 64, HQ, HKV, D, HI, DI, 8, BLK, 0,
                                     0.1f, QSA_SCORE_RELU_SUM, NULL, NULL, 0, 1, (void*)(uintptr_t)4096, need, NULL,
                                     NULL, NULL);
  if (st != QSA_ERR_INVALID_ARGUMENT) return fail("null input accepted", st);
  st = qsa_prefill_host(dummy, dummy, dummy, dummy, dummy, dummy, 1, 64, 64, HQ, HKV, D, HI, DI, 8, BLK, 0, 0.1f,
                        QSA_SCORE_RELU_SUM, NULL, NULL, 0, 1, (void*)(uintptr_t)4096, 16, NULL, NULL, NULL);
  if (st != QSA_ERR_WORKSPACE_TOO_SMALL) return fail("small scratch accepted", st);
  printf("check ok: abi %d, %zu device bytes for a 4096-token prefill\n", qsa_abi_version(), need);
  return 0;
}

static int run(const char* dir, int T, unsigned long long seed) {
  g_state = seed;
  const size_t nq = (size_t)T * HQ * D, nk = (size_t)T * HKV * D, nqi = (size_t)T * HI * DI, nki = (size_t)T * DI;
  uint16_t *q, *k, *v, *qi, *ki, *out;
  if (cudaMallocHost((void**)&q, nq * 2) || cudaMallocHost((void**)&k, nk * 2) || cudaMallocHost((void**)&v, nk * 2) ||
      cudaMallocHost((void**)&qi, nqi * 2) || cudaMallocHost((void**)&ki, nki * 2) ||
      cudaMallocHost((void**)&out, nq * 2))
    return fail("cudaMallocHost", 0);
  fill(q, nq, 0.15f);
  fill(k, nk, 0.15f);
  fill(v, nk, 0.15f);
  fill(qi, nqi, 0.2f);
  fill(ki, nki, 0.2f);
  const size_t need = qsa_prefill_host_device_bytes(1, T, T, HQ, HKV, D, HI, DI, K, BLK, 0, 0, 0, 2);
  void* dev = NULL;
  if (need == 0 || cudaMalloc(&dev, need)) return fail("device scratch", (int)(need == 0));
  cudaStream_t s;
  if (cudaStreamCreate(&s)) return fail("stream", 0);
  qsa_status_t st = qsa_prefill_host(q, k, v, qi, ki, out, 1, T, T, HQ, HKV, D, HI, DI, K, BLK, 0, 1.0f / sqrtf((float)D),
                                     QSA_SCORE_RELU_SUM, NULL, NULL, 0, 2, dev, need, NULL, NULL, s);
  if (st != QSA_OK) return fail("qsa_prefill_host", st);
  if (cudaStreamSynchronize(s)) return fail("synchronize", 0);
  st = qsa_get_device_status(s);
  if (st != QSA_OK) return fail("device status", st);
  size_t bad = 0;
  for (size_t i = 0; i < nq; ++i) bad += (out[i] & 0x7F80u) == 0x7F80u;   /* inf or NaN */
  if (bad) return fail("non-finite outputs", (int)bad);
  if (save(dir, "q", q, nq * 2) || save(dir, "k", k, nk * 2) || save(dir, "v", v, nk * 2) ||
      save(dir, "qi", qi, nqi * 2) || save(dir, "ki", ki, nki * 2) || save(dir, "out", out, nq * 2))
    return fail("write", 0);
  printf("run ok: %d tokens, %zu device bytes\n", T, need);
  cudaFree(dev);
  cudaStreamDestroy(s);
  return 0;
}

int main(int argc, char** argv) {
  if (argc >= 2 && strcmp(argv[1], "check") == 0) return check();
  if (argc >= 5 && strcmp(argv[1], "run") == 0) return run(argv[2], atoi(argv[3]), strtoull(argv[4], NULL, 10));
  fprintf(stderr, "usage: %s check | run DIR T SEED\n", argv[0]);
  return 2;
}
