/* Plain C client (C11: the CUDA runtime headers use anonymous unions) of the whole path through
 * libmla.so: create a cache, fill the window, run the attention call for a query chunk, make
 * the chunk part of the window (mla_cache_append of its hidden states, or mla_cache_commit of
 * the latents the attention call computed), and read the status word, with device buffers from
 * the CUDA runtime.  tests/test_c_abi.py compiles and links it without a GPU; on a GPU
 * (tests/test_gpu_c_client.py) it runs as a rollout of a few frames of a small layer and exits
 * 0 when every call succeeded and the outputs are finite.  Inputs are seeded uniform values in
 * [-1, 1) (weights scaled by 1/sqrt(fan_in)), converted to bf16 on the host.  With a directory
 * argument it also writes every input and output there as raw bf16 (w_*.bin, x<frame>.bin,
 * out<frame>.bin), so that a test can replay the rollout in the fp64 oracle. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "mla.h"

static uint32_t g_state = 12345u;
static float uniform(void) { /* xorshift32 in [-1, 1) */
  g_state ^= g_state << 13;
  g_state ^= g_state >> 17;
  g_state ^= g_state << 5;
  return (float)(g_state >> 8) / 8388608.0f - 1.0f;
}

static uint16_t to_bf16(float f) { /* round to nearest even */
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static float from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static const char* g_dump_dir = NULL;

/* Write n bf16 values to <g_dump_dir>/<name>.bin (nothing without a directory). */
static int dump(const char* name, const uint16_t* v, size_t n) {
  char path[4096];
  FILE* f;
  if (!g_dump_dir) return 0;
  snprintf(path, sizeof path, "%s/%s.bin", g_dump_dir, name);
  f = fopen(path, "wb");
  if (!f) return 1;
  if (fwrite(v, 2, n, f) != n) {
    fclose(f);
    return 1;
  }
  return fclose(f) != 0;
}

static void* device_random(size_t n, float scale, const char* name) {
  uint16_t* host = (uint16_t*)malloc(n * 2);
  void* dev = NULL;
  if (!host) return NULL;
  for (size_t i = 0; i < n; ++i) host[i] = to_bf16(scale * uniform());
  if (dump(name, host, n) != 0 || cudaMalloc(&dev, n * 2) != cudaSuccess ||
      cudaMemcpy(dev, host, n * 2, cudaMemcpyHostToDevice) != cudaSuccess)
    dev = NULL;
  free(host);
  return dev;
}

#define CHECK(call)                                                                      \
  do {                                                                                   \
    mla_status s_ = (call);                                                              \
    if (s_ != MLA_OK) {                                                                  \
      fprintf(stderr, "%s: %s: %s\n", #call, mla_status_string(s_), mla_last_error());   \
      return 1;                                                                          \
    }                                                                                    \
  } while (0)

int main(int argc, char** argv) {
  mla_config c;
  if (argc > 1) g_dump_dir = argv[1];
  memset(&c, 0, sizeof c);
  c.hidden = 1536;
  c.n_heads = 12;
  c.d_head = 128;
  c.d_nope = 128;
  c.d_latent = 192;
  c.d_rope = 32;
  c.rope_t = 8;
  c.rope_h = 12;
  c.rope_w = 12;
  c.rope_base = 10000.0;
  c.frame_h = 4;
  c.frame_w = 6;
  c.window_frames = 2;
  c.max_chunk_frames = 1;
  c.batch = 1;
  CHECK(mla_config_check(&c));

  const size_t d = 1536, F = 24, nh = 12;
  const float s_in = 1.0f / sqrtf((float)d);
  mla_weights w;
  memset(&w, 0, sizeof w);
  w.w_q = device_random(nh * 128 * d, s_in, "w_q");
  w.w_qr = device_random(nh * 32 * d, s_in, "w_qr");
  w.w_dkv = device_random(192 * d, s_in, "w_dkv");
  w.w_kr = device_random(32 * d, s_in, "w_kr");
  w.w_uk = device_random(nh * 128 * 192, 1.0f / sqrtf(192.0f), "w_uk");
  w.w_uv = device_random(nh * 128 * 192, 1.0f / sqrtf(192.0f), "w_uv");
  w.w_o = device_random(d * nh * 128, 1.0f / sqrtf((float)(nh * 128)), "w_o");
  if (!w.w_q || !w.w_qr || !w.w_dkv || !w.w_kr || !w.w_uk || !w.w_uv || !w.w_o) {
    fprintf(stderr, "no device memory (is there a GPU?)\n");
    return 2;
  }

  mla_cache* cache = NULL;
  CHECK(mla_cache_create(&c, &w, NULL, &cache));
  /* create has synchronised and keeps its own derived weights: the caller's may go */
  cudaFree((void*)w.w_q);
  cudaFree((void*)w.w_qr);
  cudaFree((void*)w.w_dkv);
  cudaFree((void*)w.w_kr);
  cudaFree((void*)w.w_uk);
  cudaFree((void*)w.w_uv);
  cudaFree((void*)w.w_o);

  void* out = NULL;
  if (cudaMalloc(&out, F * d * 2) != cudaSuccess) return 2;
  uint16_t* host_out = (uint16_t*)malloc(F * d * 2);
  if (!host_out) return 2;
  int bad = 0;
  for (int frame = 0; frame < 5; ++frame) {
    char name[32];
    snprintf(name, sizeof name, "x%d", frame);
    void* x = device_random(F * d, 1.0f, name);
    if (!x) return 2;
    if (frame > 0) {   /* the chunk attends to the window, then joins it */
      CHECK(mla_window_attention(cache, x, 1, out, NULL));
      CHECK(mla_cache_sync(cache, NULL));
      if (cudaMemcpy(host_out, out, F * d * 2, cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
      for (size_t i = 0; i < F * d; ++i) bad += !isfinite(from_bf16(host_out[i]));
      snprintf(name, sizeof name, "out%d", frame);
      if (dump(name, host_out, F * d) != 0) return 2;
    }
    if (frame % 2)
      CHECK(mla_cache_commit(cache, 1, NULL));   /* the latents the attention call computed */
    else
      CHECK(mla_cache_append(cache, x, 1, NULL));
    CHECK(mla_cache_sync(cache, NULL));   /* x is the caller's until the append has run */
    cudaFree(x);
  }
  int64_t appended = 0;
  int32_t valid = 0;
  CHECK(mla_cache_state(cache, &appended, &valid));
  CHECK(mla_cache_sync(cache, NULL));
  mla_cache_destroy(cache);
  cudaFree(out);
  free(host_out);
  printf("frames_appended %lld valid_frames %d non_finite %d\n", (long long)appended, (int)valid, bad);
  return (appended == 5 && valid == 2 && bad == 0) ? 0 : 1;
}
