/* Plain C99 client of libmla.so's host-only calls (no GPU needed): compiled and run by
 * tests/test_c_abi.py, which checks every printed value against the Python binding and the
 * oracle's definitions.  It proves that include/mla.h is a C header and that the calls work
 * through the C ABI alone.  Output: one "key value" pair per line. */
#include <stdio.h>
#include <string.h>

#include "mla.h"

static mla_config wan_config(int32_t sink_frames) {
  mla_config c;
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
  c.frame_h = 30;
  c.frame_w = 52;
  c.window_frames = 21;
  c.max_chunk_frames = 3;
  c.batch = 1;
  c.softmax_scale = 0.0f;
  c.d_q = 0;
  c.sink_frames = sink_frames;
  return c;
}

int main(void) {
  mla_config c = wan_config(0);
  printf("check_wan %d\n", (int)mla_config_check(&c));

  mla_config odd = wan_config(0);
  odd.rope_t = 7;
  odd.rope_h = 13;
  printf("check_odd_rope %d\n", (int)mla_config_check(&odd));

  mla_config narrow = wan_config(0);
  narrow.d_latent = 128;
  printf("check_latent_128 %d\n", (int)mla_config_check(&narrow));

  printf("check_null %d\n", (int)mla_config_check(NULL));

  printf("ring_bytes %llu\n", (unsigned long long)mla_ring_bytes(&c));
  printf("device_bytes %llu\n", (unsigned long long)mla_cache_device_bytes(&c));

  static const int64_t frames[] = {0, 1, 20, 21, 22, 41, 42, 1000003};
  static const int32_t tokens[] = {0, 1, 777, 1559};
  for (int s = 0; s <= 1; ++s) {
    mla_config cs = wan_config(s);
    for (size_t i = 0; i < sizeof frames / sizeof frames[0]; ++i)
      for (size_t k = 0; k < sizeof tokens / sizeof tokens[0]; ++k) {
        int64_t slot = -1;
        const mla_status st = mla_ring_slot(&cs, frames[i], tokens[k], &slot);
        printf("slot_%d_%lld_%d %d %lld\n", s, (long long)frames[i], (int)tokens[k], (int)st,
               (long long)slot);
      }
  }

  int64_t slot = -1;
  const mla_status bad = mla_ring_slot(&c, 3, 1560, &slot);
  const char* msg = mla_last_error();
  printf("slot_bad_token %d %d\n", (int)bad, msg != NULL && strlen(msg) > 0);

  printf("status_name_0 %s\n", mla_status_string(MLA_OK));
  printf("status_name_5 %s\n", mla_status_string(MLA_ERR_DEVICE_TIMEOUT));
  return 0;
}
