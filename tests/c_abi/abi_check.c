/* A plain C99 client of libgattn: compiled and run by tests/test_abi_c.py without a GPU.
 *
 * Prints the gattn_cfg layout as the C compiler sees it (checked against the Python
 * mirror), then drives calls that the library answers on the host before any launch:
 * status strings, RoPE table sizes, workspace sizes and argument validation. */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "gattn.h"

static gattn_cfg base_cfg(void) {
  gattn_cfg c;
  memset(&c, 0, sizeof(c));
  c.num_heads = 8;
  c.num_kv_heads = 1;
  c.head_dim = 256;
  c.rope_theta = 1e4f;
  c.scalar = 256.f;
  c.norm_eps = 1e-6f;
  return c;
}

int main(void) {
  printf("sizeof=%zu\n", sizeof(gattn_cfg));
  printf("offset rope_table=%zu\n", offsetof(gattn_cfg, rope_table));
  printf("offset q_norm_w=%zu\n", offsetof(gattn_cfg, q_norm_w));
  printf("offset keys_transformed=%zu\n", offsetof(gattn_cfg, keys_transformed));
  printf("version=%s\n", gattn_version());
  printf("status6=%s\n", gattn_status_string(GATTN_ERR_DEVICE_BOUNDS));
  printf("rope_bytes=%zu\n", gattn_rope_table_bytes(100, 128));
  printf("rope_bytes_bad=%zu\n", gattn_rope_table_bytes(100, 3));

  gattn_cfg c = base_cfg();
  printf("prefill_ws=%zu\n", gattn_prefill_workspace_size(&c, 2, 300));
  printf("decode_ws=%zu\n", gattn_decode_workspace_size(&c, 4, 2048));
  /* host-side rejections: no launch happens for any of these */
  void* fake = (void*)(uintptr_t)0x10000;
  int st = gattn_prefill(NULL, fake, fake, NULL, fake, 1, 16, &c, fake, 1 << 20, NULL);
  printf("prefill_null_q=%d\n", st);
  printf("last_error_set=%d\n", gattn_last_error()[0] != 0);
  c.head_dim = 128;
  st = gattn_decode(fake, fake, fake, fake, fake, 1, 16, &c, fake, 1 << 20, NULL);
  printf("decode_d128=%d\n", st);
  c = base_cfg();
  c.keys_transformed = 1;
  c.k_eq_v = 1;
  st = gattn_decode(fake, fake, NULL, fake, fake, 1, 16, &c, fake, 1 << 20, NULL);
  printf("decode_kt_keqv=%d\n", st);
  c = base_cfg();
  st = gattn_prefill(fake, fake, fake, NULL, fake, 0, 16, &c, fake, 1 << 20, NULL);
  printf("prefill_empty=%d\n", st);
  st = gattn_kv_quantize(fake, fake, fake, 4, 100, NULL);
  printf("quantize_d100=%d\n", st);
  return 0;
}
