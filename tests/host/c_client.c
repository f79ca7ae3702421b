/* A plain C11 client of libkv2 (include/kv2.h), built with -pedantic -Werror
 * and run by tests/test_abi.py: the header is C, the library links from C,
 * and the calls that return before any device work behave as documented.
 * Only fake (never dereferenced) device pointers are used. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kv2.h"

static int failures = 0;
#define EXPECT(cond)                                               \
  do {                                                             \
    if (!(cond)) {                                                 \
      fprintf(stderr, "line %d: %s (%s)\n", __LINE__, #cond, kv2_last_error()); \
      ++failures;                                                  \
    }                                                              \
  } while (0)

static void* fake(uintptr_t a) { return (void*)a; }

static kv2_cache paged_cache(void) {
  kv2_cache c;
  memset(&c, 0, sizeof c);
  c.B = 1; c.H_kv = 2; c.d = 128; c.M = 64; c.r = 8; c.capacity = 256;
  c.k_code = (uint32_t*)fake(0x1000); c.v_code = (uint32_t*)fake(0x2000);
  c.k_sz = (uint32_t*)fake(0x3000); c.v_sz = (uint32_t*)fake(0x4000);
  c.cidx = fake(0x5000); c.psac = (uint16_t*)fake(0x6000);
  c.centroids = (const uint16_t*)fake(0x7000); c.P = (const float*)fake(0x8000);
  c.w = (const float*)fake(0x9000); c.Wg = (const float*)fake(0xA000);
  c.block_table = (const int32_t*)fake(0xB000); c.page_tokens = 128;
  return c;
}

int main(void) {
  kv2_cache c = paged_cache();
  EXPECT(kv2_version() >= 200);
  EXPECT(strcmp(kv2_status_string(KV2_ERR_CAPACITY), "KV2_ERR_CAPACITY") == 0);
  /* NULL descriptor, capacity overflow, unsupported group */
  EXPECT(kv2_quantize_append(NULL, NULL, NULL, 1, 0, 1, NULL) == KV2_ERR_INVALID_ARG);
  EXPECT(strlen(kv2_last_error()) > 0);
  EXPECT(kv2_quantize_append(&c, fake(0xC000), fake(0xD000), 10, 250, 1, NULL) == KV2_ERR_CAPACITY);
  c.group = 48;
  EXPECT(kv2_quantize_append(&c, fake(0xC000), fake(0xD000), 1, 0, 1, NULL) == KV2_ERR_UNSUPPORTED);
  c.group = 0;
  /* a page image: 2 heads x 128 tokens x (32+32+16+16+1+16) bytes */
  EXPECT(kv2_page_bytes(&c) == (size_t)2 * 128 * 113);
  EXPECT(kv2_page_store(&c, 3, 2, fake(0xE000), NULL) == KV2_ERR_INVALID_ARG);
  /* workspace queries are pure host arithmetic */
  EXPECT(kv2_top1_workspace_size(2, 3, 4, 5000) == (size_t)2 * 3 * 4 * 2 * 8);
  EXPECT(kv2_fit_workspace_size(2, 128) == (size_t)2 * 2 * 128 * 128 * 8);
  EXPECT(kv2_fit_workspace_size(2, 96) == 0);
  if (failures == 0) printf("c client ok\n");
  return failures ? 1 : 0;
}
