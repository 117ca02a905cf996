/* A plain C99 client of the C ABI: include/pa.h compiled with -std=c99
 * -pedantic -Werror and linked against libpa.so, calling the host-side
 * parts that need no GPU (version, status text, workspace sizes, argument
 * checks that return before any device work).  Built and run by
 * tests/test_abi_c.py. */
#include <stdio.h>
#include <string.h>

#include "pa.h"

static int failures = 0;
#define CHECK(c)                                                        \
  do {                                                                  \
    if (!(c)) {                                                         \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #c); \
      ++failures;                                                       \
    }                                                                   \
  } while (0)

int main(void) {
  pa_cache_desc bf16 = {1000, 16, 8, 128, PA_DTYPE_BF16, 1.0f, 1.0f};
  pa_cache_desc f32 = {1000, 16, 8, 128, PA_DTYPE_F32, 1.0f, 1.0f};
  /* FP8 pages with head_dim 64: no compiled kernel */
  pa_cache_desc fp8_d64 = {1000, 16, 8, 64, PA_DTYPE_FP8_E4M3, 0.25f, 0.5f};
  void *fake = (void *)(size_t)0x10000; /* aligned, never dereferenced */
  int32_t *ifake = (int32_t *)fake;
  size_t ws;

  CHECK(pa_version() >= 300);
  CHECK(strcmp(pa_status_string(PA_OK), "PA_OK") == 0);
  CHECK(strcmp(pa_status_string(PA_ERR_UNSUPPORTED), "PA_ERR_UNSUPPORTED") == 0);

  ws = pa_decode_workspace_bytes(&bf16, 32, 32, 128);
  CHECK(ws > 0 && ws % 256 == 0);
  CHECK(pa_decode_workspace_bytes(&bf16, 32, 31, 128) == 0); /* 31 heads on 8 KV heads */
  CHECK(pa_decode_workspace_bytes(NULL, 32, 32, 128) == 0);
  CHECK(pa_decode_shared_prefix_workspace_bytes(&bf16, 32, 32, 128, 4) >= ws);

  /* refusals before any device work */
  CHECK(pa_decode(NULL, fake, fake, fake, fake, ifake, ifake, 2, 32, 4, 0.1f, fake, ws, NULL,
                  NULL) == PA_ERR_INVALID_ARG);
  CHECK(strlen(pa_last_error_message()) > 0);
  CHECK(pa_decode_splitk(&fp8_d64, fake, fake, fake, ifake, ifake, 2, 32, 4, 0.1f, 512, 1,
                         (float *)fake, (float *)fake, (float *)fake, NULL,
                         NULL) == PA_ERR_UNSUPPORTED);
  CHECK(pa_prefill(&f32, fake, fake, fake, fake, ifake, ifake, ifake, 2, 64, 32, 16, 32, 0.1f,
                   NULL, NULL) == PA_ERR_UNSUPPORTED);
  CHECK(strstr(pa_last_error_message(), "bf16") != NULL);
  CHECK(pa_prefill(&bf16, fake, fake, fake, fake, ifake, ifake, ifake, 0, 64, 32, 16, 32, 0.1f,
                   NULL, NULL) == PA_OK); /* empty batch */
  CHECK(pa_write_kv_cache(&bf16, fake, fake, fake, fake, (const int64_t *)fake, 0, NULL,
                          NULL) == PA_OK); /* no tokens */
  CHECK(pa_reduce(fake, (const float *)fake, (const float *)fake, (const float *)fake, ifake, 0,
                  32, 128, 512, 4, PA_DTYPE_BF16, NULL, NULL) == PA_OK);
  if (failures) {
    fprintf(stderr, "%d checks failed\n", failures);
    return 1;
  }
  printf("C client: ok\n");
  return 0;
}
