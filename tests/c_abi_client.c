/* A plain C99 client of the library's C ABI: it includes only gqa.h, links against the shared
 * library, and makes the calls that need no GPU (version, status strings, workspace sizes and the
 * host-side argument checks). Exit status 0 when every check holds. */
#include <stdio.h>

#include "gqa.h"

static int failures = 0;

static void check(int ok, const char* what) {
  if (!ok) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  char fake_storage[256];
  void* fake = fake_storage; /* never dereferenced: every call below is rejected on the host */
  printf("%s\n", gqa_version());
  check(gqa_status_string(GQA_OK) != NULL, "status string");
  check(gqa_decode_workspace_size(8, 32, 8, 8192, 128, GQA_BF16, 148) > 0, "decode workspace size");
  check(gqa_decode_workspace_size(8, 30, 8, 8192, 128, GQA_BF16, 148) == 0, "h_q % h_kv != 0");
  check(gqa_prefill_backward_workspace_size(1, 32, 4096) > 0, "backward workspace size");
  check(gqa_prefill(NULL, fake, fake, fake, NULL, NULL, NULL, 1, 4, 2, 8, 8, 64, 0.125f, 1, 0,
                    GQA_BF16, NULL) == GQA_ERR_INVALID_ARG, "prefill with a null query");
  check(gqa_prefill(fake, fake, fake, fake, NULL, NULL, NULL, 1, 4, 2, 8, 8, 96, 0.125f, 1, 0,
                    GQA_BF16, NULL) == GQA_ERR_UNSUPPORTED, "prefill with bf16 d_h = 96");
  check(gqa_decode(fake, fake, fake, fake, NULL, NULL, NULL, 1, 4, 2, 8, 64, 0.125f, 0, GQA_BF16,
                   NULL, 1 << 20, 1, NULL) == GQA_ERR_WORKSPACE, "decode without a workspace");
  check(kv_append(fake, fake, NULL, NULL, NULL, 1, 2, 0, 8, 64, GQA_BF16, NULL) == GQA_OK,
        "append of zero rows");
  check(gqa_get_device_error(NULL, NULL) == GQA_ERR_INVALID_ARG, "device error without a code");
  return failures == 0 ? 0 : 1;
}
