/*
 * Host-side use of the C ABI from plain C (no CUDA headers, no device):
 * the header compiles as C, the library links, and the calls that need no
 * GPU answer as the header states - status strings, the version, size
 * queries of invalid requests, and argument rejections before any launch.
 * Prints "ok" and exits 0 when every check holds.
 */
#include <stdio.h>
#include <string.h>

#include "tq.h"

static int failures = 0;

#define CHECK(cond)                                                   \
  do {                                                                \
    if (!(cond)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
      ++failures;                                                     \
    }                                                                 \
  } while (0)

int main(void) {
  CHECK(tq_version() > 0);
  CHECK(tq_status_string(TQ_OK) != NULL && strlen(tq_status_string(TQ_OK)) > 0);
  CHECK(tq_status_string(TQ_EINVAL) != NULL);
  CHECK(tq_status_string(TQ_EWORKSPACE) != NULL);
  CHECK(tq_status_string(12345) != NULL);
  /* size queries of invalid requests answer 0 */
  CHECK(tq_decode_workspace_size(NULL, NULL, 1, 4, 1, 10) == 0);
  CHECK(tq_decode_window_workspace_size(NULL, NULL, 1, 4, 1, 10, 4) == 0);
  /* calls with a missing handle or buffer are rejected on the host */
  CHECK(tq_quantize_kv(NULL, NULL, TQ_F32, 1, 64, NULL, 1, 0, 0, NULL, NULL, NULL, 1, NULL) == TQ_EINVAL);
  CHECK(tq_decode_attention(NULL, NULL, NULL, TQ_F32, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 4, 1, 0, NULL,
                            0.125f, NULL, NULL, 0, NULL) == TQ_EINVAL);
  CHECK(tq_decode_attention_append(NULL, NULL, NULL, TQ_F32, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0,
                                   1, 4, 1, 1, NULL, 0.125f, NULL, NULL, 0, NULL) == TQ_EINVAL);
  CHECK(tq_decode_attention_nsn_append(NULL, NULL, NULL, TQ_F32, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                                       NULL, NULL, NULL, NULL, NULL, 4, 1, 4, 1, 1, NULL, 0.125f, NULL, NULL, 0,
                                       NULL) == TQ_EINVAL);
  CHECK(tq_free_rotation(NULL) == TQ_OK);   /* NULL is accepted */
  if (failures) return 1;
  printf("ok\n");
  return 0;
}
