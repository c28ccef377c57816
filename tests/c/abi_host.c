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

/* The decode layer shown in the README, compiled (never called here: it
 * needs a GPU), so that its calls keep matching the header. */
int readme_decode_layer(const void* d_k, const void* d_v, const void* d_q, const int64_t* d_qpos, uint8_t* d_kcodes,
                        uint8_t* d_ksigns, float* d_knorms, uint8_t* d_vcodes, uint8_t* d_vsigns, float* d_vnorms,
                        float* d_out, void* d_ws, int B, int Hq, int Hkv, int64_t T, void* stream);
int readme_decode_layer(const void* d_k, const void* d_v, const void* d_q, const int64_t* d_qpos, uint8_t* d_kcodes,
                        uint8_t* d_ksigns, float* d_knorms, uint8_t* d_vcodes, uint8_t* d_vsigns, float* d_vnorms,
                        float* d_out, void* d_ws, int B, int Hq, int Hkv, int64_t T, void* stream) {
  const int64_t n = (int64_t)B * Hkv * T;
  tq_rotation *hk, *hv;
  tq_build_rotation_seeded(128, 2, TQ_ROT_HADAMARD, TQ_RES_QJL, 1234, 128, 10000.0, 1 << 20, &hk);
  tq_build_rotation_seeded(128, 2, TQ_ROT_HADAMARD, TQ_RES_QJL, 1235, 128, 0.0, 0, &hv);
  tq_quantize_kv(hk, d_k, TQ_BF16, n, 128, NULL, T, 0, 1, d_kcodes, d_ksigns, d_knorms, 1, stream);
  tq_quantize_kv(hv, d_v, TQ_BF16, n, 128, NULL, T, 0, 0, d_vcodes, d_vsigns, d_vnorms, 1, stream);
  size_t ws_bytes = tq_decode_workspace_size(hk, hv, B, Hq, Hkv, T);
  int st = tq_decode_attention(hk, hv, d_q, TQ_BF16, d_qpos, d_kcodes, d_ksigns, d_knorms, d_vcodes, d_vsigns,
                               d_vnorms, T, B, Hq, Hkv, T, NULL, 0.08838835f, d_out, d_ws, ws_bytes, stream);
  tq_free_rotation(hk);
  tq_free_rotation(hv);
  return st;
}

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
