/* Plain C11 client of the library's C ABI (include/qstate.h): checks that
 * the header compiles as C and that the GPU-free paths behave as declared
 * (size queries, status strings, argument validation before any launch).
 * Prints one line per check; exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "qstate.h"

static int failures = 0;

static void check(int ok, const char* what) {
  printf("%s %s\n", ok ? "ok  " : "FAIL", what);
  if (!ok) ++failures;
}

int main(void) {
  qs_config c = {1024, 128, 128, 4, 32, 1, QS_DECAY_SCALAR, QS_SCALE_DYNAMIC, QS_ROUND_NEAREST};
  size_t codes = 0, scales = 0, shadow = 0;
  check(qstate_query_sizes(&c, &codes, &scales, &shadow) == QS_OK, "query_sizes accepts a valid config");
  check(codes == (size_t)1024 * 128 * 128 / 2, "INT4 codes: Dv*Dk/2 bytes per tile");
  check(scales == (size_t)1024 * 128 * (128 / 32) * 4, "scales: one float per row and group");
  check(shadow == 0, "no shadow outside the yoked policy");

  qs_config y = c;
  y.policy = QS_SCALE_YOKED;
  check(qstate_query_sizes(&y, &codes, &scales, &shadow) == QS_OK && shadow == (size_t)1024 * 128 * 128 * 4,
        "yoked: an FP32 shadow of the state");

  qs_config bad = c;
  bad.bits = 5;
  check(qstate_query_sizes(&bad, &codes, &scales, &shadow) != QS_OK, "unsupported bit width rejected");
  check(qstate_query_sizes(NULL, &codes, &scales, &shadow) == QS_ERR_INVALID_ARG, "NULL config rejected");

  check(qstate_decode_step(&c, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) ==
            QS_ERR_INVALID_ARG,
        "decode_step rejects NULL buffers before any launch");
  check(qstate_readout(&c, NULL, NULL, NULL, NULL, NULL) == QS_ERR_INVALID_ARG,
        "readout rejects NULL buffers before any launch");

  qs_config pf = c;
  pf.delta = 1;
  check(qstate_prefill_tf32(&pf, 8, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) == QS_ERR_UNSUPPORTED,
        "tensor-core prefill rejects the delta rule");

  unsigned int timed_out = 0;
  check(qstate_prefill_tf32_wait_selfcheck(0, &timed_out) == QS_ERR_INVALID_ARG,
        "wait self-check rejects a zero poll limit before any launch");

  size_t in_b = 0, out_b = 0;
  check(qstate_pipeline_query_sizes(&c, 3, &in_b, &out_b) == QS_OK && out_b == (size_t)3 * 1024 * 128 * 4 &&
            in_b == (size_t)1024 * (128 + 128 + 128 + 1 + 1) * 4,
        "pipeline sizes");
  qs_pipeline* pl = NULL;
  check(qstate_pipeline_create(0, &c, 3, &pl) == QS_ERR_INVALID_ARG && pl == NULL,
        "pipeline rejects zero families before any CUDA call");
  check(qstate_pipeline_create(1, &c, 1, &pl) == QS_ERR_INVALID_ARG,
        "pipeline rejects a depth below 2");
  check(qstate_pipeline_step(NULL, NULL, NULL, NULL, NULL, NULL, 0) == QS_ERR_INVALID_ARG,
        "pipeline step rejects a NULL pipeline");
  check(qstate_pipeline_destroy(NULL) == QS_OK, "destroying NULL is a no-op");

  const char* s = qstate_status_string(QS_OK);
  check(s != NULL && strlen(s) > 0, "status strings are defined");
  check(qstate_version() > 0, "version is positive");
  return failures == 0 ? 0 : 1;
}
