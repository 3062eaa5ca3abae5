/* A plain C caller of the library: includes only tq.h, links libtq.so, and exercises the
 * host-side calls (no GPU needed).  Prints one line per check; exits non-zero on the first
 * failure.  Built and run by tests/test_abi.py. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "tq.h"

#define CHECK(cond, what)                              \
  do {                                                 \
    if (!(cond)) {                                     \
      printf("FAIL %s\n", what);                       \
      return 1;                                        \
    }                                                  \
    printf("ok %s\n", what);                           \
  } while (0)

int main(void) {
  CHECK(tq_version() >= 100, "version");
  CHECK(strcmp(tq_status_str(TQ_ERR_BOUNDS), "TQ_ERR_BOUNDS") == 0, "status string");

  /* the host copy of a dev_status word, decoded */
  int32_t word = 0;
  CHECK(tq_check(&word) == TQ_OK, "tq_check of a clear word");
  word = TQ_ERR_TIMEOUT;
  CHECK(tq_check(&word) == TQ_ERR_TIMEOUT && strlen(tq_last_error()) > 0, "tq_check of a timeout");
  word = 99;
  CHECK(tq_check(&word) == TQ_ERR_INVALID_ARG, "tq_check of a value that is no status");
  CHECK(tq_check(NULL) == TQ_ERR_INVALID_ARG, "tq_check of NULL");

  tq_config cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.head_dim = 128;
  cfg.key_bits = 3;
  cfg.key_qjl = 1;
  cfg.qjl_m = 128;
  cfg.value_bits = 3;
  cfg.page_tokens = 256;
  cfg.rotation = TQ_ROT_HADAMARD;
  cfg.value_qjl = 0;
  cfg.dither = 0;
  cfg.key_corrected_norm = 0;
  CHECK(tq_validate_config(&cfg) == TQ_OK, "validate config");
  /* KN, KR, VN 512 B each, merged key nibbles 64 * 256 B, 3-bit values 48 * 256 B */
  CHECK(tq_page_bytes(&cfg) == 3 * 512 + 64 * 256 + 48 * 256, "page bytes");
  cfg.value_qjl = 1;
  CHECK(tq_page_bytes(&cfg) == 3 * 512 + 64 * 256 + 48 * 256 + 16 * 256 + 512, "page bytes, values with QJL");
  cfg.value_qjl = 0;
  cfg.dither = 1;
  CHECK(tq_page_bytes(&cfg) == 3 * 512 + 64 * 256 + 48 * 256 + 2 * 512, "page bytes, dithered");
  cfg.dither = 0;
  CHECK(tq_operand_bytes(&cfg) == 3 * 128 * 128 * 2, "operand bytes");
  CHECK(tq_decode_workspace_bytes(&cfg, 1, 32, 1, 16) > 0, "workspace bytes");

  /* 1-bit Beta codebook at d = 128: +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2)) */
  float c[2], b[1];
  CHECK(tq_codebook(1, 128, TQ_DENSITY_BETA, c, b) == TQ_OK, "codebook call");
  const double e_abs = exp(lgamma(64.0) - lgamma(64.5)) / sqrt(acos(-1.0));
  CHECK(fabs(c[1] - e_abs) < 1e-6 && c[0] == -c[1] && b[0] == 0.0f, "1-bit Beta centroids");

  /* the dithered quantizer's grid: uniform, symmetric, middle boundary 0 */
  float dc[8], db[7];
  CHECK(tq_dither_codebook(3, 128, TQ_DENSITY_BETA, dc, db) == TQ_OK, "dither codebook call");
  CHECK(dc[0] == -dc[7] && db[3] == 0.0f && fabs((dc[2] - dc[1]) - (dc[1] - dc[0])) < 1e-6, "dither grid");

  /* host-side argument errors are returned, nothing is enqueued, the detail is kept */
  CHECK(tq_compress_kv(&cfg, NULL, NULL, 0, NULL, NULL, TQ_F16, 16, NULL, NULL, NULL) == TQ_ERR_INVALID_ARG,
        "null arguments rejected");
  CHECK(strlen(tq_last_error()) > 0, "last error detail");
  cfg.head_dim = 96;
  CHECK(tq_validate_config(&cfg) == TQ_ERR_UNSUPPORTED && tq_page_bytes(&cfg) == 0, "unsupported head_dim");
  return 0;
}
