/* The C ABI used from plain C11: the headers compile as C, and the host-only
 * entry points (weight layout size, DP schedule, error text) run without a
 * GPU.  Prints "<weights_bytes> <n_batches> <batch ids...>" on success. */
#include <stdio.h>
#include <string.h>

#include "rm.h"
#include "rm_ops.h"

int main(void) {
  rm_config cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.arch = RM_ENC_POSTLN;
  cfg.n_layers = 2;
  cfg.hidden = 128;
  cfg.n_heads = 2;
  cfg.ffn = 512;
  cfg.vocab = 1000;
  cfg.max_pos = 64;
  cfg.weight_dtype = RM_F32;
  cfg.gelu = RM_GELU_ERF;
  cfg.ln_eps = 1e-12f;
  cfg.max_batch_seqs = 4;
  cfg.max_tokens = 128;
  cfg.max_len = 64;
  cfg.sched_max_batch = 4;
  cfg.sched_c0 = 2;
  cfg.sched_c1 = 1;
  cfg.attn_impl = RM_ATTN_FUSED;
  cfg.sched_objective = RM_SCHED_LATENCY;
  const size_t wb = rm_weights_bytes(&cfg);
  if (wb == 0) {
    fprintf(stderr, "rm_weights_bytes: %s\n", rm_last_error());
    return 1;
  }
  const int32_t lengths[4] = {5, 5, 5, 5};
  int32_t batches[4];
  const int nb = rm_schedule_cfg(&cfg, lengths, 4, batches);
  if (nb < 0) {
    fprintf(stderr, "rm_schedule_cfg: %s\n", rm_last_error());
    return 1;
  }
  /* an invalid call is an error code and a message, not a crash */
  if (rm_schedule_cfg(&cfg, lengths, -1, batches) != RM_E_INVAL || rm_last_error()[0] == '\0') return 1;
  printf("%zu %d", wb, nb);
  for (int i = 0; i < 4; ++i) printf(" %d", batches[i]);
  printf("\n");
  return 0;
}
