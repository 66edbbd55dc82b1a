/* A plain C11 client of libnf4ls: the header compiles as C and the host-side calls
 * work from C without any CUDA device (code tables, size queries, argument and
 * config refusals).  Built and run by tests/test_c_client.py; prints "ok" and
 * returns 0, or names the first failed check and returns 1. */
#include <stdio.h>
#include <string.h>

#include "nf4ls.h"

#define CHECK(cond)                                                            \
  do {                                                                         \
    if (!(cond)) {                                                             \
      printf("FAILED %s:%d: %s (%s)\n", __FILE__, __LINE__, #cond, nf4ls_last_error()); \
      return 1;                                                                \
    }                                                                          \
  } while (0)

int main(void) {
  CHECK(nf4ls_version() > 0);

  /* code tables: 16 NF4 entries from -1 to 1 with an exact zero, 256 nested entries */
  float nf4[16], code8[256];
  uint64_t hash = 0;
  CHECK(nf4ls_codebooks(nf4, code8, &hash) == NF4LS_OK);
  CHECK(nf4[0] == -1.0f && nf4[15] == 1.0f && hash != 0);
  int zeros = 0;
  for (int i = 0; i < 16; ++i) zeros += nf4[i] == 0.0f;
  CHECK(zeros == 1);
  for (int i = 1; i < 256; ++i) CHECK(code8[i - 1] < code8[i]);

  /* one Llama-8B-shaped layer at batch 4 x 512 */
  nf4ls_layer_cfg l;
  memset(&l, 0, sizeof l);
  l.hidden = 4096;
  l.inter = 14336;
  l.n_q = 32;
  l.n_kv = 8;
  l.head_dim = 128;
  l.batch = 4;
  l.seq = 512;
  l.rope_theta = 500000.0f;
  l.rms_eps = 1e-5f;
  l.lora_r = 16;
  l.lora_alpha = 32.0f;
  const size_t shard = nf4ls_shard_bytes(&l);
  CHECK(shard > 112513052u && shard < 113000000u);
  CHECK(nf4ls_shard_quantized_bytes(&l) > 0 && nf4ls_workspace_bytes(&l) > 0);
  /* LoRA stride: A_q, B_q, A_v, B_v = 16 x 4096 + 4096 x 16 + 16 x 4096 + 1024 x 16 */
  CHECK(nf4ls_lora_stride(&l) == (size_t)(16 * 4096 * 3 + 1024 * 16));

  nf4ls_model_cfg mc;
  memset(&mc, 0, sizeof mc);
  mc.layer = l;
  mc.n_layers = 32;
  mc.vocab = 128256;
  mc.lr = 2e-4f;
  mc.beta1 = 0.9f;
  mc.beta2 = 0.999f;
  mc.adam_eps = 1e-8f;
  CHECK(nf4ls_model_workspace_bytes(&mc) > nf4ls_workspace_bytes(&l));
  CHECK(nf4ls_adapter_file_bytes(&mc) == 64 + 12 * (size_t)32 * nf4ls_lora_stride(&l));

  /* refusals on the host: a bad config, a bad pool depth, null arguments */
  nf4ls_layer_cfg bad = l;
  bad.head_dim = 96;
  CHECK(layer_forward(&bad, NULL, NULL, NULL, NULL, NULL, 0, NULL) != NF4LS_OK);
  size_t off = 0, bytes = shard;
  nf4ls_pool* pool = NULL;
  CHECK(nf4ls_pool_create((const void*)64, &off, &bytes, 1, 9, (void*)256, shard, &pool) == NF4LS_INVALID_ARG);
  CHECK(pool == NULL);
  CHECK(nf4ls_set_gemm_half(7) == NF4LS_INVALID_ARG);
  int32_t step = -1;
  CHECK(nf4ls_adapter_load("/nonexistent/adapter.bin", &mc, NULL, &step, NULL) == NF4LS_INVALID_ARG);
  CHECK(step == -1);
  CHECK(strlen(nf4ls_last_error()) > 0);
  printf("ok\n");
  return 0;
}
