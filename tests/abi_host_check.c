/* A plain C host program against the xkv C ABI: it includes only xkv.h, links
 * libxkv.so and exercises the calls that need no GPU (version, status
 * strings, workspace queries and argument validation, which return before any
 * device work).  Prints "ok" and exits 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "xkv.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

/* the Llama-3.1-8B shape: batch 4, 32 query / 8 KV heads of 128, T = 65536,
 * ranks 512, top-k 256 chunks of 8, sink 8, recent 32 */
static xkv_sr_params llama_params(void) {
  xkv_sr_params p;
  memset(&p, 0, sizeof p);
  p.batch = 4;
  p.n_q_heads = 32;
  p.n_kv_heads = 8;
  p.head_dim = 128;
  p.T = 65536;
  p.rank_k = 512;
  p.rank_v = 512;
  p.chunk = 8;
  p.topk = 256;
  p.sink = 8;
  p.recent = 32;
  p.rope_theta = 500000.0f;
  p.dtype = XKV_BF16;
  p.a_k_batch_stride = p.T * p.rank_k;
  p.a_v_batch_stride = p.T * p.rank_v;
  p.bt_k_batch_stride = (int64_t)p.n_kv_heads * p.head_dim * p.rank_k;
  p.bt_v_batch_stride = (int64_t)p.n_kv_heads * p.head_dim * p.rank_v;
  return p;
}

int main(void) {
  expect(xkv_version() > 0, "version");
  for (int s = XKV_OK; s <= XKV_ERR_DEVICE_TIMEOUT; ++s)
    expect(xkv_status_string((xkv_status)s) != NULL && xkv_status_string((xkv_status)s)[0] != '\0', "status string");

  xkv_sr_params p = llama_params();
  size_t bytes = 0;
  expect(xkv_sr_workspace_size(&p, &bytes) == XKV_OK && bytes > 0, "SR workspace size");
  expect(xkv_sr_workspace_size(&p, NULL) == XKV_ERR_INVALID_ARG, "SR workspace size without output");
  expect(xkv_sr_workspace_size(NULL, &bytes) == XKV_ERR_INVALID_ARG, "SR workspace size without params");

  xkv_sr_params bad = p;
  bad.topk = 8193; /* more chunks than the middle holds */
  expect(xkv_sr_workspace_size(&bad, &bytes) == XKV_ERR_INVALID_ARG, "top-k above n_mid");
  bad = p;
  bad.n_q_heads = 30; /* not a multiple of the KV heads */
  expect(xkv_sr_workspace_size(&bad, &bytes) == XKV_ERR_INVALID_ARG, "GQA grouping");

  /* the decode call rejects missing buffers before touching the device */
  expect(xkv_sr_attention_decode(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
             XKV_ERR_INVALID_ARG,
         "SR decode without buffers");

  /* xK-SR: the value cache is [B][T][d]; its batch stride must cover T d */
  xkv_sr_params xk = p;
  xk.a_v_batch_stride = p.T * p.n_kv_heads * p.head_dim;
  size_t xbytes = 0;
  expect(xkv_xk_sr_workspace_size(&xk, &xbytes) == XKV_OK && xbytes > 0, "xK-SR workspace size");
  xk.a_v_batch_stride = p.T * p.head_dim;
  expect(xkv_xk_sr_workspace_size(&xk, &xbytes) == XKV_ERR_INVALID_ARG, "xK-SR value stride");

  /* NER / energy rank argument checks */
  size_t nbytes = 0;
  expect(xkv_ner_workspace_size(4096, 1024, &nbytes) == XKV_OK && nbytes > 0, "NER workspace size");
  expect(xkv_ner_workspace_size(4096, 1000, &nbytes) == XKV_ERR_INVALID_ARG, "NER block must divide n");
  int32_t fake_rank[4];
  expect(xkv_energy_rank((const float*)0x10000, 4096, 1024, 0.0, fake_rank, NULL, (void*)0x20000, nbytes, NULL) ==
             XKV_ERR_INVALID_ARG,
         "energy share must be positive");

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
