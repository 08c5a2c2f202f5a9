/* A plain C99 client of the library: it includes only include/csa.h, links against
 * libcsa_b200.so and checks the host-side behaviour of the ABI (argument checks and
 * workspace sizes), which needs no GPU. Prints "ok" and exits 0 on success. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "csa.h"

#define CHECK(cond)                                                    \
  do {                                                                 \
    if (!(cond)) {                                                     \
      printf("failed: %s (line %d)\n", #cond, __LINE__);               \
      return 1;                                                        \
    }                                                                  \
  } while (0)

static void* fake(void) { return (void*)(uintptr_t)(1u << 20); } /* never dereferenced */

int main(void) {
  CHECK(strcmp(csa_status_string(CSA_OK), "ok") == 0);
  CHECK(csa_indexer_topk_workspace_size(4, 262144, 1024) > 4u * 262144u * 12u);
  CHECK(csa_attn_workspace_size(4, 128, 1024 + CSA_WINDOW) > 0);
  CHECK(csa_prefill_workspace_size(65536, 65536, 128, 1024) > 0);

  csa_topk_args t;
  memset(&t, 0, sizeof t);
  t.B = 2; t.H_I = 64; t.k = 512; t.Nmax = 1000; /* not a multiple of 128 */
  t.n_entries = fake(); t.q_fp4 = fake(); t.q_sf = fake(); t.w = fake();
  t.k_fp4 = fake(); t.k_sf = fake(); t.idx = fake();
  CHECK(csa_indexer_topk(&t, fake(), 1u << 30, NULL) == CSA_ERR_INVALID_ARG);
  t.Nmax = 1024; t.H_I = 8;
  CHECK(csa_indexer_topk_bf16(&t, fake(), 1u << 30, NULL) == CSA_ERR_UNSUPPORTED);
  t.H_I = 64; t.B = 0;
  CHECK(csa_indexer_topk(&t, fake(), 1u << 30, NULL) == CSA_OK);

  csa_attn_args a;
  memset(&a, 0, sizeof a);
  a.B = 1; a.H = 96; a.k = 64; a.Nmax = 128; a.rope_base = 10000.f;
  CHECK(csa_sparse_attn_decode(&a, fake(), 1u << 30, NULL) == CSA_ERR_UNSUPPORTED);
  a.H = 128;
  CHECK(csa_sparse_attn_decode_noalloc(&a, NULL) == CSA_ERR_INVALID_ARG); /* null pointers */

  csa_compress_args c;
  memset(&c, 0, sizeof c);
  c.B = 1; c.T = 64; c.m = 0;
  CHECK(csa_compress(&c, NULL) == CSA_ERR_INVALID_ARG);

  csa_iquery_args q;
  memset(&q, 0, sizeof q);
  q.T = 4; q.r = 100; q.H_I = 64;
  CHECK(csa_indexer_query(&q, NULL) == CSA_ERR_INVALID_ARG);

  csa_oproj_args o;
  memset(&o, 0, sizeof o);
  o.T = 4; o.H = 128; o.G = 3; o.d_g = 1024; o.d_model = 7168;
  CHECK(csa_grouped_out_proj(&o, fake(), 1u << 30, NULL) == CSA_ERR_UNSUPPORTED);

  csa_append_args p;
  memset(&p, 0, sizeof p);
  p.B = 1; p.m = 0;
  CHECK(csa_decode_append(&p, NULL) == CSA_ERR_INVALID_ARG);

  csa_ikey_args k;
  memset(&k, 0, sizeof k);
  k.B = 1; k.T = 64; k.m = 4; k.Nmax = 100;
  CHECK(csa_compress_index_keys(&k, NULL) == CSA_ERR_INVALID_ARG);

  csa_prefill_args f;
  memset(&f, 0, sizeof f);
  f.P = 6; f.T = 10; f.m = 4; f.H = 128; f.H_I = 64; f.k = 64; f.Nmax = 128;
  CHECK(csa_prefill(&f, fake(), 1u << 30, NULL) == CSA_ERR_INVALID_ARG); /* P % m != 0 */

  printf("ok\n");
  return 0;
}
