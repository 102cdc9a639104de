/* A plain C11 consumer of the library's C ABI: it includes the header as C (not C++), links
 * the shared library and calls the entry points that need no GPU, printing one line each.
 * test_abi.py builds it with gcc, runs it and checks the lines against the Python binding. */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "q1m.h"

static void print_bounds(const char* tag, int64_t m, const int64_t* ends) {
  printf("%s %lld", tag, (long long)m);
  for (int64_t i = 0; i < m; ++i) printf(" %lld", (long long)ends[i]);
  printf("\n");
}

int main(void) {
  q1m_params p;
  memset(&p, 0, sizeof p);
  p.in_dtype = Q1M_BF16;
  p.out_dtype = Q1M_F32;
  p.rope_base = 1e4;
  p.yarn_s = 2.0;
  p.dca_chunk = 384;
  p.local_window = 128;
  p.vs_vertical = 20;
  p.vs_slash = 70;
  p.vs_last_q = 64;
  p.vs_force_local = 8;
  p.prefill_chunk = 256;
  printf("version %s\n", q1m_version());

  int64_t ends[64];
  print_bounds("fixed", q1m_prefill_bounds(1500, &p, ends, 64), ends);
  p.equal_cost_chunks = 3;
  print_bounds("equal", q1m_prefill_bounds(1500, &p, ends, 64), ends);
  printf("too_many %lld\n", (long long)q1m_prefill_bounds(1500, &p, ends, 2));
  p.equal_cost_chunks = 0;

  printf("workspace %zu\n", q1m_workspace_bytes(1500, 4, 2, 128, &p));
  printf("host_workspace %zu\n", q1m_host_workspace_bytes(1500, 4, 2, 128, &p));
  printf("decode_scratch %zu\n", q1m_dca_decode_scratch_bytes(4, 128));

  q1m_status st = q1m_dca_sparse_prefill(NULL, NULL, NULL, NULL, NULL, 1500, 4, 2, 128, &p, NULL,
                                         0, NULL);
  printf("null_status %d\n", (int)st);
  printf("null_message %s\n", q1m_last_error());

  /* the parameter block's layout as the C compiler lays it out */
#define FIELD(f) printf("offset_%s %zu\n", #f, offsetof(q1m_params, f))
  printf("sizeof_params %zu\n", sizeof(q1m_params));
  FIELD(in_dtype);
  FIELD(out_dtype);
  FIELD(rope_base);
  FIELD(yarn_s);
  FIELD(dca_chunk);
  FIELD(local_window);
  FIELD(vs_vertical);
  FIELD(vs_slash);
  FIELD(vs_last_q);
  FIELD(vs_force_local);
  FIELD(prefill_chunk);
  FIELD(equal_cost_chunks);
#undef FIELD
  return 0;
}
