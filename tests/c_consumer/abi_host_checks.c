/*
 * A plain C99 program that uses the h3b library through include/h3b.h alone and
 * links to libh3b.so. It checks the host-side contract only: workspace sizing,
 * argument validation, status strings and the quick return of empty problems.
 * Nothing here queries a device or launches a kernel, so it runs on a machine
 * without a GPU. Prints "OK" and exits 0 when every check holds.
 */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "h3b.h"

static int failures = 0;

#define EXPECT(cond)                                                         \
  do {                                                                       \
    if (!(cond)) {                                                           \
      fprintf(stderr, "FAIL line %d: %s (%s)\n", __LINE__, #cond,            \
              h3b_last_error_detail());                                      \
      ++failures;                                                            \
    }                                                                        \
  } while (0)

/* Struct layouts as the C compiler sees them, one "struct field offset size" line
   per field, for the binding's test to compare with its own mirror of the structs. */
#define FIELD(S, F) printf("%s %s %zu %zu\n", #S, #F, offsetof(S, F), sizeof(((S*)0)->F))

static void print_layouts(void) {
  printf("sizeof h3b_dims %zu\n", sizeof(h3b_dims));
  FIELD(h3b_dims, B); FIELD(h3b_dims, T); FIELD(h3b_dims, H); FIELD(h3b_dims, W);
  FIELD(h3b_dims, d); FIELD(h3b_dims, n_heads); FIELD(h3b_dims, head_dim); FIELD(h3b_dims, d_ff);
  FIELD(h3b_dims, rope_t); FIELD(h3b_dims, rope_h); FIELD(h3b_dims, rope_w);
  FIELD(h3b_dims, rope_theta); FIELD(h3b_dims, ln_eps); FIELD(h3b_dims, qkv_int8); FIELD(h3b_dims, wo_bf16);
  printf("sizeof h3b_block_weights %zu\n", sizeof(h3b_block_weights));
  FIELD(h3b_block_weights, w_ada); FIELD(h3b_block_weights, b_ada); FIELD(h3b_block_weights, wqkv);
  FIELD(h3b_block_weights, sqkv); FIELD(h3b_block_weights, wqkv_bf16); FIELD(h3b_block_weights, bqkv);
  FIELD(h3b_block_weights, wo); FIELD(h3b_block_weights, so); FIELD(h3b_block_weights, bo);
  FIELD(h3b_block_weights, w1); FIELD(h3b_block_weights, s1); FIELD(h3b_block_weights, b1);
  FIELD(h3b_block_weights, w2); FIELD(h3b_block_weights, s2); FIELD(h3b_block_weights, b2);
  FIELD(h3b_block_weights, wo_bf16);
  printf("sizeof h3b_kernel_time %zu\n", sizeof(h3b_kernel_time));
  FIELD(h3b_kernel_time, name); FIELD(h3b_kernel_time, launches); FIELD(h3b_kernel_time, total_ms);
}

/* 2 x 16 x 16 latent grid, d = 256 (4 heads of 64), d_ff = 1024. */
static h3b_dims small_dims(void) {
  h3b_dims d;
  memset(&d, 0, sizeof d);
  d.B = 1; d.T = 2; d.H = 16; d.W = 16;
  d.d = 256; d.n_heads = 4; d.head_dim = 64; d.d_ff = 1024;
  d.rope_t = 16; d.rope_h = 24; d.rope_w = 24;
  d.rope_theta = 10000.0f; d.ln_eps = 1e-6f;
  d.qkv_int8 = 1; d.wo_bf16 = 0;
  return d;
}

int main(void) {
  const h3b_dims d = small_dims();
  print_layouts();
  size_t bytes = 0;

  /* workspace: at least the int8 activations (L x d_ff) and bf16 Q, K, V, O (8 L d bytes) */
  EXPECT(h3b_workspace_size(&d, &bytes) == H3B_OK);
  EXPECT(bytes >= (size_t)512 * 1024 + (size_t)8 * 512 * 256);
  EXPECT(h3b_workspace_size(NULL, &bytes) == H3B_ERR_ARG);

  h3b_dims bad = d;
  bad.head_dim = 96;
  EXPECT(h3b_workspace_size(&bad, &bytes) == H3B_ERR_SHAPE);
  EXPECT(strlen(h3b_last_error_detail()) > 0);
  bad = d;
  bad.rope_t = 15;
  EXPECT(h3b_workspace_size(&bad, &bytes) == H3B_ERR_SHAPE);
  bad = d;
  bad.T = 65536; bad.H = 65536; bad.W = 2; /* 2^33 tokens */
  EXPECT(h3b_workspace_size(&bad, &bytes) == H3B_ERR_SHAPE);

  /* status strings exist for every status */
  {
    const h3b_status all[] = {H3B_OK, H3B_ERR_ARG, H3B_ERR_SHAPE, H3B_ERR_ALIGN, H3B_ERR_WORKSPACE,
                              H3B_ERR_ARCH, H3B_ERR_CUDA, H3B_ERR_DEVICE_CHECK};
    size_t i;
    for (i = 0; i < sizeof all / sizeof all[0]; ++i) EXPECT(strlen(h3b_status_string(all[i])) > 0);
  }

  /* block entry point: argument, alignment and workspace errors come before any device query */
  {
    h3b_block_weights w;
    memset(&w, 0, sizeof w);
    void* x = (void*)0x20000;
    const float* c = (const float*)0x30000;
    void* ws = (void*)0x40000;
    EXPECT(h3b_block_forward(&d, &w, c, NULL, ws, bytes, NULL) == H3B_ERR_ARG);
    EXPECT(h3b_block_forward(&d, &w, c, (char*)x + 2, ws, bytes, NULL) == H3B_ERR_ALIGN);
    EXPECT(h3b_block_forward(&d, &w, c, x, (char*)ws + 16, bytes, NULL) == H3B_ERR_ALIGN);
    EXPECT(h3b_block_forward(&d, &w, c, x, ws, bytes - 1, NULL) == H3B_ERR_WORKSPACE);
  }

  /* token pairing needs an even W */
  {
    h3b_dims odd = d;
    odd.W = 15;
    EXPECT(h3b_token_pair(&odd, (const void*)0x1000, (void*)0x2000, NULL, NULL) == H3B_ERR_SHAPE);
  }

  /* GEMM sizes and pointers */
  EXPECT(h3b_gemm_i8_s32((const int8_t*)0x1000, (const int8_t*)0x2000, (int32_t*)0x3000, 128, 24, 128, NULL) ==
         H3B_ERR_SHAPE);
  EXPECT(h3b_gemm_i8_s32(NULL, (const int8_t*)0x2000, (int32_t*)0x3000, 128, 256, 128, NULL) == H3B_ERR_ARG);

  /* empty problems return OK once their sizes are checked */
  EXPECT(h3b_gemm_i8_s32(NULL, NULL, NULL, 0, 256, 128, NULL) == H3B_OK);
  EXPECT(h3b_quantize_rows(NULL, 0, 256, NULL, NULL, NULL, NULL) == H3B_OK);
  EXPECT(h3b_range_apply(NULL, NULL, 0, NULL) == H3B_OK);
  EXPECT(h3b_range_apply(NULL, NULL, 4, NULL) == H3B_ERR_SHAPE);

  /* the bounded-wait test hook checks its arguments on the host */
  {
    int waited = -1;
    EXPECT(h3b_test_bounded_wait(10ull, &waited) == H3B_ERR_ARG);
    EXPECT(h3b_test_bounded_wait(1000000ull, NULL) == H3B_ERR_ARG);
    EXPECT(waited == -1);
  }

  /* the profiler's host side: nothing recorded yet */
  {
    h3b_kernel_time kt[4];
    EXPECT(h3b_profile_enable(1) == H3B_OK);
    EXPECT(h3b_profile_enable(0) == H3B_OK);
    EXPECT(h3b_profile_read(kt, 4) == 0);
    EXPECT(h3b_profile_read(NULL, 4) < 0);
  }

  printf("%s\n", failures ? "FAILED" : "OK");
  return failures ? 1 : 0;
}
