/* Strict C99 client of include/rope_attn.h: it compiles against the header alone, links
 * librope_attn.so and exercises the host-side part of the ABI (workspace sizing, status
 * strings, argument validation), none of which touches a GPU.  Exit code 0 = all good. */
#include <stdio.h>
#include <string.h>

#include "rope_attn.h"

static int failures = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    fprintf(stderr, "FAILED: %s\n", what);
    ++failures;
  }
}

int main(void) {
  ra_problem p;
  memset(&p, 0, sizeof p);
  p.B = 2;
  p.H = 32;
  p.n = 8192;
  p.d = 128;
  p.dtype = RA_BF16;
  p.causal = 1;
  p.base = 1e4;
  const size_t ws = rope_attn_workspace_bytes(&p);
  /* the rotated bf16 Q~ and K~ dominate the workspace */
  expect(ws >= (size_t)2 * 2 * 32 * 8192 * 128 * 2, "headline workspace holds Q~ and K~");
  expect(ws % 1024 == 0, "workspace size is a multiple of 1 KiB");
  expect(rope_attn_proj_workspace_bytes(&p) == (size_t)1024 + 3 * (size_t)2 * 8192 * 32 * 128 * 2,
         "projection workspace is the error word and three merged gradients");

  ra_problem bad = p;
  bad.d = 3;
  expect(rope_attn_workspace_bytes(&bad) == 0, "odd d has no workspace");
  bad = p;
  bad.reserved = 1;
  expect(rope_attn_workspace_bytes(&bad) == 0, "reserved must be zero");

  expect(strcmp(rope_attn_status_string(RA_OK), "ok") == 0, "status string of RA_OK");
  expect(rope_attn_status_string(RA_ERR_TIMEOUT) != NULL, "status string of RA_ERR_TIMEOUT");

  /* null operands are rejected before any launch */
  expect(rope_attn_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, ws, NULL) ==
             RA_ERR_INVALID_ARG,
         "fwd rejects null operands");
  expect(rope_attn_loss(&p, NULL, NULL, NULL, NULL, NULL, ws, NULL) == RA_ERR_INVALID_ARG,
         "loss rejects null operands");
  expect(rope_attn_bwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                       NULL, ws, NULL) == RA_ERR_INVALID_ARG,
         "bwd rejects null operands");
  expect(rope_attn_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
             RA_ERR_INVALID_ARG,
         "fwd rejects a null problem");

  if (failures == 0) printf("c abi ok: workspace %zu bytes\n", ws);
  return failures == 0 ? 0 : 1;
}
