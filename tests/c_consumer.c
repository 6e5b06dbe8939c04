/*
 * A plain C99 program that uses the library through include/dmuon.h alone
 * (no C++, no Python, no CUDA headers), exercising the calls that need no
 * GPU: the backend string, option defaults, workspace sizes and the argument
 * checks that reject a call before anything is enqueued.  Prints "ok" and
 * exits 0 when every check holds; otherwise names the failed check.
 */
#include <stdio.h>
#include <string.h>

#include "dmuon.h"

static int failures = 0;

#define CHECK(cond)                                              \
  do {                                                           \
    if (!(cond)) {                                               \
      fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
      ++failures;                                                \
    }                                                            \
  } while (0)

int main(void) {
  const char* backend = dmuon_backend_string();
  dmuon_step_options o;
  dmuon_shape s[2];
  void* params[2];
  const void* grads[2];
  float* bufs[2];
  size_t ws;

  CHECK(backend != NULL && strstr(backend, "sm_100a") != NULL);

  memset(&o, 0xff, sizeof o);
  dmuon_step_options_default(&o);
  CHECK(o.struct_size == sizeof(dmuon_step_options));
  CHECK(o.ns_steps == 5 && o.nesterov == 1 && o.ns_a == 1.5f && o.ns_b == -0.5f);
  CHECK(o.lr_scale == DMUON_LR_PLAIN && o.max_grad_norm == 0.0f && o.grad_norm_out == NULL);

  /* One 256 x 512 bf16 matrix, 5 steps: two iterates, the 256 x 256 Gram and
   * four 1 KiB scalar regions. */
  s[0].rows = 256; s[0].cols = 512; s[0].param_dtype = DMUON_BF16; s[0].grad_dtype = DMUON_BF16;
  ws = dmuon_workspace_bytes(s, 1, 5);
  CHECK(ws == 2u * 256u * 512u * 2u + 256u * 256u * 2u + 4u * 1024u);
  CHECK(dmuon_ns_workspace_bytes(256, 512, DMUON_BF16) == ws);

  params[0] = (void*)(size_t)0x10000; grads[0] = (const void*)(size_t)0x20000;
  bufs[0] = (float*)(size_t)0x30000;
  params[1] = params[0]; grads[1] = grads[0]; bufs[1] = bufs[0];
  s[1] = s[0];

  /* count == 0 is a no-op. */
  CHECK(dmuon_muon_step_batched(params, grads, bufs, s, 0, 0.02f, 0.95f, 1, 0.0f, 5, NULL) == DMUON_OK);
  /* Rejected on the host, with a message. */
  CHECK(dmuon_muon_step_batched(params, grads, bufs, s, -1, 0.02f, 0.95f, 1, 0.0f, 5, NULL) ==
        DMUON_ERR_INVALID_ARG);
  s[1].rows = 0;
  CHECK(dmuon_muon_step_batched(params, grads, bufs, s, 2, 0.02f, 0.95f, 1, 0.0f, 5, NULL) ==
        DMUON_ERR_INVALID_ARG);
  CHECK(strlen(dmuon_last_error()) > 0);
  s[1].rows = 256;
  s[1].param_dtype = 7;
  CHECK(dmuon_muon_step_batched(params, grads, bufs, s, 2, 0.02f, 0.95f, 1, 0.0f, 5, NULL) ==
        DMUON_ERR_UNSUPPORTED);
  s[1].param_dtype = DMUON_BF16;
  CHECK(dmuon_ns_orthogonalize(NULL, 4, 4, 5, NULL) == DMUON_ERR_INVALID_ARG);
  o.struct_size = 8;
  CHECK(dmuon_muon_step_batched_opts(params, grads, bufs, s, 1, &o, NULL, 0, NULL) == DMUON_ERR_INVALID_ARG);
  /* Matrices without gradients are skipped: nothing to do, success. */
  grads[0] = NULL; grads[1] = NULL;
  CHECK(dmuon_muon_step_batched(params, grads, bufs, s, 2, 0.02f, 0.95f, 1, 0.0f, 5, NULL) == DMUON_OK);

  if (failures) return 1;
  printf("ok\n");
  return 0;
}
