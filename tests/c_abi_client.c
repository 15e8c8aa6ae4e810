/*
 * c_abi_client.c: a plain C99 client of the SFA C ABI.
 *
 * It includes only include/sfa.h, links libsfa.so and runs the entry points
 * that need no GPU: the default configuration, validation, the state layout,
 * status strings, and the rejection of a NULL handle by every call that takes
 * one (no call may reach the GPU with it).  Prints "ok" and exits 0 when
 * every check holds.  Built and run by tests/test_abi_host.py.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "sfa.h"

#define CHECK(c)                                                     \
  do {                                                               \
    if (!(c)) {                                                      \
      fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #c); \
      return 1;                                                      \
    }                                                                \
  } while (0)

int main(void) {
  sfa_config c;
  sfa_state_layout lay;
  int dummy_input[8];

  sfa_config_default(&c);
  CHECK(c.window_k == 16 && c.ring_size == 16 && c.n_slots == 64);
  CHECK(c.in_dtype == SFA_BF16 && c.slots == NULL);
  c.n_layers = 24;
  c.n_q_heads = 14;
  c.n_kv_heads = 2;
  c.head_dim = 64;
  CHECK(sfa_config_validate(&c) == SFA_ERR_INVALID_ARG); /* no slots yet */
  /* validation only checks the slots pointer for NULL and alignment */
  c.slots = (const float*)(uintptr_t)256;
  CHECK(sfa_config_validate(&c) == SFA_OK);
  c.head_dim = 96;
  CHECK(sfa_config_validate(&c) == SFA_ERR_UNSUPPORTED);
  c.head_dim = 64;

  CHECK(sfa_state_layout_for(&c, 3, &lay) == SFA_OK);
  CHECK(lay.total_bytes == lay.header_bytes + lay.stream_stride * 24 * 3);
  CHECK(lay.off_ring > lay.off_ring_sum && lay.off_ring_sum > lay.off_field);
  CHECK(sfa_state_layout_for(&c, 0, &lay) == SFA_ERR_INVALID_ARG);

  CHECK(sfa_abi_version() == SFA_ABI_VERSION);
  CHECK(strcmp(sfa_status_string(SFA_OK), "ok") == 0);
  CHECK(strcmp(sfa_status_string(12345), "unknown status") == 0);

  /* every call that takes a handle rejects NULL before any CUDA work */
  CHECK(sfa_destroy(NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_state_bytes(NULL, 1) == 0);
  CHECK(sfa_prefill_workspace_bytes(NULL, 1, 64) == 0);
  CHECK(sfa_prefill_layers_workspace_bytes(NULL, 1, 1, 64) == 0);
  CHECK(sfa_state_reset(NULL, dummy_input, 1, NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_prefill(NULL, dummy_input, dummy_input, dummy_input, 8, 1, dummy_input,
                    (float*)dummy_input, dummy_input, 0, NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_prefill_static_ws(NULL, dummy_input, dummy_input, dummy_input, 8, 1, dummy_input,
                              (float*)dummy_input, NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_decode_step(NULL, dummy_input, dummy_input, dummy_input, 1, dummy_input,
                        (float*)dummy_input, NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_decode_step_ex(NULL, 0, 1, NULL, 1, dummy_input, dummy_input, dummy_input, 1,
                           dummy_input, (float*)dummy_input, NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_set_decode_input_prefetch(NULL, 1) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_check_device_status(NULL, NULL) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_debug_set_wait_limit(NULL, 0, -1) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_debug_set_paths(NULL, -1, 1) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_set_output_mode(NULL, SFA_OUT_BF16) == SFA_ERR_INVALID_ARG);
  CHECK(sfa_prefill_ragged(NULL, NULL, NULL, NULL, 1, NULL, 1, NULL, NULL, NULL, 0, NULL) == SFA_ERR_INVALID_ARG);

  printf("ok\n");
  return 0;
}
