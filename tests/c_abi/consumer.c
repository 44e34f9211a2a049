/* A plain C consumer of the Wukong C ABI: includes the public header, links libwukong.so and
 * calls the entry points that need no GPU (status strings, argument checks that return
 * before any device call). Built and run by tests/test_c_abi_consumer.py. */
#include <stdio.h>
#include <string.h>

#include "wukong.h"

static int fails = 0;

static void expect(int cond, const char* what) {
  if (!cond) {
    printf("FAIL: %s\n", what);
    ++fails;
  }
}

int main(void) {
  float dummy[64];
  const char* ok = wk_status_string(WK_OK);
  expect(ok != NULL && strlen(ok) > 0, "status string of WK_OK");
  expect(wk_status_string(WK_ERR_UNSUPPORTED) != NULL, "status string of WK_ERR_UNSUPPORTED");
  /* null handles and null arguments are rejected without a device */
  expect(wk_stack_forward(NULL, dummy, dummy, 1, NULL) == WK_ERR_INVALID_ARG, "forward, null handle");
  int64_t ticket = 7;
  expect(wk_stack_forward_host_async(NULL, dummy, dummy, 1, NULL, &ticket) == WK_ERR_INVALID_ARG && ticket == 7,
         "streamed host forward, null handle");
  expect(wk_stack_host_wait(NULL, -1) == WK_ERR_INVALID_ARG, "host wait, null handle");
  expect(wk_stack_backward(NULL, dummy, dummy, dummy, NULL, 8, NULL) == WK_ERR_INVALID_ARG, "backward, null handle");
  expect(wk_stack_backward_events(NULL, dummy, dummy, dummy, NULL, 8, NULL, NULL) == WK_ERR_INVALID_ARG,
         "backward with events, null handle");
  expect(wk_stack_create(NULL, NULL, NULL) == WK_ERR_INVALID_ARG, "create, null config");
  wk_stack_destroy(NULL);
  printf("%s\n", fails ? "c abi consumer: FAILED" : "c abi consumer: ok");
  return fails ? 1 : 0;
}
