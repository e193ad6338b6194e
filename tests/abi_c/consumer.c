/* A plain C99 consumer of libmqkv: includes the public headers, links the
 * shared library and calls the entry points that need no GPU (status text,
 * size queries, argument validation).  tests/test_abi.py compiles it with
 * -pedantic -Werror, runs it and compares what it prints with the Python
 * binding's answers for the same arguments. */
#include <stdio.h>
#include <string.h>

#include "include/mqkv.h"
#include "include/mqkv_debug.h"

int main(void) {
  const mq_shape shape = {3, 32, 8, 128, 128, 32};
  const int32_t lens[3] = {1000, 0, 4097};
  int st;
  for (st = 0; st < 6; ++st) {
    const char* s = mq_status_string((mq_status)st);
    if (s == NULL || s[0] == '\0') return 1;
  }
  printf("layout_bytes %zu\n", mq_layout_bytes(&shape, lens));
  printf("packed_upper %zu\n", mq_packed_bytes_upper_bound(&shape, lens));
  printf("decode_ws %zu\n", mq_decode_workspace_bytes(&shape, lens));
  /* invalid arguments: size queries answer 0 and leave a reason */
  if (mq_layout_bytes(NULL, lens) != 0) return 2;
  if (strlen(mq_last_error()) == 0) return 3;
  {
    mq_shape bad = shape;
    bad.group_size = 16;
    if (mq_layout_bytes(&bad, lens) != 0) return 4;
  }
  if (mq_debug_arm_wait_timeout(0x80000000u) != MQ_ERR_INVALID_ARG) return 5;
  printf("ok\n");
  return 0;
}
