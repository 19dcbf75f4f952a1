/*
 * A C (not C++) program against include/vi.h and libvi.so: the header must
 * compile as C99, and the library must link and answer its host-only calls
 * (no GPU is needed: no call here reaches a kernel launch).
 *
 * Build: gcc -std=c99 -Wall -Wextra -I include -o abi_check abi_check.c \
 *            -L clip_temporal_modules_b200 -lvi -Wl,-rpath,<dir of libvi.so>
 */
#include <stdio.h>
#include <string.h>

#include "vi.h"

int main(void) {
  printf("vi_version %d\n", vi_version());
  printf("status -3 = %s\n", vi_status_string(VI_ERR_UNSUPPORTED));
  /* A host-side rejection: F not a multiple of N; nothing is launched. */
  int st = vi_dual_attn((const void*)0x100000, (const void*)0x200000, (const void*)0x300000,
                        (void*)0x400000, 65, 4, 2, 2, 64, 8, 8, 16, (vi_stream_t)0);
  printf("bad F %% N -> %s\n", vi_status_string(st));
  /* An empty call (no positions) succeeds without touching any pointer. */
  st = vi_temporal_conv(NULL, NULL, NULL, NULL, 64, 4, 0, 64, 3, (vi_stream_t)0);
  printf("empty conv -> %s\n", vi_status_string(st));
  return (vi_version() >= 100 && st == VI_OK) ? 0 : 1;
}
