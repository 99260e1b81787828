/* A plain C99 client of libattn.so: the header must compile as C and the library must
 * link and answer its host-side queries without a GPU.  Used by tests/test_abi.py
 * (compiled with gcc -std=c99 -Wall -Wextra -Werror and run).  Every call here either
 * needs no device or is rejected by the host-side validation before anything launches. */
#include <stdio.h>
#include <string.h>

#include "attn.h"

int main(void) {
    void *p = (void *)(size_t)0x1000; /* never dereferenced: the calls below fail validation first */
    size_t fwd_ws = attn_fwd_workspace_size(2, 1024, 2048, 16, 4, 128, ATTN_BF16);
    size_t bwd_ws = attn_bwd_workspace_size(2, 1024, 2048, 16, 4, 128, ATTN_BF16);
    attn_status st;

    if (attn_version() <= 0) return 1;
    if (fwd_ws != 256) return 2;
    /* D [16, 2048] float32 rounded to 256 bytes, the float32 dQ accumulator, the counter */
    if (bwd_ws != (size_t)16 * 2048 * 4 + (size_t)2048 * 16 * 128 * 4 + 256) return 3;

    /* head dim 96 is outside {32, 64, 128}: rejected on the host */
    st = attn_fwd(p, p, p, NULL, 2, 1024, 1024, 2048, 16, 4, 96, 0.0883883f, 1, ATTN_BF16, p, (float *)p, p,
                  fwd_ws, NULL);
    if (st != ATTN_ERR_UNSUPPORTED) return 4;
    if (strlen(attn_last_error_message()) == 0) return 5;

    /* a NULL operand is an invalid argument */
    st = attn_fwd(NULL, p, p, NULL, 2, 1024, 1024, 2048, 16, 4, 128, 0.0883883f, 0, ATTN_BF16, p, (float *)p, p,
                  fwd_ws, NULL);
    if (st != ATTN_ERR_INVALID_ARG) return 6;

    printf("attn %d: %s / %s\n", (int)attn_version(), attn_status_string(ATTN_ERR_UNSUPPORTED),
           attn_status_string(st));
    return 0;
}
