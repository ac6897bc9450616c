/* A plain C99 user of the C ABI: includes ep.h, links libep.so and makes the
 * host-side calls that need no GPU (sizes, handle life cycle, argument
 * rejection, status names).  Built and run by tests/test_c_consumer.py; it
 * also prints ep_recv_rows_upper_bound for the sizes given on the command
 * line (triples T k E, block_m 128) so the test can check them.
 * Exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "ep.h"

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "check failed, line %d: %s\n", __LINE__, #cond); \
            return 1;                                                 \
        }                                                             \
    } while (0)

int main(int argc, char** argv)
{
    /* an address host code never dereferences: handle creation makes no CUDA call */
    void* const fake_ws = (void*)(uintptr_t)0x7f0000000000ull;
    const size_t need = ep_workspace_bytes(1024, 8, 256, 8, 128);
    ep_handle_t h = NULL;
    int64_t n = 0;
    int i;

    CHECK(need > 0);
    CHECK(ep_workspace_bytes(1024, 8, 256, 7, 128) == 0); /* E % R != 0 */
    CHECK(ep_workspace_bytes(1024, 0, 256, 8, 128) == 0);
    CHECK(ep_recv_rows_upper_bound(-1, 8, 256, 128) == -1);

    CHECK(ep_handle_create(fake_ws, need - 1, 1024, 8, 256, 8, 128, &h) ==
          EP_ERR_WORKSPACE_TOO_SMALL);
    CHECK(h == NULL);
    CHECK(ep_handle_create((char*)fake_ws + 16, need, 1024, 8, 256, 8, 128, &h) ==
          EP_ERR_ALIGNMENT);
    CHECK(ep_handle_create(fake_ws, need, 1024, 8, 256, 8, 128, &h) == EP_OK);
    CHECK(h != NULL);

    /* no layout yet: data calls report the state error and enqueue nothing */
    CHECK(ep_dispatch(h, fake_ws, 7168, EP_FMT_BF16, fake_ws, NULL, 64, NULL) == EP_ERR_STATE);
    CHECK(ep_combine(h, fake_ws, 64, (const float*)fake_ws, 7168, fake_ws, NULL) ==
          EP_ERR_STATE);
    /* bad arguments */
    CHECK(ep_layout(h, (const int64_t*)fake_ws, 1025, NULL) == EP_ERR_INVALID_ARG);
    CHECK(ep_layout(h, NULL, 4, NULL) == EP_ERR_INVALID_ARG);
    CHECK(ep_layout(NULL, (const int64_t*)fake_ws, 4, NULL) == EP_ERR_INVALID_ARG);
    /* views lie inside the workspace */
    CHECK(ep_handle_view(h, EP_VIEW_DST_ROW, &n) != NULL);
    CHECK((const char*)ep_handle_view(h, EP_VIEW_DST_ROW, &n) >= (const char*)fake_ws);
    CHECK((const char*)ep_handle_view(h, EP_VIEW_DST_ROW, &n) <
          (const char*)fake_ws + need);
    /* nothing ran: the error word is clear without touching a device */
    CHECK(ep_handle_check(h, NULL) == EP_OK);
    ep_handle_destroy(h);
    ep_handle_destroy(NULL);

    CHECK(strcmp(ep_strerror(EP_OK), "EP_OK") == 0);
    CHECK(strstr(ep_strerror(EP_ERR_CAPACITY), "CAPACITY") != NULL);
    CHECK(ep_last_error_message() != NULL);

    for (i = 1; i + 2 < argc; i += 3) {
        const int T = atoi(argv[i]), k = atoi(argv[i + 1]), E = atoi(argv[i + 2]);
        printf("%lld\n", (long long)ep_recv_rows_upper_bound(T, k, E, 128));
    }
    return 0;
}
