/* A plain C consumer of the library: include/dsa.h must compile as C99 and
 * the shared library must link and answer the calls that need no GPU
 * (version, status strings, workspace sizes, host-side argument errors). */
#include <stdio.h>
#include <string.h>

#include "dsa.h"

int main(void)
{
    if (dsa_version() != ((DSA_VERSION_MAJOR << 16) | DSA_VERSION_MINOR)) return 1;
    if (strcmp(dsa_status_string(DSA_ERR_WORKSPACE), "DSA_ERR_WORKSPACE") != 0) return 2;
    if (dsa_decode_workspace_size(64, 65536, 128, 128, 2048) < (size_t)64 * 65536 * 4) return 3;
    if (dsa_split_workspace_size(8, 4, 131072, 128, 128, 512) == 0) return 4;
    /* argument errors come back before anything is enqueued */
    if (dsa_topk(NULL, 10, 0, 1, 10, 4, NULL, NULL, 0, NULL) != DSA_ERR_INVALID_ARG) return 5;
    if (dsa_merge_partials(NULL, 0, NULL, 0, 2, 4, 128, 128, NULL, NULL, NULL) != DSA_ERR_INVALID_ARG) return 6;
    if (dsa_quantize_e4m3(NULL, DSA_BF16, 4, 128, NULL, NULL, NULL) != DSA_ERR_INVALID_ARG) return 7;
    puts("ok");
    return 0;
}
