/* A plain C99 caller of the library: the header must compile as C (no C++ in it) and the
 * host-only entry points must link and run without a GPU.  Built and run by
 * test_c_abi_from_c.py; prints one line of results. */
#include <stdio.h>

#include "eqlin.h"

int main(void) {
    int64_t path = -1, dw_tokens = -1;
    const int s1 = eqlin_query_plan(96, 96, 4, EQLIN_BF16, EQLIN_ATTR_PATH, &path);
    const int s2 = eqlin_query_plan(32, 32, 16, EQLIN_F16, EQLIN_ATTR_DW_TOKENS, &dw_tokens);
    const int odd = eqlin_check_shape(96, 96, 3, EQLIN_BF16, EQLIN_BF16);
    const int null_handle = eqlin_forward(NULL, NULL, NULL, 4, NULL);
    printf("query=%d path=%lld dw_query=%d dw_tokens=%lld odd_g=%d null_forward=%d version=%d timeout_text=%s\n",
           s1, (long long)path, s2, (long long)dw_tokens, odd, null_handle, eqlin_version(),
           eqlin_status_string(EQLIN_ERR_TIMEOUT));
    return 0;
}
