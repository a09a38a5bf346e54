/* A plain C99 program against the library's header: it shows that the boundary
 * is a C ABI (no C++ or torch types) and exercises the host-only entry points.
 * It prints one line per query; tests/test_abi.py compares them with the
 * Python binding. No CUDA call is made. */
#include <stdio.h>
#include <string.h>

#include "bsa.h"

int main(void) {
    bsa_params p;
    memset(&p, 0, sizeof p);
    p.B = 1; p.heads = 32; p.T = 24; p.H = 48; p.W = 80; p.d = 128;
    p.chunk_t = 4; p.chunk_h = 4; p.chunk_w = 8;
    p.mode = BSA_SEL_TOPK; p.topk = 45;
    p.cdf_p = 0.9f; p.cdf_cap_frac = 0.25f;

    int64_t rows = 0, nnz = 0;
    bsa_shape s;
    int rc = bsa_plan_sizes(&p, &rows, &nnz);
    printf("plan_sizes %d %lld %lld\n", rc, (long long)rows, (long long)nnz);
    rc = bsa_shape_info(&p, &s);
    printf("shape %d %lld %lld %lld %d %d %d %d\n", rc, (long long)s.BH, (long long)s.N,
           (long long)s.rows, s.d, s.Nc, s.Nq, s.Nk);
    printf("workspace %zu %zu\n", bsa_workspace_size(&p), bsa_backward_workspace_size(&p));

    /* argument errors come back as status codes, before any device work */
    printf("null_q %d\n", bsa_plan(&p, NULL, NULL, NULL, 0, NULL, NULL, 0, NULL));
    printf("null_bwd_ex %d\n", bsa_backward_ex(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                                                0, NULL, 0, NULL, NULL, NULL, 20000000u, 3, NULL));
    printf("null_status %d\n", bsa_read_status(NULL, NULL));
    p.d = 96;
    printf("bad_d %d %s\n", bsa_plan_sizes(&p, &rows, &nnz), bsa_status_string(BSA_ERR_UNSUPPORTED));
    printf("version %d\n", bsa_version());
    return 0;
}
