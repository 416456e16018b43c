/* A plain C99 client of the library's C ABI (include/gdn.h), built with gcc and
 * linked against libgdn.so. It exercises only entry points that need no GPU:
 * the size queries, argument validation and the status strings. Exit status 0
 * means every check held; each failure prints one line. */
#include <stdio.h>
#include <string.h>

#include "gdn.h"

static int failures = 0;

static void expect(int cond, const char *what) {
    if (!cond) {
        printf("FAIL %s\n", what);
        ++failures;
    }
}

int main(void) {
    /* B=1, T=8192, Hq=16, Hv=32, K=V=128, bf16 */
    gdn_problem p;
    memset(&p, 0, sizeof(p));
    p.B = 1; p.T = 8192; p.Hq = 16; p.Hv = 32; p.K = 128; p.V = 128;
    p.dtype = GDN_DTYPE_BF16;
    p.scale = 0.08838834764831845f;

    const size_t fwd = gdn_fwd_workspace_size(&p), bwd = gdn_bwd_workspace_size(&p);
    const size_t saved = gdn_saved_size(&p);
    expect(fwd > 0 && bwd > 0 && saved > 0, "sizes of a valid problem are nonzero");
    expect(fwd % 256 == 0 && bwd % 256 == 0 && saved % 256 == 0, "sizes are 256-byte multiples");
    /* the saved buffer holds at least gamma, Ainv and every chunk's bf16 entry state */
    const size_t chunks = 8192 / 64;
    expect(saved >= 4u * 8192 * 32 + 2u * chunks * 32 * 64 * 64 + 2u * chunks * 32 * 128 * 128,
           "saved holds gamma, Ainv and the chunk states");

    /* packed batch: three sequences, one of them empty */
    const int32_t cu[4] = {0, 100, 100, 300};
    gdn_problem pv = p;
    pv.T = 300; pv.num_seqs = 3; pv.cu_seqlens = cu; pv.cu_seqlens_host = cu;
    expect(gdn_fwd_workspace_size(&pv) > 0, "packed batch is valid");

    /* invalid problems: size 0 from the queries, rejected before anything is enqueued */
    gdn_problem bad = p;
    bad.Hq = 3; /* 32 % 3 != 0 */
    expect(gdn_fwd_workspace_size(&bad) == 0 && gdn_saved_size(&bad) == 0, "Hv % Hq != 0 sizes 0");
    expect(gdn_chunk_fwd(&bad, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
               GDN_ERR_INVALID_ARG, "Hv % Hq != 0 rejected");
    bad = p;
    bad.K = 96;
    expect(gdn_fwd_workspace_size(&bad) == 0, "K = 96 sizes 0");
    expect(gdn_recurrent_fwd(&bad, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL) ==
               GDN_ERR_UNSUPPORTED, "K = 96 unsupported");
    const int32_t cu_bad[3] = {0, 200, 100};
    bad = pv;
    bad.num_seqs = 2; bad.T = 100; bad.cu_seqlens = cu_bad; bad.cu_seqlens_host = cu_bad;
    expect(gdn_fwd_workspace_size(&bad) == 0, "decreasing cu_seqlens sizes 0");
    expect(gdn_chunk_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
               GDN_ERR_INVALID_ARG, "null problem rejected");

    expect(strcmp(gdn_status_string(GDN_ERR_WORKSPACE), "GDN_ERR_WORKSPACE") == 0, "status string");
    expect(strstr(gdn_version(), "sm_100a") != NULL, "version names sm_100a");

    printf("%s fwd_ws=%zu bwd_ws=%zu saved=%zu failures=%d\n", gdn_version(), fwd, bwd, saved, failures);
    return failures ? 1 : 0;
}
