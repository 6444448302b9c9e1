/* A plain C99 caller of the library's host-only entry points: built and run
 * by tests/test_c_abi.py, so that the header is checked as C (not C++) and
 * the exported symbols are used through the C ABI alone, with no Python in
 * between.  Prints one "key value..." line per result; exits 0 when every
 * call returned what it should. */
#include <stdio.h>
#include <string.h>

#include "pv.h"

static int failures = 0;

static void expect(int ok, const char* what) {
    if (!ok) {
        char msg[256];
        pv_last_error(msg, sizeof msg);
        printf("FAIL %s (%s)\n", what, msg);
        ++failures;
    }
}

int main(void) {
    printf("version %s\n", pv_version());

    /* the steady-state geometry: 30 layers, 24 x 128, 40 x 22 tokens per
     * latent frame, 3 first frames, 18 ring slots, 4 steps, one stream */
    pv_kv_config c;
    memset(&c, 0, sizeof c);
    c.layers = 30;
    c.heads = 24;
    c.head_dim = 128;
    c.frame_w = 40;
    c.frame_h = 22;
    c.first_frames = 3;
    c.ring_slots = 18;
    c.steps = 4;
    c.max_streams = 1;
    c.rope_pairs_t = 22;
    c.rope_pairs_h = 21;
    c.rope_pairs_w = 21;
    c.max_frames = 64;
    c.rope_theta = 10000.0;
    size_t kv_bytes = 0, ws_bytes = 0;
    expect(pv_kv_required_bytes(&c, &kv_bytes, &ws_bytes) == PV_OK, "required_bytes");
    printf("kv_bytes %zu\n", kv_bytes);

    /* a bookkeeping-only handle walked to chunk 28 */
    pv_kv h = NULL;
    expect(pv_kv_init(&h, &c, NULL, 0, NULL, 0) == PV_OK, "init");
    expect(pv_kv_begin_chunk(h, 0, 3) == PV_OK, "first chunk");
    expect(pv_kv_begin_sink(h, 0) == PV_OK, "sink pass");
    for (int j = 1; j <= 28; ++j) expect(pv_kv_begin_chunk(h, 0, 1) == PV_OK, "next chunk");
    pv_kv_state st;
    expect(pv_kv_get_state(h, 0, &st) == PV_OK, "get_state");
    printf("state %d %d %d %d %d %d\n", st.phase, st.chunk, st.fill, st.slot, st.frame0,
           st.n_keys);
    /* misuse is a status, not an abort: three frames after the first chunk */
    const pv_status bad = pv_kv_begin_chunk(h, 0, 3);
    char msg[256];
    pv_last_error(msg, sizeof msg);
    printf("misuse %d %d\n", (int)bad, (int)(strlen(msg) > 0));
    expect(bad != PV_OK, "misuse rejected");
    expect(pv_kv_destroy(h) == PV_OK, "destroy");

    /* the attention plan of the steady chunk */
    const int n_q = 880, n_k = 18480;
    int grid = 0, mode = -1;
    long long ranges[161];
    expect(pv_attn_plan(1, &n_q, &n_k, 24, 148, 4 * 160, &grid, &mode, ranges) == PV_OK, "plan");
    printf("plan %d %d %lld %lld\n", grid, mode, ranges[37], ranges[grid]);

    /* the shifted 40-step schedule of the blog's chapter 1 */
    double sig[41];
    int ts[40];
    expect(pv_sigma_schedule(40, 12.0, 0.0, sig, ts) == PV_OK, "sigma_schedule");
    printf("timesteps %d %d %d %d %d %d\n", ts[0], ts[1], ts[2], ts[3], ts[4], ts[5]);
    printf("sigma_end %.17g\n", sig[40]);

    printf("failures %d\n", failures);
    return failures == 0 ? 0 : 1;
}
