/*
 * A plain C99 caller of liblq's C ABI (include/lq.h), with no CUDA or C++
 * headers: the header compiles as C, the library links, and the host-only
 * calls behave as declared -- workspace sizing and layout, config
 * validation, create / destroy, the host-side refusals of calls made out of
 * order or with bad pointers, the export's argument checks, resume
 * validation and the error text.  No call
 * here launches a kernel or touches a device pointer (create only records
 * the workspace address), so it runs on a machine without a GPU.
 * Exit status 0 when every check holds; otherwise the failing line.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "lq.h"

static int failures = 0;
#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "check failed, line %d: %s\n", __LINE__, #cond); \
            ++failures;                                               \
        }                                                             \
    } while (0)

static lq_config config(int32_t batch, int32_t heads, int32_t d, int32_t window) {
    lq_config c;
    memset(&c, 0, sizeof(c));
    c.batch = batch;
    c.heads = heads;
    c.d_k = d;
    c.d_v = d;
    c.window = window;
    c.n_comp_rows = 2;
    c.n_comp_cols = 2;
    c.gate = LQ_GATE_SCALAR;
    c.mode = LQ_MODE_WINDOW;
    c.smooth = 1;
    c.select = LQ_SELECT_L2;
    c.in_dtype = LQ_DTYPE_BF16;
    c.ragged = 0;
    return c;
}

int main(void) {
    /* sizing and layout of the default decode workload (64 x 32 heads, d = 128, W = 64) */
    lq_config cfg = config(64, 32, 128, 64);
    const size_t need = lq_workspace_bytes(&cfg);
    lq_layout lay;
    CHECK(need > 0);
    CHECK(lq_workspace_layout(&cfg, &lay) == LQ_OK);
    CHECK(lay.total_bytes == need);
    CHECK(lay.codes != LQ_ABSENT && lay.codes % 256 == 0);
    CHECK(lay.state_f32 == LQ_ABSENT);                 /* windowed mode keeps no FP32 state */
    CHECK(lay.fill == LQ_ABSENT);                      /* shared window phase */
    CHECK(lay.comp_index_stride == 4 && lay.window_pad == 64);

    /* invalid configs: sized 0 and refused */
    lq_config bad = cfg;
    bad.d_k = bad.d_v = 96;
    CHECK(lq_workspace_bytes(&bad) == 0);
    CHECK(lq_workspace_layout(&bad, &lay) != LQ_OK);
    bad = cfg;
    bad.n_comp_rows = 9;
    CHECK(lq_workspace_bytes(&bad) == 0);
    CHECK(lq_workspace_bytes(NULL) == 0);

    /* create checks the workspace; the address is recorded, never dereferenced here */
    lq_handle h = NULL;
    void *fake = (void *)(uintptr_t)(1u << 20);
    CHECK(lq_state_create(&cfg, NULL, need, &h) == LQ_ERR_WORKSPACE);
    CHECK(lq_state_create(&cfg, (void *)((uintptr_t)fake + 16), need, &h) == LQ_ERR_WORKSPACE);
    CHECK(lq_state_create(&cfg, fake, need - 1, &h) == LQ_ERR_WORKSPACE);
    CHECK(lq_last_error_string() != NULL && strlen(lq_last_error_string()) > 0);
    CHECK(lq_state_create(&cfg, fake, need, &h) == LQ_OK && h != NULL);
    CHECK(lq_window_fill(h) == 0);

    /* out of order and bad pointers are refused on the host, before any launch */
    const void *p = (const void *)(uintptr_t)(1u << 21);
    const float *pf = (const float *)p;
    float *po = (float *)(uintptr_t)(1u << 21);
    CHECK(lq_decode_step(h, p, p, p, pf, pf, po, NULL) == LQ_ERR_STATE);
    CHECK(lq_window_flush(h, NULL) == LQ_ERR_STATE);
    CHECK(lq_decode_step(h, NULL, p, p, pf, pf, po, NULL) == LQ_ERR_INVALID_ARG);
    CHECK(lq_decode_step(h, (const void *)((uintptr_t)p + 8), p, p, pf, pf, po, NULL) == LQ_ERR_INVALID_ARG);
    CHECK(lq_decode_step_active(h, p, p, p, pf, pf, NULL, po, NULL) == LQ_ERR_STATE);   /* not ragged */

    /* export: a NULL destination set, a region the mode lacks and a call
     * before the prefill are refused on the host, before any copy */
    lq_export ex;
    memset(&ex, 0, sizeof(ex));
    CHECK(lq_state_export(NULL, &ex, NULL) == LQ_ERR_INVALID_ARG);
    CHECK(lq_state_export(h, NULL, NULL) == LQ_ERR_INVALID_ARG);
    ex.state_f32 = po;                                 /* windowed handles keep no FP32 state */
    CHECK(lq_state_export(h, &ex, NULL) == LQ_ERR_INVALID_ARG);
    ex.state_f32 = NULL;
    ex.codes = (int8_t *)po;
    CHECK(lq_state_export(h, &ex, NULL) == LQ_ERR_STATE);

    /* resume: the shared phase may hold 0..W buffered tokens */
    CHECK(lq_state_resume(h, -1) == LQ_ERR_INVALID_ARG);
    CHECK(lq_state_resume(h, 65) == LQ_ERR_INVALID_ARG);
    CHECK(lq_state_resume(h, 17) == LQ_OK);
    CHECK(lq_window_fill(h) == 17);

    CHECK(lq_state_destroy(h) == LQ_OK);
    CHECK(lq_state_destroy(NULL) == LQ_ERR_INVALID_ARG);
    CHECK(lq_window_fill(NULL) == -1);
    CHECK(lq_prefill_state(NULL, NULL, NULL) == LQ_ERR_INVALID_ARG);

    /* a ragged handle keeps its counts on the device: fill() reports -1 */
    lq_config rag = config(3, 2, 64, 8);
    rag.ragged = 1;
    const size_t need_r = lq_workspace_bytes(&rag);
    CHECK(need_r > 0);
    CHECK(lq_workspace_layout(&rag, &lay) == LQ_OK && lay.fill != LQ_ABSENT);
    lq_handle hr = NULL;
    CHECK(lq_state_create(&rag, fake, need_r, &hr) == LQ_OK);
    CHECK(lq_window_fill(hr) == -1);
    CHECK(lq_state_resume(hr, 1) == LQ_ERR_INVALID_ARG);
    CHECK(lq_state_resume(hr, 0) == LQ_OK);
    CHECK(lq_state_destroy(hr) == LQ_OK);

    if (failures == 0) printf("c abi ok\n");
    return failures == 0 ? 0 : 1;
}
