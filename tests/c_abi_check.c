/* A plain C11 client of include/julia_decide.h: the header must compile as C and
 * the library must be callable from C.  It serializes the explainer's worked
 * example ("Julia-1: one score per mask token", "From a state to one decision":
 * a 10-id question, options of 4, 3 and 4 ids and a 9-id state give markers at
 * 12, 17 and 21 in 37 tokens), reads the encoding report, and checks the error
 * paths that need no device.  Prints "ok" and exits 0 on success. */
#include <stdio.h>
#include <string.h>

#include "julia_decide.h"

#define CHECK(c)                                                   \
    do {                                                           \
        if (!(c)) {                                                \
            fprintf(stderr, "check failed line %d: %s\n", __LINE__, #c); \
            return 1;                                              \
        }                                                          \
    } while (0)

/* A scorer that gives every option of a row the same probability: no group
 * ever keeps a single winner, so each keeps its first two candidates. */
static jd_status uniform_scorer(void *user, const jd_row *rows, int32_t n_rows, float *probs) {
    int *calls = (int *)user;
    ++*calls;
    for (int32_t r = 0; r < n_rows; ++r)
        for (int32_t k = 0; k < rows[r].k; ++k) *probs++ = 1.0f / (float)rows[r].k;
    return JD_OK;
}

int main(void) {
    int32_t q[10], o0[4], o1[3], o2[4], st[9];
    for (int i = 0; i < 10; ++i) q[i] = 100 + i;
    for (int i = 0; i < 4; ++i) o0[i] = 200 + i;
    for (int i = 0; i < 3; ++i) o1[i] = 300 + i;
    for (int i = 0; i < 4; ++i) o2[i] = 400 + i;
    for (int i = 0; i < 9; ++i) st[i] = 500 + i;
    const int32_t *opts_ids[3] = {o0, o1, o2};
    const int32_t n_ids[3] = {4, 3, 4};
    jd_row row = {st, 9, q, 10, opts_ids, n_ids, 3, JD_CHOICE};
    jd_encode_opts eo = {1024, 512, 1, 2, 1, 4, 256000};

    CHECK(strstr(jd_version(), "sm_100a") != NULL);

    jd_batch *b = NULL;
    int32_t bad = 7;
    CHECK(jd_serialize(&row, 1, &eo, &b, &bad) == JD_OK);
    CHECK(bad == -1 && b != NULL);
    CHECK(b->n_rows == 1 && b->n_tokens == 37 && b->n_markers == 3);
    CHECK(b->mask_pos[0] == 12 && b->mask_pos[1] == 17 && b->mask_pos[2] == 21);
    CHECK(b->tokens[0] == eo.bos && b->tokens[11] == eo.eos && b->tokens[36] == eo.eos);
    CHECK(b->tokens[12] == eo.mask && b->tokens[13] == 200);

    jd_encoding_info info;
    CHECK(jd_batch_info(b, &info) == JD_OK);
    CHECK(info.length == 37 && info.head_length == 27 && info.state_length == 9);
    CHECK(info.n_options == 3 && info.truncated == 0);
    jd_batch_free(b);

    jd_encoding_info info2;
    CHECK(jd_rows_encoding_info(&row, 1, &eo, &info2, &bad) == JD_OK);
    CHECK(memcmp(&info, &info2, sizeof info) == 0);

    /* always errors: one option; a special id outside the vocabulary */
    jd_row one = row;
    one.k = 1;
    CHECK(jd_serialize(&one, 1, &eo, &b, &bad) == JD_ERR_OPTION_COUNT && b == NULL && bad == 0);
    CHECK(strlen(jd_last_error()) > 0);
    jd_encode_opts bad_mask = eo;
    bad_mask.mask = 256000;
    CHECK(jd_serialize(&row, 1, &bad_mask, &b, &bad) == JD_ERR_TOKEN_RANGE && bad == -1);
    /* strict: a head over budget */
    jd_encode_opts tight = eo;
    tight.head_budget = 26;
    CHECK(jd_serialize(&row, 1, &tight, &b, &bad) == JD_ERR_OVERFLOW);
    /* non-strict: the same budget caps the options and reports it */
    tight.strict = 0;
    CHECK(jd_rows_encoding_info(&row, 1, &tight, &info, &bad) == JD_OK);
    CHECK(info.head_length <= 26 && (info.truncated & JD_TRUNC_OPTION_CAP));

    /* the Router on the explainer's example ("More than 20 options: the Router"):
     * sixty labels cost three calls in the first round and one final call */
    int32_t lab_ids[60];
    const int32_t *labels[60];
    int32_t lab_n[60];
    for (int i = 0; i < 60; ++i) {
        lab_ids[i] = 1000 + i;
        labels[i] = &lab_ids[i];
        lab_n[i] = 1;
    }
    jd_route_request req = {st, 9, q, 10, labels, lab_n, 60};
    int32_t winner = -1, rounds[4] = {0, 0, 0, 0}, fc[20];
    float wp = 0.f;
    jd_route_outputs ro = {&winner, &wp, fc, NULL, rounds, 4, 0};
    int scorer_calls = 0;
    CHECK(jd_route_scored(&req, 1, uniform_scorer, &scorer_calls, &ro) == JD_OK);
    CHECK(ro.n_rounds == 2 && rounds[0] == 3 && rounds[1] == 1 && scorer_calls == 2);
    /* groups 0-19, 20-39, 40-59 keep their first two; the final call's tie goes to the first */
    CHECK(fc[0] == 0 && fc[1] == 1 && fc[2] == 20 && fc[3] == 21 && fc[4] == 40 && fc[5] == 41 && fc[6] == -1);
    CHECK(winner == 0 && wp > 0.16f && wp < 0.17f);
    ro.winner = NULL;
    CHECK(jd_route_scored(&req, 1, uniform_scorer, &scorer_calls, &ro) == JD_ERR_INVALID_ARG);

    /* a model needs arguments; NULL ones are refused before any device work */
    jd_model *m = NULL;
    CHECK(jd_model_create(NULL, "w.jdw", 0, &m) == JD_ERR_INVALID_ARG && m == NULL);
    jd_model_destroy(NULL);
    printf("ok\n");
    return 0;
}
