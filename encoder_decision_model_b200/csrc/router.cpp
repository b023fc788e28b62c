// Narrowing tournament for choice questions with more candidates than one
// call takes ("Julia-1: one score per mask token", "More than 20 options: the
// Router"; "Julia-1 MLX", "API": up to 4,096 options).
//
// Per round, every request still holding more than 20 candidates is split, in
// order, into consecutive groups of at most 20; all groups of all requests are
// scored in one batch; a group keeps its winner alone when that probability is
// above 0.95 and every other is below 0.045, otherwise its two most probable
// candidates (lower index first on ties), in their original order; a group of
// one candidate passes through unscored.  When 20 or fewer remain, one final
// call per request picks the winner.  jd_route_host scores through the model;
// jd_route_scored runs the same tournament on a caller's scoring callback.

#include <algorithm>
#include <cstring>
#include <vector>

#include "host_common.h"

namespace {

constexpr int kGroup = 20;
constexpr int kMaxLabels = 4096;

struct Pending {
    int req;
    int first;  // index into the request's candidate list
    int size;
};

// Scores rows in chunks that fit the model's capacity; probs[m] in row order.
jd_status score_rows(jd_model *m, const std::vector<jd_row> &rows, const jd_encode_opts *opts, void *stream,
                     int32_t max_tokens, int32_t max_rows, int32_t max_markers, std::vector<float> &probs) {
    probs.clear();
    size_t i = 0;
    while (i < rows.size()) {
        // grow the chunk greedily within the capacity (serialised lengths bounded by max_length)
        size_t j = i;
        long toks = 0, marks = 0;
        while (j < rows.size() && (long)(j - i) < max_rows) {
            long len = 3L + rows[j].n_question + rows[j].k + rows[j].n_state;
            for (int k = 0; k < rows[j].k; ++k) len += rows[j].n_option_ids[k];
            len = std::min<long>(len, opts->max_length);
            if (j > i && (toks + len > max_tokens || marks + rows[j].k > max_markers)) break;
            toks += len;
            marks += rows[j].k;
            ++j;
        }
        jd_batch *hb = nullptr;
        int32_t bad = -1;
        jd_status s = jd_serialize(rows.data() + i, (int32_t)(j - i), opts, &hb, &bad);
        if (s != JD_OK) return s;
        std::vector<float> p(hb->n_markers);
        std::vector<int32_t> choice(hb->n_rows);
        std::vector<float> score(hb->n_rows), noul(hb->n_rows), maxp(hb->n_rows);
        jd_host_outputs ho{nullptr, p.data(), choice.data(), score.data(), noul.data(), maxp.data(), 0, 0};
        s = jd_decide_packed_host(m, hb, &ho, stream);
        jd_batch_free(hb);
        if (s != JD_OK) return s;
        probs.insert(probs.end(), p.begin(), p.end());
        i = j;
    }
    return JD_OK;
}

void survivors(const float *p, int n, std::vector<int> &keep) {
    std::vector<int> order(n);
    for (int i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return p[a] > p[b]; });
    const int best = order[0];
    bool alone = p[best] > 0.95f;
    for (int i = 0; i < n && alone; ++i)
        if (i != best && !(p[i] < 0.045f)) alone = false;
    keep.clear();
    if (alone) {
        keep.push_back(best);
    } else {
        keep.push_back(std::min(order[0], order[1]));
        keep.push_back(std::max(order[0], order[1]));
    }
}

// Scoring through the model (jd_route_host): chunks within the capacity, serialised with opts.
struct ModelScorer {
    jd_model *m;
    const jd_encode_opts *opts;
    void *stream;
    int32_t max_tokens, max_rows, max_markers;
};

jd_status model_scorer(void *user, const jd_row *rows, int32_t n_rows, float *probs) {
    const ModelScorer &ms = *static_cast<const ModelScorer *>(user);
    std::vector<jd_row> v(rows, rows + n_rows);
    std::vector<float> p;
    jd_status s = score_rows(ms.m, v, ms.opts, ms.stream, ms.max_tokens, ms.max_rows, ms.max_markers, p);
    if (s != JD_OK) return s;
    size_t n_opts = 0;
    for (int32_t i = 0; i < n_rows; ++i) n_opts += (size_t)rows[i].k;
    if (p.size() != n_opts) return jd::fail(JD_ERR_INVALID_ARG, "scored %zu options for %zu", p.size(), n_opts);
    std::copy(p.begin(), p.end(), probs);
    return JD_OK;
}

// One round's scoring: probs gets every option of every row, in row order.
jd_status score(jd_route_scorer scorer, void *user, const std::vector<jd_row> &rows, size_t n_opts,
                std::vector<float> &probs) {
    probs.assign(n_opts, 0.f);
    if (rows.empty()) return JD_OK;
    jd_status s = scorer(user, rows.data(), (int32_t)rows.size(), probs.data());
    if (s != JD_OK && jd_last_error()[0] == 0) jd::fail(s, "the scorer returned %d", (int)s);
    return s;
}

// The tournament, scoring each round's rows through `scorer`.
jd_status route_core(const jd_route_request *reqs, int32_t n_requests, jd_route_scorer scorer, void *user,
                     jd_route_outputs *out) {
    if (!scorer || !out || (n_requests > 0 && !reqs) || n_requests < 0)
        return jd::fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (n_requests > 0 && !out->winner) return jd::fail(JD_ERR_INVALID_ARG, "out->winner is NULL");
    if (out->rows_per_round && out->max_rounds < 0) return jd::fail(JD_ERR_INVALID_ARG, "max_rounds < 0");
    for (int r = 0; r < n_requests; ++r)
        if (reqs[r].n_labels < 1 || reqs[r].n_labels > kMaxLabels || !reqs[r].labels || !reqs[r].n_label_ids)
            return jd::fail(JD_ERR_INVALID_ARG, "request %d: 1..4096 labels required", r);

    std::vector<std::vector<int>> cands(n_requests);
    for (int r = 0; r < n_requests; ++r) {
        cands[r].resize(reqs[r].n_labels);
        for (int i = 0; i < reqs[r].n_labels; ++i) cands[r][i] = i;
    }
    int round = 0;
    std::vector<const int32_t *> optp;
    std::vector<int32_t> optn;
    std::vector<float> probs;
    std::vector<int> keep;
    auto build_row = [&](int r, const int *idx, int n, size_t slot) {
        for (int k = 0; k < n; ++k) {
            optp[slot + k] = reqs[r].labels[idx[k]];
            optn[slot + k] = reqs[r].n_label_ids[idx[k]];
        }
        jd_row row;
        row.state = reqs[r].state;
        row.n_state = reqs[r].n_state;
        row.question = reqs[r].question;
        row.n_question = reqs[r].n_question;
        row.options = optp.data() + slot;
        row.n_option_ids = optn.data() + slot;
        row.k = n;
        row.type = JD_CHOICE;
        return row;
    };

    for (;;) {
        std::vector<Pending> pend;
        size_t n_opts = 0;
        for (int r = 0; r < n_requests; ++r) {
            const int nc = (int)cands[r].size();
            if (nc <= kGroup) continue;
            for (int f = 0; f < nc; f += kGroup) {
                const int sz = std::min(kGroup, nc - f);
                pend.push_back({r, f, sz});
                if (sz > 1) n_opts += sz;
            }
        }
        if (pend.empty()) break;
        optp.assign(n_opts, nullptr);
        optn.assign(n_opts, 0);
        std::vector<jd_row> rows;
        std::vector<int> row_of(pend.size(), -1);
        size_t slot = 0;
        for (size_t g = 0; g < pend.size(); ++g) {
            if (pend[g].size < 2) continue;
            row_of[g] = (int)rows.size();
            rows.push_back(build_row(pend[g].req, cands[pend[g].req].data() + pend[g].first, pend[g].size, slot));
            slot += pend[g].size;
        }
        jd_status s = score(scorer, user, rows, n_opts, probs);
        if (s != JD_OK) return s;
        if (out->rows_per_round && round < out->max_rounds) out->rows_per_round[round] = (int32_t)rows.size();
        ++round;
        std::vector<std::vector<int>> next(n_requests);
        for (int r = 0; r < n_requests; ++r)
            if ((int)cands[r].size() <= kGroup) next[r] = cands[r];
        size_t off = 0;
        for (size_t g = 0; g < pend.size(); ++g) {
            const Pending &pg = pend[g];
            const int *c = cands[pg.req].data() + pg.first;
            if (row_of[g] < 0) {
                next[pg.req].push_back(c[0]);
                continue;
            }
            survivors(probs.data() + off, pg.size, keep);
            for (int k : keep) next[pg.req].push_back(c[k]);
            off += pg.size;
        }
        cands.swap(next);
    }

    // final call per request with two or more candidates left
    size_t n_opts = 0;
    for (int r = 0; r < n_requests; ++r)
        if (cands[r].size() > 1) n_opts += cands[r].size();
    optp.assign(n_opts, nullptr);
    optn.assign(n_opts, 0);
    std::vector<jd_row> rows;
    std::vector<int> row_req;
    size_t slot = 0;
    for (int r = 0; r < n_requests; ++r) {
        const int nc = (int)cands[r].size();
        if (out->final_candidates)
            for (int k = 0; k < kGroup; ++k) out->final_candidates[(size_t)r * kGroup + k] = k < nc ? cands[r][k] : -1;
        if (nc == 1) {
            out->winner[r] = cands[r][0];
            if (out->winner_p) out->winner_p[r] = 1.0f;
            if (out->final_probs)
                for (int k = 0; k < kGroup; ++k) out->final_probs[(size_t)r * kGroup + k] = k == 0 ? 1.0f : 0.f;
            continue;
        }
        rows.push_back(build_row(r, cands[r].data(), nc, slot));
        row_req.push_back(r);
        slot += nc;
    }
    if (!rows.empty()) {
        jd_status s = score(scorer, user, rows, n_opts, probs);
        if (s != JD_OK) return s;
        if (out->rows_per_round && round < out->max_rounds) out->rows_per_round[round] = (int32_t)rows.size();
        ++round;
        size_t off = 0;
        for (size_t i = 0; i < rows.size(); ++i) {
            const int r = row_req[i];
            const int nc = (int)cands[r].size();
            int best = 0;
            for (int k = 1; k < nc; ++k)
                if (probs[off + k] > probs[off + best]) best = k;
            out->winner[r] = cands[r][best];
            if (out->winner_p) out->winner_p[r] = probs[off + best];
            if (out->final_probs)
                for (int k = 0; k < kGroup; ++k) out->final_probs[(size_t)r * kGroup + k] = k < nc ? probs[off + k] : 0.f;
            off += nc;
        }
    }
    out->n_rounds = round;
    return JD_OK;
}

}  // namespace

extern "C" jd_status jd_route_scored(const jd_route_request *requests, int32_t n_requests, jd_route_scorer scorer,
                                     void *user, jd_route_outputs *out) {
    jd::clear_error();
    return route_core(requests, n_requests, scorer, user, out);
}

extern "C" jd_status jd_route_host(jd_model *m, const jd_route_request *reqs, int32_t n_requests,
                                   const jd_encode_opts *opts, int32_t max_tokens, int32_t max_rows,
                                   int32_t max_markers, jd_route_outputs *out, void *stream) {
    jd::clear_error();
    if (!m || !opts || !out || (n_requests > 0 && !reqs) || n_requests < 0)
        return jd::fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (max_tokens < 1 || max_rows < 1 || max_markers < kGroup)
        return jd::fail(JD_ERR_INVALID_ARG, "chunk capacities too small");
    ModelScorer ms{m, opts, stream, max_tokens, max_rows, max_markers};
    return route_core(reqs, n_requests, model_scorer, &ms, out);
}
