// Marker serialiser and packer (host).
//
// "Julia-1: one score per mask token", section "From a state to one decision":
// the question comes first, every option follows its own <mask> marker and the
// state comes last -- <bos> question <eos> (<mask> option)_k <eos> state <eos>
// -- with 2..20 options of at most 48 tokens, question plus options within a
// head budget and 8192 tokens in all; strict encoding raises on overflow.
// Rows are packed back to back without padding ("julia1 -- Rust runtime for
// Julia-1", section "Why it is faster": no padding).
//
// Budget accounting: "head" is every token before the state (bos, question,
// eos, markers, option ids, eos); the row total is head + state + final eos.
// Non-strict truncation order: options to 48 ids; then one common cap on all
// options that fits the head budget (question clipped from its end if even a
// cap of one id does not fit); then the state clipped to max_length.

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "host_common.h"

namespace {

constexpr int kMaxOptionIds = 48;
constexpr int kMinOptions = 2;
constexpr int kMaxOptions = 20;
constexpr int kMaxLength = 8192;

struct RowPlan {
    int nq = 0;                 // question ids kept
    int ns = 0;                 // state ids kept
    int olen[kMaxOptions] = {}; // option ids kept
    int head = 0;
    uint8_t trunc = 0;
};

bool ids_in_range(const int32_t *p, int n, int vocab) {
    for (int i = 0; i < n; ++i)
        if (p[i] < 0 || p[i] >= vocab) return false;
    return true;
}

jd_status plan_row(const jd_row &r, const jd_encode_opts &o, RowPlan &pl) {
    if (r.type < 0 || r.type > 2) return jd::fail(JD_ERR_INVALID_ARG, "row type %d is not choice/score/noul", r.type);
    if (r.k < kMinOptions || r.k > kMaxOptions)
        return jd::fail(JD_ERR_OPTION_COUNT, "%d options: a question takes 2 to 20", r.k);
    if (r.type == JD_NOUL && r.k != 2)
        return jd::fail(JD_ERR_OPTION_COUNT, "a noul question takes exactly two options [false, true]");
    if (r.n_question < 0 || r.n_state < 0 || (r.n_question && !r.question) || (r.n_state && !r.state) ||
        !r.options || !r.n_option_ids)
        return jd::fail(JD_ERR_INVALID_ARG, "row has a null array or a negative length");
    for (int k = 0; k < r.k; ++k)
        if (r.n_option_ids[k] < 0 || (r.n_option_ids[k] && !r.options[k]))
            return jd::fail(JD_ERR_INVALID_ARG, "option %d has a null array or a negative length", k);
    if (!ids_in_range(r.question, r.n_question, o.vocab))
        return jd::fail(JD_ERR_TOKEN_RANGE, "question: token id outside [0, %d)", o.vocab);
    for (int k = 0; k < r.k; ++k)
        if (!ids_in_range(r.options[k], r.n_option_ids[k], o.vocab))
            return jd::fail(JD_ERR_TOKEN_RANGE, "option %d: token id outside [0, %d)", k, o.vocab);
    if (!ids_in_range(r.state, r.n_state, o.vocab))
        return jd::fail(JD_ERR_TOKEN_RANGE, "state: token id outside [0, %d)", o.vocab);

    pl.nq = r.n_question;
    pl.ns = r.n_state;
    pl.trunc = 0;
    long sum = 0;
    for (int k = 0; k < r.k; ++k) { pl.olen[k] = r.n_option_ids[k]; sum += pl.olen[k]; }

    if (o.strict) {
        for (int k = 0; k < r.k; ++k)
            if (pl.olen[k] > kMaxOptionIds) return jd::fail(JD_ERR_OVERFLOW, "option %d is longer than 48 tokens", k);
        long head = 3L + pl.nq + r.k + sum;
        if (head > o.head_budget)
            return jd::fail(JD_ERR_OVERFLOW, "question plus options take %ld tokens, over the head budget %d", head,
                            o.head_budget);
        if (head + pl.ns + 1 > o.max_length) return jd::fail(JD_ERR_OVERFLOW, "sequence longer than max_length");
        pl.head = (int)head;
        return JD_OK;
    }

    // (1) options to 48 ids
    bool clipped = false;
    for (int k = 0; k < r.k; ++k)
        if (pl.olen[k] > kMaxOptionIds) { pl.olen[k] = kMaxOptionIds; clipped = true; }
    if (clipped) pl.trunc |= JD_TRUNC_OPTION_48;
    long fixed = 3L + pl.nq + r.k;
    sum = 0;
    int longest = 0;
    for (int k = 0; k < r.k; ++k) { sum += pl.olen[k]; longest = std::max(longest, pl.olen[k]); }
    if (fixed + sum > o.head_budget) {
        // (2) one common cap on every option: the largest that fits
        int cap = 0;
        for (int c = longest; c >= 1; --c) {
            long s = 0;
            for (int k = 0; k < r.k; ++k) s += std::min(pl.olen[k], c);
            if (fixed + s <= o.head_budget) { cap = c; break; }
        }
        if (cap > 0) {
            for (int k = 0; k < r.k; ++k) pl.olen[k] = std::min(pl.olen[k], cap);
            pl.trunc |= JD_TRUNC_OPTION_CAP;
        } else {
            long s1 = 0;
            bool any = false;
            for (int k = 0; k < r.k; ++k) {
                if (pl.olen[k] > 1) any = true;
                pl.olen[k] = std::min(pl.olen[k], 1);
                s1 += pl.olen[k];
            }
            if (any) pl.trunc |= JD_TRUNC_OPTION_CAP;
            long room = (long)o.head_budget - (3L + r.k + s1);
            if (room < 0) return jd::fail(JD_ERR_OVERFLOW, "head budget too small for the markers alone");
            pl.nq = (int)std::min<long>(pl.nq, room);
            pl.trunc |= JD_TRUNC_QUESTION;
        }
    }
    long head = 3L + pl.nq + r.k;
    for (int k = 0; k < r.k; ++k) head += pl.olen[k];
    long room_state = (long)o.max_length - head - 1;
    if (room_state < 0) return jd::fail(JD_ERR_OVERFLOW, "max_length too small for the head");
    if (pl.ns > room_state) { pl.ns = (int)room_state; pl.trunc |= JD_TRUNC_STATE; }
    pl.head = (int)head;
    return JD_OK;
}

template <class T>
T *xalloc(size_t n) {
    return static_cast<T *>(std::malloc(std::max<size_t>(n, 1) * sizeof(T)));
}

}  // namespace

extern "C" jd_status jd_serialize(const jd_row *rows, int32_t n_rows, const jd_encode_opts *opts, jd_batch **out,
                                  int32_t *bad_row) {
    jd::clear_error();
    if (bad_row) *bad_row = -1;
    if (!out) return jd::fail(JD_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!opts || (n_rows > 0 && !rows) || n_rows < 0) return jd::fail(JD_ERR_INVALID_ARG, "rows/opts invalid");
    if (opts->max_length < 1 || opts->max_length > kMaxLength || opts->head_budget < 1 || opts->vocab < 1)
        return jd::fail(JD_ERR_INVALID_ARG, "max_length must be in [1, 8192] and head_budget >= 1");
    const int32_t special[3] = {opts->bos, opts->eos, opts->mask};
    if (!ids_in_range(special, 3, opts->vocab))
        return jd::fail(JD_ERR_TOKEN_RANGE, "bos/eos/mask id outside [0, %d)", opts->vocab);

    std::vector<RowPlan> plans(n_rows);
    long T = 0, M = 0;
    int maxlen = 0;
    for (int r = 0; r < n_rows; ++r) {
        jd_status st = plan_row(rows[r], *opts, plans[r]);
        if (st != JD_OK) {
            if (bad_row) *bad_row = r;
            return st;
        }
        long len = plans[r].head + plans[r].ns + 1;
        T += len;
        M += rows[r].k;
        maxlen = std::max<int>(maxlen, (int)len);
    }
    if (T > 0x7fffffffL) return jd::fail(JD_ERR_INVALID_ARG, "batch too large");

    jd_batch *b = xalloc<jd_batch>(1);
    if (!b) return jd::fail(JD_ERR_INVALID_ARG, "host allocation failed");
    std::memset(b, 0, sizeof(*b));
    b->n_rows = n_rows;
    b->n_tokens = (int32_t)T;
    b->n_markers = (int32_t)M;
    b->max_row_len = maxlen;
    b->tokens = xalloc<int32_t>(T);
    b->cu_seqlens = xalloc<int32_t>(n_rows + 1);
    b->mask_pos = xalloc<int32_t>(M);
    b->opt_off = xalloc<int32_t>(n_rows + 1);
    b->row_type = xalloc<int32_t>(n_rows);
    b->head_len = xalloc<int32_t>(n_rows);
    b->trunc = xalloc<uint8_t>(n_rows);
    if (!b->tokens || !b->cu_seqlens || !b->mask_pos || !b->opt_off || !b->row_type || !b->head_len || !b->trunc) {
        jd_batch_free(b);
        return jd::fail(JD_ERR_INVALID_ARG, "host allocation failed");
    }

    int32_t *t = b->tokens;
    int32_t pos = 0, m = 0;
    b->cu_seqlens[0] = 0;
    b->opt_off[0] = 0;
    for (int r = 0; r < n_rows; ++r) {
        const jd_row &row = rows[r];
        const RowPlan &pl = plans[r];
        int32_t start = pos;
        t[pos++] = opts->bos;
        if (pl.nq) std::memcpy(t + pos, row.question, sizeof(int32_t) * pl.nq);
        pos += pl.nq;
        t[pos++] = opts->eos;
        for (int k = 0; k < row.k; ++k) {
            b->mask_pos[m++] = pos;
            t[pos++] = opts->mask;
            if (pl.olen[k]) std::memcpy(t + pos, row.options[k], sizeof(int32_t) * pl.olen[k]);
            pos += pl.olen[k];
        }
        t[pos++] = opts->eos;
        if (pl.ns) std::memcpy(t + pos, row.state, sizeof(int32_t) * pl.ns);
        pos += pl.ns;
        t[pos++] = opts->eos;
        b->cu_seqlens[r + 1] = pos;
        b->opt_off[r + 1] = m;
        b->row_type[r] = row.type;
        b->head_len[r] = pl.head;
        b->trunc[r] = pl.trunc;
        (void)start;
    }
    *out = b;
    return JD_OK;
}

extern "C" void jd_batch_free(jd_batch *b) {
    if (!b) return;
    std::free(b->tokens);
    std::free(b->cu_seqlens);
    std::free(b->mask_pos);
    std::free(b->opt_off);
    std::free(b->row_type);
    std::free(b->head_len);
    std::free(b->trunc);
    std::free(b);
}

extern "C" jd_status jd_batch_info(const jd_batch *b, jd_encoding_info *per_row) {
    jd::clear_error();
    if (!b || !per_row) return jd::fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (b->n_rows > 0 && (!b->cu_seqlens || !b->opt_off || !b->head_len || !b->trunc))
        return jd::fail(JD_ERR_INVALID_ARG, "not a host batch from jd_serialize (no head_len / trunc)");
    for (int r = 0; r < b->n_rows; ++r) {
        jd_encoding_info &e = per_row[r];
        e.length = b->cu_seqlens[r + 1] - b->cu_seqlens[r];
        e.head_length = b->head_len[r];
        e.state_length = e.length - e.head_length - 1;
        e.n_options = b->opt_off[r + 1] - b->opt_off[r];
        e.truncated = b->trunc[r];
    }
    return JD_OK;
}

extern "C" jd_status jd_rows_encoding_info(const jd_row *rows, int32_t n_rows, const jd_encode_opts *opts,
                                           jd_encoding_info *per_row, int32_t *bad_row) {
    if (bad_row) *bad_row = -1;
    if (!per_row && n_rows > 0) {
        jd::clear_error();
        return jd::fail(JD_ERR_INVALID_ARG, "per_row is NULL");
    }
    jd_batch *b = nullptr;
    jd_status s = jd_serialize(rows, n_rows, opts, &b, bad_row);
    if (s != JD_OK) return s;
    s = jd_batch_info(b, per_row);
    jd_batch_free(b);
    return s;
}
