// Launchers of the device-side router rounds (route.cu).  Every launcher queues work on the
// given stream and returns the launch status; none allocates memory.
#pragma once

#include <cuda_runtime.h>

namespace jd {

// The request pool and the encoding options of a route (device pointers; layout in route.cu).
struct RouteArgs {
    int n_req;
    const int *req;   // [n_req * 6]
    const int *lab;   // [labels * 2]
    const int *ids;
    int strict, head_budget, max_length;
    int bos, eos, mask;
};

// One row of a round: its request's candidates [first, first + k) and the ids kept.
struct RoutePlan {
    int nq, ns, k, head, len;
    int olen[20];
};

// Counters of a round (device int[8]): rows, tokens, markers, longest row, error bits.
constexpr int RC_ROWS = 0, RC_TOKENS = 1, RC_MARKERS = 2, RC_LONGEST = 3, RC_ERR = 4, RC_COUNT = 8;
// Error bits (strict encoding, or a budget too small for the markers alone).
constexpr int RE_OPTION_48 = 1, RE_HEAD_BUDGET = 2, RE_MAX_LENGTH = 4;

// cand[lab_first(r) + j] = j, nc[r] = number of labels.
cudaError_t launch_route_init(const RouteArgs &a, int *cand, int *nc, cudaStream_t st);
// Rows of a round (final_round: one row per request with two or more candidates), their plans,
// token and marker offsets (cu, opt: rows + 1 entries) and the counters.  max_rows bounds the
// row count (the arrays' size).
cudaError_t launch_route_plan_round(const RouteArgs &a, const int *cand, const int *nc, int final_round,
                                    int max_rows, int *row_off, int *row_desc, RoutePlan *plan, int *cu, int *opt,
                                    int *cnt, cudaStream_t st);
// The packed rows into tokens / mask_pos / row_type (sized by the caller for the counts read back).
cudaError_t launch_route_write(const RouteArgs &a, const int *cand, const int *row_desc, const RoutePlan *plan,
                               const int *cu, const int *opt, int n_rows, int *tokens, int *mask_pos, int *row_type,
                               cudaStream_t st);
// The survivor rule on the round's probabilities; the next candidates into cand_next / nc_next.
cudaError_t launch_route_survive(const RouteArgs &a, const int *cand, const int *nc, int *cand_next, int *nc_next,
                                 const int *row_off, const int *opt, const float *probs, cudaStream_t st);
// Winners and final-call outputs of every request.
cudaError_t launch_route_final(const RouteArgs &a, const int *cand, const int *nc, const int *row_off,
                               const int *opt, const float *probs, int *winner, float *winner_p, int *fin_c,
                               float *fin_p, cudaStream_t st);

}  // namespace jd
