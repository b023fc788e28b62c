// Router rounds on the device ("Julia-1: one score per mask token", "More than 20 options: the
// Router"): the candidates of every request stay in device memory; per round the rows of all
// groups are planned (the serializer's budget rules), packed into a varlen batch and, after the
// forward pass, narrowed by the survivor rule, with no host serialisation between rounds.
//
// Layout of the request pool (int32, uploaded once per call):
//   req[r * 6 + 0..5]  question begin, question length, state begin, state length,
//                      first label index, number of labels
//   lab[l * 2 + 0..1]  label begin, label length         (begins index `ids`)
//   ids[]              every id of every request
// Candidates of request r live at cand[lab_first(r) + j], j < nc[r] (label indices within r).

#include "common.cuh"
#include "route_kernels.h"

namespace jd {

namespace {

constexpr int RG = 20;          // candidates per group and options per row at most
constexpr int RMAX_OPT_IDS = 48;

__device__ __forceinline__ int rows_of(int nc, bool final_round) {
    if (final_round) return nc >= 2 ? 1 : 0;
    if (nc <= RG) return 0;
    const int groups = (nc + RG - 1) / RG;
    const int last = nc - RG * (groups - 1);
    return groups - (last == 1 ? 1 : 0);
}

// Exclusive scan of per-thread partial sums over one CTA of 1024 threads (two values at once).
__device__ __forceinline__ void block_scan2(int &a, int &b, int (*part)[1024]) {
    const int tid = threadIdx.x;
    part[0][tid] = a;
    part[1][tid] = b;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int va = tid >= off ? part[0][tid - off] : 0;
        const int vb = tid >= off ? part[1][tid - off] : 0;
        __syncthreads();
        part[0][tid] += va;
        part[1][tid] += vb;
        __syncthreads();
    }
    a = tid ? part[0][tid - 1] : 0;
    b = tid ? part[1][tid - 1] : 0;
}

}  // namespace

// One CTA of 1024 threads: rows of this round per request, their offsets and descriptors
// (request, first candidate, group size), and the row count in cnt[RC_ROWS].
__global__ void __launch_bounds__(1024) k_route_rows(int n_req, const int *__restrict__ nc, int final_round,
                                                     int *__restrict__ row_off, int *__restrict__ row_desc,
                                                     int *__restrict__ cnt) {
    __shared__ int part[2][1024];
    const int per = (n_req + 1023) / 1024;
    const int r0 = threadIdx.x * per, r1 = min(n_req, r0 + per);
    int nrows = 0, dummy = 0;
    for (int r = r0; r < r1; ++r) nrows += rows_of(nc[r], final_round != 0);
    int run = nrows;
    block_scan2(run, dummy, part);
    for (int r = r0; r < r1; ++r) {
        row_off[r] = run;
        const int n = nc[r];
        if (final_round) {
            if (n >= 2) {
                row_desc[3 * run] = r;
                row_desc[3 * run + 1] = 0;
                row_desc[3 * run + 2] = n;
                ++run;
            }
        } else if (n > RG) {
            for (int f = 0; f < n; f += RG) {
                const int sz = min(RG, n - f);
                if (sz < 2) continue;
                row_desc[3 * run] = r;
                row_desc[3 * run + 1] = f;
                row_desc[3 * run + 2] = sz;
                ++run;
            }
        }
    }
    if (threadIdx.x == 1023) {
        row_off[n_req] = run;
        cnt[RC_ROWS] = run;
    }
}

// One thread per row (grid over an upper bound; rows past cnt[RC_ROWS] exit): the row's plan,
// the same rules as the host serializer (strict: a failure sets cnt[RC_ERR]; non-strict: options
// to 48 ids, one common cap within the head budget, the question clipped last, the state to
// max_length).
__global__ void __launch_bounds__(128) k_route_plan(RouteArgs a, const int *__restrict__ cand,
                                                    const int *__restrict__ row_desc, RoutePlan *__restrict__ plan,
                                                    int *__restrict__ cnt) {
    const int row = blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= cnt[RC_ROWS]) return;
    const int r = row_desc[3 * row], first = row_desc[3 * row + 1], k = row_desc[3 * row + 2];
    const int *rq = a.req + 6 * r;
    RoutePlan pl;
    pl.nq = rq[1];
    pl.ns = rq[3];
    pl.k = k;
    int sum = 0, longest = 0;
    for (int j = 0; j < k; ++j) {
        const int lab = rq[4] + cand[rq[4] + first + j];
        pl.olen[j] = a.lab[2 * lab + 1];
        sum += pl.olen[j];
    }
    pl.len = 0;
    if (a.strict) {
        for (int j = 0; j < k; ++j)
            if (pl.olen[j] > RMAX_OPT_IDS) {
                atomicOr(&cnt[RC_ERR], RE_OPTION_48);
                return;
            }
        const long head = 3L + pl.nq + k + sum;
        if (head > a.head_budget) {
            atomicOr(&cnt[RC_ERR], RE_HEAD_BUDGET);
            return;
        }
        if (head + pl.ns + 1 > a.max_length) {
            atomicOr(&cnt[RC_ERR], RE_MAX_LENGTH);
            return;
        }
        pl.head = (int)head;
    } else {
        for (int j = 0; j < k; ++j) pl.olen[j] = min(pl.olen[j], RMAX_OPT_IDS);
        const long fixed = 3L + pl.nq + k;
        sum = 0;
        for (int j = 0; j < k; ++j) {
            sum += pl.olen[j];
            longest = max(longest, pl.olen[j]);
        }
        if (fixed + sum > a.head_budget) {
            int cap = 0;
            for (int c = longest; c >= 1; --c) {
                long s = 0;
                for (int j = 0; j < k; ++j) s += min(pl.olen[j], c);
                if (fixed + s <= a.head_budget) {
                    cap = c;
                    break;
                }
            }
            if (cap > 0) {
                for (int j = 0; j < k; ++j) pl.olen[j] = min(pl.olen[j], cap);
            } else {
                long s1 = 0;
                for (int j = 0; j < k; ++j) {
                    pl.olen[j] = min(pl.olen[j], 1);
                    s1 += pl.olen[j];
                }
                const long room = (long)a.head_budget - (3L + k + s1);
                if (room < 0) {
                    atomicOr(&cnt[RC_ERR], RE_HEAD_BUDGET);
                    return;
                }
                pl.nq = (int)min((long)pl.nq, room);
            }
        }
        long head = 3L + pl.nq + k;
        for (int j = 0; j < k; ++j) head += pl.olen[j];
        const long room_state = (long)a.max_length - head - 1;
        if (room_state < 0) {
            atomicOr(&cnt[RC_ERR], RE_MAX_LENGTH);
            return;
        }
        if (pl.ns > room_state) pl.ns = (int)room_state;
        pl.head = (int)head;
    }
    pl.len = pl.head + pl.ns + 1;
    plan[row] = pl;
}

// One CTA of 1024 threads: token and marker offsets of the rows (cu, opt: n_rows + 1 entries),
// the totals and the longest row into cnt.
__global__ void __launch_bounds__(1024) k_route_scan(const RoutePlan *__restrict__ plan, int *__restrict__ cu,
                                                     int *__restrict__ opt, int *__restrict__ cnt) {
    __shared__ int part[2][1024];
    __shared__ int mx[32];
    const int n = cnt[RC_ROWS];
    const int per = (n + 1023) / 1024;
    const int r0 = threadIdx.x * per, r1 = min(n, r0 + per);
    int t = 0, m = 0, longest = 0;
    for (int r = r0; r < r1; ++r) {
        t += plan[r].len;
        m += plan[r].k;
        longest = max(longest, plan[r].len);
    }
    block_scan2(t, m, part);
    for (int r = r0; r < r1; ++r) {
        cu[r] = t;
        opt[r] = m;
        t += plan[r].len;
        m += plan[r].k;
    }
    for (int o = 16; o; o >>= 1) longest = max(longest, __shfl_xor_sync(0xffffffffu, longest, o));
    if ((threadIdx.x & 31) == 0) mx[threadIdx.x >> 5] = longest;
    __syncthreads();
    if (threadIdx.x == 1023) {
        cu[n] = t;
        opt[n] = m;
        cnt[RC_TOKENS] = t;
        cnt[RC_MARKERS] = m;
        int L = 0;
        for (int w = 0; w < 32; ++w) L = max(L, mx[w]);
        cnt[RC_LONGEST] = L;
    }
}

// One CTA per row: <bos> question <eos> (<mask> option)_k <eos> state <eos>, the marker positions
// and the row type (choice).  Launched with the row count read back by the host.
__global__ void __launch_bounds__(128) k_route_write(RouteArgs a, const int *__restrict__ cand,
                                                     const int *__restrict__ row_desc,
                                                     const RoutePlan *__restrict__ plan, const int *__restrict__ cu,
                                                     const int *__restrict__ opt, int *__restrict__ tokens,
                                                     int *__restrict__ mask_pos, int *__restrict__ row_type) {
    __shared__ int pos[RG + 1];
    __shared__ int lab_beg[RG];
    const int row = blockIdx.x;
    const RoutePlan pl = plan[row];
    const int r = row_desc[3 * row], first = row_desc[3 * row + 1];
    const int *rq = a.req + 6 * r;
    const int start = cu[row];
    if (threadIdx.x == 0) {
        int p = start + 2 + pl.nq;  // first marker: after <bos>, the question and <eos>
        for (int j = 0; j < pl.k; ++j) {
            pos[j] = p;
            p += 1 + pl.olen[j];
            lab_beg[j] = a.lab[2 * (rq[4] + cand[rq[4] + first + j])];
        }
        pos[pl.k] = p;  // the <eos> after the options
        tokens[start] = a.bos;
        tokens[start + 1 + pl.nq] = a.eos;
        tokens[p] = a.eos;
        tokens[p + 1 + pl.ns] = a.eos;
        row_type[row] = 0;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < pl.nq; i += blockDim.x) tokens[start + 1 + i] = a.ids[rq[0] + i];
    for (int j = 0; j < pl.k; ++j) {
        if (threadIdx.x == 0) {
            tokens[pos[j]] = a.mask;
            mask_pos[opt[row] + j] = pos[j];
        }
        for (int i = threadIdx.x; i < pl.olen[j]; i += blockDim.x) tokens[pos[j] + 1 + i] = a.ids[lab_beg[j] + i];
    }
    const int s0 = pos[pl.k] + 1;
    for (int i = threadIdx.x; i < pl.ns; i += blockDim.x) tokens[s0 + i] = a.ids[rq[2] + i];
}

// One thread per request: the survivor rule on each scored group of this round (in order), the
// next round's candidates appended in group order; requests with 20 or fewer keep theirs.
__global__ void __launch_bounds__(128) k_route_survive(RouteArgs a, const int *__restrict__ cand,
                                                       const int *__restrict__ nc, int *__restrict__ cand_next,
                                                       int *__restrict__ nc_next, const int *__restrict__ row_off,
                                                       const int *__restrict__ opt,
                                                       const float *__restrict__ probs) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= a.n_req) return;
    const int base = a.req[6 * r + 4];
    const int n = nc[r];
    const int *c = cand + base;
    int *o = cand_next + base;
    if (n <= RG) {
        for (int j = 0; j < n; ++j) o[j] = c[j];
        nc_next[r] = n;
        return;
    }
    int out = 0, row = row_off[r];
    for (int f = 0; f < n; f += RG) {
        const int sz = min(RG, n - f);
        if (sz < 2) {
            o[out++] = c[f];
            continue;
        }
        const float *p = probs + opt[row++];
        // most and second most probable, lower index first on ties
        int best = 0;
        for (int j = 1; j < sz; ++j)
            if (p[j] > p[best]) best = j;
        int second = -1;
        for (int j = 0; j < sz; ++j)
            if (j != best && (second < 0 || p[j] > p[second])) second = j;
        bool alone = p[best] > 0.95f;
        for (int j = 0; j < sz && alone; ++j)
            if (j != best && !(p[j] < 0.045f)) alone = false;
        if (alone) {
            o[out++] = c[f + best];
        } else {
            o[out++] = c[f + min(best, second)];
            o[out++] = c[f + max(best, second)];
        }
    }
    nc_next[r] = out;
}

// One thread per request: the final call's winner (first of equal maxima), its probability and
// the final candidates and probabilities (20 slots, -1 / 0 padded); a lone candidate wins with
// probability 1 unscored.
__global__ void __launch_bounds__(128) k_route_final(RouteArgs a, const int *__restrict__ cand,
                                                     const int *__restrict__ nc, const int *__restrict__ row_off,
                                                     const int *__restrict__ opt, const float *__restrict__ probs,
                                                     int *__restrict__ winner, float *__restrict__ winner_p,
                                                     int *__restrict__ fin_c, float *__restrict__ fin_p) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= a.n_req) return;
    const int *c = cand + a.req[6 * r + 4];
    const int n = nc[r];
    for (int k = 0; k < RG; ++k) fin_c[(size_t)r * RG + k] = k < n ? c[k] : -1;
    if (n == 1) {
        winner[r] = c[0];
        winner_p[r] = 1.0f;
        for (int k = 0; k < RG; ++k) fin_p[(size_t)r * RG + k] = k == 0 ? 1.0f : 0.f;
        return;
    }
    const float *p = probs + opt[row_off[r]];
    int best = 0;
    for (int k = 1; k < n; ++k)
        if (p[k] > p[best]) best = k;
    winner[r] = c[best];
    winner_p[r] = p[best];
    for (int k = 0; k < RG; ++k) fin_p[(size_t)r * RG + k] = k < n ? p[k] : 0.f;
}

__global__ void k_route_init(int n_req, const int *__restrict__ req, int *__restrict__ cand, int *__restrict__ nc) {
    const int r = blockIdx.x;
    if (r >= n_req) return;
    const int base = req[6 * r + 4], n = req[6 * r + 5];
    for (int j = threadIdx.x; j < n; j += blockDim.x) cand[base + j] = j;
    if (threadIdx.x == 0) nc[r] = n;
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_route_init(const RouteArgs &a, int *cand, int *nc, cudaStream_t st) {
    if (a.n_req <= 0) return cudaSuccess;
    k_route_init<<<a.n_req, 128, 0, st>>>(a.n_req, a.req, cand, nc);
    return cudaGetLastError();
}

cudaError_t launch_route_plan_round(const RouteArgs &a, const int *cand, const int *nc, int final_round,
                                    int max_rows, int *row_off, int *row_desc, RoutePlan *plan, int *cu, int *opt,
                                    int *cnt, cudaStream_t st) {
    k_route_rows<<<1, 1024, 0, st>>>(a.n_req, nc, final_round, row_off, row_desc, cnt);
    if (max_rows > 0) k_route_plan<<<(max_rows + 127) / 128, 128, 0, st>>>(a, cand, row_desc, plan, cnt);
    k_route_scan<<<1, 1024, 0, st>>>(plan, cu, opt, cnt);
    return cudaGetLastError();
}

cudaError_t launch_route_write(const RouteArgs &a, const int *cand, const int *row_desc, const RoutePlan *plan,
                               const int *cu, const int *opt, int n_rows, int *tokens, int *mask_pos, int *row_type,
                               cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    k_route_write<<<n_rows, 128, 0, st>>>(a, cand, row_desc, plan, cu, opt, tokens, mask_pos, row_type);
    return cudaGetLastError();
}

cudaError_t launch_route_survive(const RouteArgs &a, const int *cand, const int *nc, int *cand_next, int *nc_next,
                                 const int *row_off, const int *opt, const float *probs, cudaStream_t st) {
    if (a.n_req <= 0) return cudaSuccess;
    k_route_survive<<<(a.n_req + 127) / 128, 128, 0, st>>>(a, cand, nc, cand_next, nc_next, row_off, opt, probs);
    return cudaGetLastError();
}

cudaError_t launch_route_final(const RouteArgs &a, const int *cand, const int *nc, const int *row_off,
                               const int *opt, const float *probs, int *winner, float *winner_p, int *fin_c,
                               float *fin_p, cudaStream_t st) {
    if (a.n_req <= 0) return cudaSuccess;
    k_route_final<<<(a.n_req + 127) / 128, 128, 0, st>>>(a, cand, nc, row_off, opt, probs, winner, winner_p, fin_c,
                                                         fin_p);
    return cudaGetLastError();
}

}  // namespace jd
