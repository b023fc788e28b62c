// Varlen bidirectional attention inside each packed row.
//
// "Julia-1 MLX", "Performance": every third layer attends globally, the others
// within +-64 tokens (local_attention = 128); a blockwise evaluation "computes
// the same attention exactly".  "julia1 -- Rust runtime for Julia-1", "Why it
// is faster": sequences are packed back to back without padding, sliding-
// window layers compute only their band.
//
// Work unit: one 64-query block of one row and one head.  The key/value tiles
// visited are the row's tiles (global) or the three 64-key tiles covering
// [q0 - 64, q0 + 128) (local); tiles never cross into the scores of another
// row (keys outside the row are masked before the softmax).
//
// BF16 path: 4 warps, each owning 16 queries; Q, K, V tiles (64 x 64 bf16,
// 128-byte swizzle) arrive by TMA into a two-stage ring; S = Q K^T and O += P V
// run on mma.sync m16n8k16 with FP32 accumulation; the softmax is the online
// (running max / running sum) form kept per warp in registers.
// FP32 path: the same tiling with plain FP32 arithmetic (validation mode).

#include "common.cuh"
#include "kernels.h"

namespace jd {

constexpr int BQ = 64;   // queries per work unit
constexpr int BK = 64;   // keys per tile

__device__ __forceinline__ int find_row(const int *qb_off, int n_rows, int tile) {
    int lo = 0, hi = n_rows - 1;  // largest r with qb_off[r] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (qb_off[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// ------------------------------------------------------------------ mma.sync helpers

// 2^x by the special-function unit (ex2.approx.ftz: results below 2^-126 flush to 0, 2^-inf = 0)
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// P (FP16) times V (FP16): the second product of every attention kernel here
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// byte offset of (row, 16-byte chunk) in a 64-wide bf16 tile with 128-byte swizzle
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <bool LOCAL>
__global__ void __launch_bounds__(128)
    k_attn_bf16(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ out, const int *__restrict__ cu,
                const int *__restrict__ qb_off, int n_rows, int window, unsigned *status) {
    // five 8 KB tiles whose 128-byte swizzle assumes a 1024-byte aligned base
    extern __shared__ uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 5 * 8192);  // 0: Q, 1..2: K/V stages
    uint8_t *sQ = sm;
    uint8_t *sK[2] = {sm + 8192, sm + 2 * 8192};
    uint8_t *sV[2] = {sm + 3 * 8192, sm + 4 * 8192};

    const int tile = blockIdx.x, h = blockIdx.y;
    if (tile >= qb_off[n_rows]) return;
    const int row = find_row(qb_off, n_rows, tile);
    const int cs = cu[row], ce = cu[row + 1];
    const int q0 = cs + (tile - qb_off[row]) * BQ;
    int kv0 = cs, kv1 = ce;
    if (LOCAL) {
        kv0 = max(cs, q0 - window);
        kv1 = min(ce, q0 + BQ + window);
    }
    const int ntiles = (kv1 - kv0 + BK - 1) / BK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[0], 8192);
        tma_load_2d(sQ, &tm, &bars[0], h * DH, q0);
        for (int t = 0; t < 2 && t < ntiles; ++t) {
            mbar_arrive_expect_tx(&bars[1 + t], 16384);
            tma_load_2d(sK[t], &tm, &bars[1 + t], D + h * DH, kv0 + t * BK);
            tma_load_2d(sV[t], &tm, &bars[1 + t], 2 * D + h * DH, kv0 + t * BK);
        }
    }
    __syncthreads();

    const float sl2 = 0.125f * 1.4426950408889634f;  // 1/sqrt(64) * log2(e)
    const int g = lane >> 2, tq = lane & 3;
    const int qi0 = q0 + warp * 16 + g, qi1 = qi0 + 8;

    bool ok = mbar_wait(&bars[0], 0, status);
    uint32_t qf[4][4];
    {
        const uint32_t base = smem_u32(sQ);
        const int r = warp * 16 + (lane & 15);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            ldsm_x4(base + sw128(r, kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }

    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    for (int t = 0; t < ntiles && ok; ++t) {
        const int s = t & 1;
        if (!mbar_wait(&bars[1 + s], (t >> 1) & 1, status)) { ok = false; break; }
        const uint32_t kb = smem_u32(sK[s]), vb = smem_u32(sV[s]);
        const int kt0 = kv0 + t * BK;

        float sc[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            const int kr = np * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kb + sw128(kr, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
                mma_bf16(sc[2 * np], qf[kk], b0, b1);
                mma_bf16(sc[2 * np + 1], qf[kk], b2, b3);
            }
        }
        // mask + running max
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kj = kt0 + j * 8 + 2 * tq + e;
                const bool in_row = kj >= cs && kj < ce;
                bool v0 = in_row, v1 = in_row;
                if (LOCAL) {
                    v0 = v0 && abs(qi0 - kj) <= window;
                    v1 = v1 && abs(qi1 - kj) <= window;
                }
                sc[j][e] = v0 ? sc[j][e] * sl2 : -INFINITY;
                sc[j][2 + e] = v1 ? sc[j][2 + e] * sl2 : -INFINITY;
                mx0 = fmaxf(mx0, sc[j][e]);
                mx1 = fmaxf(mx1, sc[j][2 + e]);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
        const float c0 = exp2f(m0 - mu0), c1 = exp2f(m1 - mu1);
        m0 = mn0;
        m1 = mn1;
        float rs0 = 0.f, rs1 = 0.f;
        uint32_t pa[4][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float p0 = exp2f(sc[j][0] - mu0), p1 = exp2f(sc[j][1] - mu0);
            const float p2 = exp2f(sc[j][2] - mu1), p3 = exp2f(sc[j][3] - mu1);
            rs0 += p0 + p1;
            rs1 += p2 + p3;
            pa[j >> 1][(j & 1) * 2 + 0] = pack_f16x2(p0, p1);
            pa[j >> 1][(j & 1) * 2 + 1] = pack_f16x2(p2, p3);
        }
        l0 = l0 * c0 + rs0;
        l1 = l1 * c1 + rs1;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            o[j][0] *= c0; o[j][1] *= c0;
            o[j][2] *= c1; o[j][3] *= c1;
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const int vr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int dp = 0; dp < 4; ++dp) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vb + sw128(vr, dp * 2 + (lane >> 4)), b0, b1, b2, b3);
                mma_f16(o[2 * dp], pa[kk], b0, b1);
                mma_f16(o[2 * dp + 1], pa[kk], b2, b3);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0 && t + 2 < ntiles) {
            mbar_arrive_expect_tx(&bars[1 + s], 16384);
            tma_load_2d(sK[s], &tm, &bars[1 + s], D + h * DH, kv0 + (t + 2) * BK);
            tma_load_2d(sV[s], &tm, &bars[1 + s], 2 * D + h * DH, kv0 + (t + 2) * BK);
        }
    }
    if (!ok) return;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;

    // stage the warp's 16 x 64 output in its own rows of the Q tile, then copy out coalesced
    uint8_t *stg = sQ;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int col = j * 8 + 2 * tq;  // element column
        const int r0 = warp * 16 + g, r1 = r0 + 8;
        *reinterpret_cast<uint32_t *>(stg + sw128(r0, col >> 3) + (col & 7) * 2) = pack_bf16x2(o[j][0] * i0, o[j][1] * i0);
        *reinterpret_cast<uint32_t *>(stg + sw128(r1, col >> 3) + (col & 7) * 2) = pack_bf16x2(o[j][2] * i1, o[j][3] * i1);
    }
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int e = lane + 32 * it;
        const int r = e >> 3, c = e & 7;
        const int qi = q0 + warp * 16 + r;
        if (qi < ce) {
            const uint4 v = *reinterpret_cast<const uint4 *>(stg + sw128(warp * 16 + r, c));
            *reinterpret_cast<uint4 *>(out + (size_t)qi * D + h * DH + c * 8) = v;
        }
    }
}


// Sliding-window (+-64) variant: the CTA's 64 queries need the 192-key band
// [q0 - 64, q0 + 128), loaded once by TMA (three 64 x 64 tiles of K and of V);
// warp w's 16 queries need only the 144 keys [q0 + 16w - 64, q0 + 16w + 80),
// i.e. nine 16-key chunks, so each warp visits just those and runs an exact
// two-pass softmax over them in registers (no running rescale).  A CTA reads
// its row's span and first query from the prep kernel's table of every 64-query
// block, independent loads in one round trip to L2: a binary search over the
// row offsets (a chain of dependent loads per CTA) cost about a fifth of the
// kernel's time, and a row lookup followed by the row's offsets a tenth.
constexpr int LW_CHUNKS = 9;  // (16 + 2 * 64) / 16
// Two heads per CTA (8 warps, 2 CTAs per SM): 16 resident warps per SM instead of 12.
constexpr int LOC_HEADS = 2;
constexpr int LOC_HEAD_BYTES = 7 * 8192;  // Q tile, 3 K tiles, 3 V tiles
// The barriers sit in front of the 1024-byte aligned tiles, inside the alignment slack, so two
// CTAs fit one SM's 228 KB with the 1 KB each CTA reserves.
constexpr int LOC_SMEM = LOC_HEADS * LOC_HEAD_BYTES + 1024;

__global__ void __launch_bounds__(128 * LOC_HEADS, 2)
    k_attn_local_bf16(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ out,
                      const int *__restrict__ qb_off, const int *__restrict__ span, int n_rows, unsigned *status) {
    extern __shared__ __align__(16) uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 8 * LOC_HEADS + 1023) &
                                              ~uintptr_t(1023));
    const int hh = (threadIdx.x >> 5) >> 2;  // head slot of this warp's group of four
    uint8_t *sQ = sm + hh * LOC_HEAD_BYTES;  // 64 x 64
    uint8_t *sK = sQ + 8192;                 // 3 tiles of 64 x 64
    uint8_t *sV = sQ + 4 * 8192;             // 3 tiles
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm_raw) + hh;

    const int tile = blockIdx.x, h = blockIdx.y * LOC_HEADS + hh;
    // the block count and the block's span are independent loads (one round trip to L2); the
    // span entries of blocks past the count exist (the table covers the grid) and are not used
    const int n_blocks = qb_off[n_rows];
    const int cs = span[3 * tile], ce = span[3 * tile + 1], q0 = span[3 * tile + 2];
    if (tile >= n_blocks) return;
    const int kbase = q0 - 64;         // band start (may precede the row: masked)
    const int warp = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;  // warp inside the head's group

    if ((threadIdx.x & 127) == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, 7 * 8192);
        tma_load_2d(sQ, &tm, bar, h * DH, q0);
        for (int t = 0; t < 3; ++t) {
            tma_load_2d(sK + t * 8192, &tm, bar, D + h * DH, kbase + t * 64);
            tma_load_2d(sV + t * 8192, &tm, bar, 2 * D + h * DH, kbase + t * 64);
        }
    }
    __syncthreads();
    if (!mbar_wait(bar, 0, status)) return;

    const float sl2 = 0.125f * 1.4426950408889634f;
    const int g = lane >> 2, tq = lane & 3;
    const int qi0 = q0 + warp * 16 + g, qi1 = qi0 + 8;
    uint32_t qf[4][4];
    {
        const uint32_t base = smem_u32(sQ);
        const int r = warp * 16 + (lane & 15);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            ldsm_x4(base + sw128(r, kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
    // S over the warp's nine 16-key chunks (band chunks warp .. warp + 8)
    float sc[2 * LW_CHUNKS][4];
#pragma unroll
    for (int j = 0; j < 2 * LW_CHUNKS; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int cc = 0; cc < LW_CHUNKS; ++cc) {
        const int kc = warp + cc;                  // 16-key chunk inside the band
        const uint32_t kb = smem_u32(sK + (kc >> 2) * 8192);
        const int kr = (kc & 3) * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kb + sw128(kr, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
            mma_bf16(sc[2 * cc], qf[kk], b0, b1);
            mma_bf16(sc[2 * cc + 1], qf[kk], b2, b3);
        }
    }
    // Masks on the raw scores; the scale goes into the exponent's FMA below.  Key kj of 8-column
    // block j lies kj - qi = 8j - 64 + (2tq + e) - g (- 8 for qi1) from the query, which is inside
    // [-63, 63] for 2 <= j < 16: only the two outer chunks at each end need the window test.
    // Four interleaved partial maxima per query row: dependency chains of 9, not 36.  A warp whose
    // 144 keys all lie in the row (most warps of rows longer than a few hundred tokens) skips the
    // per-key row tests: a warp-uniform branch between two copies of the loop.
    float mp0[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, mp1[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    const int kw = kbase + warp * 16;  // the warp's first key
    if (kw >= cs && kw + 16 * LW_CHUNKS <= ce) {
#pragma unroll
        for (int j = 0; j < 2 * LW_CHUNKS; ++j) {
            const bool edge = j < 2 || j >= 2 * LW_CHUNKS - 2;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                if (edge) {
                    const int kj = kw + j * 8 + 2 * tq + e;
                    sc[j][e] = abs(qi0 - kj) <= 64 ? sc[j][e] : -INFINITY;
                    sc[j][2 + e] = abs(qi1 - kj) <= 64 ? sc[j][2 + e] : -INFINITY;
                }
                mp0[(2 * j + e) & 3] = fmaxf(mp0[(2 * j + e) & 3], sc[j][e]);
                mp1[(2 * j + e) & 3] = fmaxf(mp1[(2 * j + e) & 3], sc[j][2 + e]);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 2 * LW_CHUNKS; ++j) {
            const bool edge = j < 2 || j >= 2 * LW_CHUNKS - 2;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int kj = kw + j * 8 + 2 * tq + e;
                const bool in_row = kj >= cs && kj < ce;
                const bool v0 = in_row && (!edge || abs(qi0 - kj) <= 64);
                const bool v1 = in_row && (!edge || abs(qi1 - kj) <= 64);
                sc[j][e] = v0 ? sc[j][e] : -INFINITY;
                sc[j][2 + e] = v1 ? sc[j][2 + e] : -INFINITY;
                mp0[(2 * j + e) & 3] = fmaxf(mp0[(2 * j + e) & 3], sc[j][e]);
                mp1[(2 * j + e) & 3] = fmaxf(mp1[(2 * j + e) & 3], sc[j][2 + e]);
            }
        }
    }
    float mx0 = fmaxf(fmaxf(mp0[0], mp0[1]), fmaxf(mp0[2], mp0[3]));
    float mx1 = fmaxf(fmaxf(mp1[0], mp1[1]), fmaxf(mp1[2], mp1[3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mu0 = mx0 == -INFINITY ? 0.f : -mx0 * sl2, mu1 = mx1 == -INFINITY ? 0.f : -mx1 * sl2;
    // P = 2^x in FP32 (one ex2.approx.ftz per key), FP32 row sums, P packed to FP16 pairs for the
    // P V products (V is FP16).  An FP16 ex2 for two keys measured slower: its conversions cost
    // more instructions than it saved on the special-function unit.
    float lp0[2] = {0.f, 0.f}, lp1[2] = {0.f, 0.f};  // two interleaved partial sums per row
    uint32_t pa[LW_CHUNKS][4];
#pragma unroll
    for (int j = 0; j < 2 * LW_CHUNKS; ++j) {
        const float p0 = ex2_ftz(fmaf(sc[j][0], sl2, mu0)), p1 = ex2_ftz(fmaf(sc[j][1], sl2, mu0));
        const float p2 = ex2_ftz(fmaf(sc[j][2], sl2, mu1)), p3 = ex2_ftz(fmaf(sc[j][3], sl2, mu1));
        lp0[j & 1] += p0 + p1;
        lp1[j & 1] += p2 + p3;
        pa[j >> 1][(j & 1) * 2 + 0] = pack_f16x2(p0, p1);
        pa[j >> 1][(j & 1) * 2 + 1] = pack_f16x2(p2, p3);
    }
    float l0 = lp0[0] + lp0[1], l1 = lp1[0] + lp1[1];
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
#pragma unroll
    for (int cc = 0; cc < LW_CHUNKS; ++cc) {
        const int kc = warp + cc;
        const uint32_t vb = smem_u32(sV + (kc >> 2) * 8192);
        const int vr = (kc & 3) * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
        for (int dp = 0; dp < 4; ++dp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vb + sw128(vr, dp * 2 + (lane >> 4)), b0, b1, b2, b3);
            mma_f16(o[2 * dp], pa[cc], b0, b1);
            mma_f16(o[2 * dp + 1], pa[cc], b2, b3);
        }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    uint8_t *stg = sQ;  // the warp's own 16 rows of the Q tile (its Q fragments are in registers)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int col = j * 8 + 2 * tq;
        const int r0 = warp * 16 + g, r1 = r0 + 8;
        *reinterpret_cast<uint32_t *>(stg + sw128(r0, col >> 3) + (col & 7) * 2) = pack_bf16x2(o[j][0] * i0, o[j][1] * i0);
        *reinterpret_cast<uint32_t *>(stg + sw128(r1, col >> 3) + (col & 7) * 2) = pack_bf16x2(o[j][2] * i1, o[j][3] * i1);
    }
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int e = lane + 32 * it;
        const int r = e >> 3, c = e & 7;
        const int qi = q0 + warp * 16 + r;
        if (qi < ce) {
            const uint4 v = *reinterpret_cast<const uint4 *>(stg + sw128(warp * 16 + r, c));
            *reinterpret_cast<uint4 *>(out + (size_t)qi * D + h * DH + c * 8) = v;
        }
    }
}


// ------------------------------------------------------------------ FP32 validation attention

template <bool LOCAL>
__global__ void __launch_bounds__(256)
    k_attn_f32(const float *__restrict__ qkv, float *__restrict__ out, const int *__restrict__ cu,
               const int *__restrict__ qb_off, int n_rows, int window) {
    __shared__ float Ks[32][DH];
    __shared__ float Vs[32][DH];
    const int tile = blockIdx.x, h = blockIdx.y;
    if (tile >= qb_off[n_rows]) return;
    const int row = find_row(qb_off, n_rows, tile);
    const int cs = cu[row], ce = cu[row + 1];
    const int q0 = cs + (tile - qb_off[row]) * BQ;
    int kv0 = cs, kv1 = ce;
    if (LOCAL) {
        kv0 = max(cs, q0 - window);
        kv1 = min(ce, q0 + BQ + window);
    }
    const int tid = threadIdx.x, qi = tid >> 2, part = tid & 3;
    const int i = q0 + qi;
    const bool vq = i < ce;
    const float sl2 = 0.125f * 1.4426950408889634f;
    float q[16], o[16];
#pragma unroll
    for (int d = 0; d < 16; ++d) {
        q[d] = vq ? qkv[(size_t)i * QKV + h * DH + part * 16 + d] * sl2 : 0.f;
        o[d] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int kt = kv0; kt < kv1; kt += 32) {
        __syncthreads();
        for (int e = tid; e < 32 * DH; e += 256) {
            const int j = e / DH, d = e % DH;
            const int kj = kt + j;
            const bool in = kj < kv1;
            Ks[j][d] = in ? qkv[(size_t)kj * QKV + D + h * DH + d] : 0.f;
            Vs[j][d] = in ? qkv[(size_t)kj * QKV + 2 * D + h * DH + d] : 0.f;
        }
        __syncthreads();
        const int nk = min(32, kv1 - kt);
        for (int j = 0; j < nk; ++j) {
            float s = 0.f;
#pragma unroll
            for (int d = 0; d < 16; ++d) s = fmaf(q[d], Ks[j][part * 16 + d], s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            const int kj = kt + j;
            const bool vis = !LOCAL || abs(i - kj) <= window;
            if (vis) {
                const float mn = fmaxf(m, s);
                const float c = exp2f(m - mn), p = exp2f(s - mn);
                l = l * c + p;
#pragma unroll
                for (int d = 0; d < 16; ++d) o[d] = o[d] * c + p * Vs[j][part * 16 + d];
                m = mn;
            }
        }
    }
    if (vq) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int d = 0; d < 16; ++d) out[(size_t)i * D + h * DH + part * 16 + d] = o[d] * inv;
    }
}

cudaError_t attn_tc_init_attributes();

cudaError_t attn_init_attributes() {
    cudaError_t e = cudaFuncSetAttribute(k_attn_local_bf16, cudaFuncAttributeMaxDynamicSharedMemorySize, LOC_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_attn_local_bf16, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    return attn_tc_init_attributes();
}

cudaError_t launch_attention(const AttnArgs &a, bool fp32, cudaStream_t st) {
    if (a.n_rows <= 0 || a.n_tokens <= 0) return cudaSuccess;
    const int max_tiles = (a.n_tokens + BQ - 1) / BQ + a.n_rows;
    dim3 grid(max_tiles, NH);
    const bool local = a.window >= 0;
    if (fp32) {
        if (local)
            k_attn_f32<true><<<grid, 256, 0, st>>>((const float *)a.qkv, (float *)a.o, a.cu_seqlens, a.qb_off,
                                                   a.n_rows, a.window);
        else
            k_attn_f32<false><<<grid, 256, 0, st>>>((const float *)a.qkv, (float *)a.o, a.cu_seqlens, a.qb_off,
                                                    a.n_rows, a.window);
    } else if (a.tm_qkv128 && !local) {
        // tcgen05 for global layers; the +-64 band stays on the mma.sync kernel below,
        // which measured faster than the band variant of the tcgen05 kernel (2 tiles per item)
        return launch_attention_tc(a, a.tm_qkv128, num_sms(), st);
    } else {
        const int smem = 5 * 8192 + 64 + 1024;
        if (local && a.window == 64)
            k_attn_local_bf16<<<dim3(max_tiles, NH / LOC_HEADS), 128 * LOC_HEADS, LOC_SMEM, st>>>(
                *a.tm_qkv, (__nv_bfloat16 *)a.o, a.qb_off, a.qb_off + qb_span_offset(a.n_rows, a.n_tokens), a.n_rows,
                a.status);
        else if (local)
            k_attn_bf16<true><<<grid, 128, smem, st>>>(*a.tm_qkv, (__nv_bfloat16 *)a.o, a.cu_seqlens, a.qb_off,
                                                       a.n_rows, a.window, a.status);
        else
            k_attn_bf16<false><<<grid, 128, smem, st>>>(*a.tm_qkv, (__nv_bfloat16 *)a.o, a.cu_seqlens, a.qb_off,
                                                        a.n_rows, a.window, a.status);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------ marker-only attention

// One CTA per (row, head): the row's marker queries against all its keys.
// "julia1 -- Rust runtime for Julia-1", "Why it is faster": the last head
// layer computes queries only for option markers; keys / values stay full.
template <typename T>
__global__ void __launch_bounds__(128)
    k_marker_attn(const T *__restrict__ qm, const T *__restrict__ qkv, T *__restrict__ om, const int *__restrict__ cu,
                  const int *__restrict__ opt_off, int nsplit, float *__restrict__ part) {
    __shared__ float Qs[32][DH];
    __shared__ float Ks[32][DH + 1];
    __shared__ float Vs[32][DH];
    __shared__ float S[32][32];
    __shared__ float Ms[32], Ls[32], Cs[32];
    const int row = blockIdx.x, h = blockIdx.y, sp = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rs = cu[row], re = cu[row + 1];
    // this CTA's share of the row's keys (split sp of nsplit, 32-key aligned)
    const int chunk = ((re - rs + nsplit - 1) / nsplit + 31) / 32 * 32;
    const int cs = min(re, rs + sp * chunk), ce = min(re, cs + chunk);
    const int mb = opt_off[row], me = opt_off[row + 1];
    const float sl2 = 0.125f * 1.4426950408889634f;
    for (int qc = mb; qc < me; qc += 32) {
        const int nq = min(32, me - qc);
        __syncthreads();
        for (int e = tid; e < 32 * DH; e += 128) {
            const int qi = e / DH, d = e % DH;
            Qs[qi][d] = qi < nq ? (float)qm[(size_t)(qc + qi) * D + h * DH + d] * sl2 : 0.f;
        }
        float oacc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) oacc[r] = 0.f;
        if (tid < 32) { Ms[tid] = -INFINITY; Ls[tid] = 0.f; }
        for (int kt = cs; kt < ce; kt += 32) {
            const int nk = min(32, ce - kt);
            __syncthreads();
            for (int e = tid; e < 32 * DH; e += 128) {
                const int j = e / DH, d = e % DH;
                const bool in = j < nk;
                Ks[j][d] = in ? (float)qkv[(size_t)(kt + j) * QKV + D + h * DH + d] : 0.f;
                Vs[j][d] = in ? (float)qkv[(size_t)(kt + j) * QKV + 2 * D + h * DH + d] : 0.f;
            }
            __syncthreads();
            for (int e = tid; e < nq * 32; e += 128) {
                const int qi = e >> 5, j = e & 31;
                float s = -INFINITY;
                if (j < nk) {
                    s = 0.f;
#pragma unroll 16
                    for (int d = 0; d < DH; ++d) s = fmaf(Qs[qi][d], Ks[j][d], s);
                }
                S[qi][j] = s;
            }
            __syncthreads();
            for (int qi = warp; qi < nq; qi += 4) {
                const float s0 = S[qi][lane];
                const float mx = warp_max(s0);
                const float mo = Ms[qi];
                const float mn = fmaxf(mo, mx);
                const float p0 = exp2f(s0 - mn);
                S[qi][lane] = p0;
                const float sum = warp_sum(p0);
                if (lane == 0) {
                    const float c = exp2f(mo - mn);
                    Cs[qi] = c;
                    Ls[qi] = Ls[qi] * c + sum;
                    Ms[qi] = mn;
                }
            }
            __syncthreads();
            // thread owns (query, dim) pairs e = tid + 128 r
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                const int e = tid + 128 * r;
                const int qi = e >> 6, d = e & 63;
                if (qi < nq) {
                    float acc = oacc[r] * Cs[qi];
                    for (int j = 0; j < nk; ++j) acc = fmaf(S[qi][j], Vs[j][d], acc);
                    oacc[r] = acc;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            const int e = tid + 128 * r;
            const int qi = e >> 6, d = e & 63;
            if (qi < nq) {
                if (nsplit == 1) {
                    om[(size_t)(qc + qi) * D + h * DH + d] = (T)(oacc[r] / Ls[qi]);
                } else {  // partial result of this key split: running max (log2), sum, unnormalised o
                    float *pe = part + ((size_t)((qc + qi) * NH + h) * nsplit + sp) * (DH + 2);
                    if (d == 0) {
                        pe[0] = Ms[qi];
                        pe[1] = Ls[qi];
                    }
                    pe[2 + d] = oacc[r];
                }
            }
        }
    }
}

// BF16 marker attention on the tensor cores (mma.sync m16n8k16): one CTA per (row, head,
// key split), two warps of 16 marker queries each (a row has at most 20 markers, so one
// 32-query pass; longer lists loop), Q by TMA from the marker-query buffer, 64-key K / V
// tiles in a two-stage TMA ring, online softmax in registers.  The SIMT kernel above
// spent two shared-memory loads per FMA on the dot products.
constexpr int MQ = 32;  // marker queries per pass
__global__ void __launch_bounds__(64)
    k_marker_attn_mma(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tm,
                      __nv_bfloat16 *__restrict__ om, const int *__restrict__ cu, const int *__restrict__ opt_off,
                      int nsplit, float *__restrict__ part, unsigned *status) {
    extern __shared__ uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = sm;                                   // 32 x 64
    uint8_t *sK[2] = {sm + 4096, sm + 4096 + 8192};     // 64 x 64 each
    uint8_t *sV[2] = {sm + 4096 + 2 * 8192, sm + 4096 + 3 * 8192};
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + 4096 + 4 * 8192);  // 0: Q, 1..2: K/V stages

    const int row = blockIdx.x, h = blockIdx.y, sp = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rs = cu[row], re = cu[row + 1];
    const int chunk = ((re - rs + nsplit - 1) / nsplit + 31) / 32 * 32;
    const int cs = min(re, rs + sp * chunk), ce = min(re, cs + chunk);
    const int mb = opt_off[row], me = opt_off[row + 1];
    const int ntiles = (ce - cs + BK - 1) / BK;
    const float sl2 = 0.125f * 1.4426950408889634f;
    const int g = lane >> 2, tq = lane & 3;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    __syncthreads();
    uint32_t qphase = 0, kvuse[2] = {0, 0};
    for (int qc = mb; qc < me; qc += MQ) {
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&bars[0], MQ * 128);
            tma_load_2d(sQ, &tmq, &bars[0], h * DH, qc);
            for (int t = 0; t < 2 && t < ntiles; ++t) {
                mbar_arrive_expect_tx(&bars[1 + t], 16384);
                tma_load_2d(sK[t], &tm, &bars[1 + t], D + h * DH, cs + t * BK);
                tma_load_2d(sV[t], &tm, &bars[1 + t], 2 * D + h * DH, cs + t * BK);
            }
        }
        bool ok = mbar_wait(&bars[0], qphase & 1, status);
        ++qphase;
        uint32_t qf[4][4];
        {
            const uint32_t base = smem_u32(sQ);
            const int r = warp * 16 + (lane & 15);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                ldsm_x4(base + sw128(r, kk * 2 + (lane >> 4)), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
        }
        float o[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        for (int t = 0; t < ntiles; ++t) {
            const int s = t & 1;
            if (ok && !mbar_wait(&bars[1 + s], kvuse[s] & 1, status)) ok = false;
            ++kvuse[s];
            if (ok) {
                const uint32_t kb = smem_u32(sK[s]), vb = smem_u32(sV[s]);
                const int kt0 = cs + t * BK;
                float sc[8][4];
#pragma unroll
                for (int j = 0; j < 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    const int kr = np * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(kb + sw128(kr, kk * 2 + ((lane >> 3) & 1)), b0, b1, b2, b3);
                        mma_bf16(sc[2 * np], qf[kk], b0, b1);
                        mma_bf16(sc[2 * np + 1], qf[kk], b2, b3);
                    }
                }
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool in = kt0 + j * 8 + 2 * tq + e < ce;  // keys of this split only
                        sc[j][e] = in ? sc[j][e] * sl2 : -INFINITY;
                        sc[j][2 + e] = in ? sc[j][2 + e] * sl2 : -INFINITY;
                        mx0 = fmaxf(mx0, sc[j][e]);
                        mx1 = fmaxf(mx1, sc[j][2 + e]);
                    }
                }
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
                const float c0 = exp2f(m0 - mu0), c1 = exp2f(m1 - mu1);
                m0 = mn0;
                m1 = mn1;
                float rs0 = 0.f, rs1 = 0.f;
                uint32_t pa[4][4];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float p0 = exp2f(sc[j][0] - mu0), p1 = exp2f(sc[j][1] - mu0);
                    const float p2 = exp2f(sc[j][2] - mu1), p3 = exp2f(sc[j][3] - mu1);
                    rs0 += p0 + p1;
                    rs1 += p2 + p3;
                    pa[j >> 1][(j & 1) * 2 + 0] = pack_f16x2(p0, p1);
                    pa[j >> 1][(j & 1) * 2 + 1] = pack_f16x2(p2, p3);
                }
                l0 = l0 * c0 + rs0;
                l1 = l1 * c1 + rs1;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    o[j][0] *= c0; o[j][1] *= c0;
                    o[j][2] *= c1; o[j][3] *= c1;
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int vr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
                    for (int dp = 0; dp < 4; ++dp) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(vb + sw128(vr, dp * 2 + (lane >> 4)), b0, b1, b2, b3);
                        mma_f16(o[2 * dp], pa[kk], b0, b1);
                        mma_f16(o[2 * dp + 1], pa[kk], b2, b3);
                    }
                }
            }
            __syncthreads();  // both warps are done with stage s
            if (threadIdx.x == 0 && t + 2 < ntiles) {
                mbar_arrive_expect_tx(&bars[1 + s], 16384);
                tma_load_2d(sK[s], &tm, &bars[1 + s], D + h * DH, cs + (t + 2) * BK);
                tma_load_2d(sV[s], &tm, &bars[1 + s], 2 * D + h * DH, cs + (t + 2) * BK);
            }
        }
        // kvuse[s] counts the completed phases of stage s across passes
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const int r0 = qc + warp * 16 + g, r1 = r0 + 8;  // marker indices of this thread's two rows
        if (ok) {
            if (nsplit == 1) {
                const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int col = h * DH + j * 8 + 2 * tq;
                    if (r0 < me)
                        *reinterpret_cast<uint32_t *>(om + (size_t)r0 * D + col) = pack_bf16x2(o[j][0] * i0, o[j][1] * i0);
                    if (r1 < me)
                        *reinterpret_cast<uint32_t *>(om + (size_t)r1 * D + col) = pack_bf16x2(o[j][2] * i1, o[j][3] * i1);
                }
            } else {  // partials of this key split: running max (log2), sum, unnormalised o
                float *p0 = part + ((size_t)(r0 * NH + h) * nsplit + sp) * (DH + 2);
                float *p1 = part + ((size_t)(r1 * NH + h) * nsplit + sp) * (DH + 2);
                if (r0 < me && tq == 0) { p0[0] = m0; p0[1] = l0; }
                if (r1 < me && tq == 0) { p1[0] = m1; p1[1] = l1; }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int d = j * 8 + 2 * tq;
                    if (r0 < me) { p0[2 + d] = o[j][0]; p0[3 + d] = o[j][1]; }
                    if (r1 < me) { p1[2 + d] = o[j][2]; p1[3 + d] = o[j][3]; }
                }
            }
        }
        __syncthreads();  // sQ and the K / V stages are free for the next pass
    }
}
constexpr int MARKER_MMA_SMEM = 4096 + 4 * 8192 + 64 + 1024;

// Merge the key splits of every (marker, head): o = sum_s 2^(m_s - m) o_s / sum_s 2^(m_s - m) l_s.
template <typename T>
__global__ void __launch_bounds__(64)
    k_marker_combine(const float *__restrict__ part, int nsplit, T *__restrict__ om) {
    const int mk = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
    const float *pe = part + (size_t)(mk * NH + h) * nsplit * (DH + 2);
    float m = -INFINITY;
    for (int s = 0; s < nsplit; ++s) m = fmaxf(m, pe[s * (DH + 2)]);
    float l = 0.f, o = 0.f;
    for (int s = 0; s < nsplit; ++s) {
        const float ms = pe[s * (DH + 2)];
        const float w = ms == -INFINITY ? 0.f : exp2f(ms - m);
        l = fmaf(pe[s * (DH + 2) + 1], w, l);
        o = fmaf(pe[s * (DH + 2) + 2 + d], w, o);
    }
    om[(size_t)mk * D + h * DH + d] = (T)(o / l);
}

// One CTA per (row, head) leaves most SMs idle on long rows: split the keys, one
// split per 1024 keys of the longest row (at most 8), within the scratch capacity.
int marker_attention_splits(int n_markers, int max_row_len, const float *part, int part_entries) {
    int nsplit = max_row_len > 1024 ? min(8, (max_row_len + 1023) / 1024) : 1;
    if (!part || n_markers <= 0) return 1;
    if (nsplit > 1 && (long)n_markers * nsplit > part_entries) nsplit = max(1, part_entries / n_markers);
    return nsplit;
}

cudaError_t launch_marker_attention(const void *qm, const void *qkv, void *om, const int *cu_seqlens,
                                    const int *opt_off, int n_rows, int n_markers, int max_row_len, float *part,
                                    int part_entries, bool fp32, const CUtensorMap *tm_q, const CUtensorMap *tm_kv,
                                    unsigned *status, cudaStream_t st) {
    if (n_rows <= 0 || n_markers <= 0) return cudaSuccess;
    const int nsplit = marker_attention_splits(n_markers, max_row_len, part, part_entries);
    dim3 grid(n_rows, NH, nsplit);
    if (fp32)
        k_marker_attn<float><<<grid, 128, 0, st>>>((const float *)qm, (const float *)qkv, (float *)om, cu_seqlens,
                                                   opt_off, nsplit, part);
    else if (tm_q && tm_kv)
        k_marker_attn_mma<<<grid, 64, MARKER_MMA_SMEM, st>>>(*tm_q, *tm_kv, (__nv_bfloat16 *)om, cu_seqlens, opt_off,
                                                             nsplit, part, status);
    else
        k_marker_attn<__nv_bfloat16><<<grid, 128, 0, st>>>((const __nv_bfloat16 *)qm, (const __nv_bfloat16 *)qkv,
                                                           (__nv_bfloat16 *)om, cu_seqlens, opt_off, nsplit, part);
    if (nsplit > 1) {
        dim3 g2(n_markers, NH);
        if (fp32)
            k_marker_combine<float><<<g2, DH, 0, st>>>(part, nsplit, (float *)om);
        else
            k_marker_combine<__nv_bfloat16><<<g2, DH, 0, st>>>(part, nsplit, (__nv_bfloat16 *)om);
    }
    return cudaGetLastError();
}

}  // namespace jd
