// Bidirectional global attention inside each packed row on the 5th-generation
// tensor cores.
//
// "Julia-1 MLX", "Performance": every third encoder layer attends over the whole
// row; so do the two head layers ("Julia-1: one score per mask token", "The
// decision head", step 2).  Rows are packed back to back ("julia1 -- Rust
// runtime for Julia-1", "Why it is faster").  A work item is one 256-query
// block of one row and one head: two 128-query tiles (the second is absent
// when the row ends inside the first) that share every K and V tile, so the
// keys and values of a row cross from L2 once per 256 queries.  With one
// 128-query tile per CTA the kernel ran at the L2-to-SM bandwidth; two tiles
// halve that traffic per query.  A persistent CTA per SM walks the item list.
//
//   warp 0 lane 0   TMA producer: both Q tiles (128 x 64, 128-byte swizzle)
//                   once per item into one of two buffers; K tiles (128 keys x
//                   64) into a four-stage ring, each stage released when its
//                   S products complete
//   warp 2 lane 0   TMA producer of the V tiles: a four-stage ring, each stage
//                   released when its PV products complete
//   warp 1          TMEM allocation; lane 0 issues tcgen05.mma:
//                     S_x = Q_x K_j^T  (M 128, N 128, K 64; A, B from shared memory)
//                     O_x += P_x V_j   (M 128, N 64, K 128; P from TMEM, V read MN-major)
//   warps 4..7      softmax of Q tile 0, warps 8..11 of Q tile 1: one query
//                   row per thread (warp w reads TMEM lane quarter w % 4), all
//                   128 keys of every tile.  The running max is kept lazily: O
//                   and the row sum are rescaled only when the max grows by
//                   more than 2^8, so P stays below 256.  P is stored as bf16
//                   pairs into TMEM, where the PV product reads it.  The two
//                   groups take turns at the exponentials (named barriers 1 and
//                   2), so that the special-function unit, which bounds that
//                   phase, is busy with one group while the other loads S,
//                   takes the row max and hands P over.
// Warp group 0 (warps 0..3, warp 3 idle) hands registers to the two softmax warp groups
// (setmaxnreg).  TMEM columns: S_x at 128 x, O_x at 256 + 64 x, P_x at 384 + 64 x.

#include "common.cuh"
#include "kernels.h"

namespace jd {

namespace {
constexpr int TQ = 128, TK = 128;
constexpr int Q_BYTES = TQ * 128;          // 128 rows x 64 bf16
constexpr int KT_BYTES = TK * 128;         // 128 keys x 64 bf16
constexpr int NK = 4;                      // K ring depth
constexpr int NV = 4;                      // V ring depth
constexpr int OFF_Q = 0;                   // [item buffer][q tile]
constexpr int OFF_K = OFF_Q + 4 * Q_BYTES;
constexpr int OFF_V = OFF_K + NK * KT_BYTES;
constexpr int OFF_BAR = OFF_V + NV * KT_BYTES;
// qfull[2], qfree[2], kfull[NK], kfree[NK], vfull[NV], vfree[NV],
// sfull[2], sfree[2], pready[2], pvdone[2], ofree[2] (the last five per Q tile)
constexpr int NBAR = 2 + 2 + 2 * NK + 2 * NV + 5 * 2;
constexpr int ATC_SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
static_assert(ATC_SMEM <= 227 * 1024, "attention shared memory");
constexpr uint32_t T_S = 0, T_O = 256, T_P = 384;
constexpr float kLazy = 8.0f;    // log2 headroom before the running max is moved
constexpr int V_WARP = 2;
constexpr int ATC_THREADS = 12 * 32;
// Registers: the launch gives every thread ATC_REGS (the compiled count, checked on the host
// before the first launch); warp group 0 (producers, MMA issue) gives up all but ATC_REGS_LOW and
// the two softmax warp groups take ATC_REGS_HIGH, 128 x LOW + 256 x HIGH <= 384 x ATC_REGS.
constexpr int ATC_REGS = 168, ATC_REGS_LOW = 120, ATC_REGS_HIGH = 192;
static_assert(128 * ATC_REGS_LOW + 256 * ATC_REGS_HIGH <= ATC_THREADS * ATC_REGS, "register split");
constexpr int BAR_G0_DONE = 1, BAR_G1_DONE = 2;  // named barriers of the softmax groups' hand-off
}  // namespace

// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x with the hardware approximation (ex2.approx.ftz; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed FP32 pairs on the FMA pipe (sm_100 f32x2 forms: one instruction per pair).
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// 2^x for a pair, on the FMA and integer pipes instead of the special-function unit.
// x = j + f with j = round(x) and f in [-1/2, 1/2]: adding 1.5 * 2^23 leaves j in the low
// mantissa bits of t (|x| < 2^22), so t - 1.5 * 2^23 is j exactly and f = x - j exactly.
// 2^f is the degree-3 polynomial of least maximum relative error on [-1/2, 1/2], found by
// the Remez exchange algorithm (|p(f) / 2^f - 1| <= 7.5e-5; the bf16 rounding P receives
// is 2^-9 = 2.0e-3), and 2^j enters as j added to p's exponent field (bits(t) << 23 is
// j << 23: the constant's own bits shift out).  x is clamped at -126, so the masked keys
// (x = -inf) give 2^-126 ~ 1e-38 for 0, still a normal float.
constexpr float EX2_C0 = 0.9999280571937561f, EX2_C1 = 0.6932609677314758f, EX2_C2 = 0.2426111251115799f,
                EX2_C3 = 0.0551716685295105f;
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float &y0, float &y1) {
    const float2 x = make_float2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const float2 t = add2(x, make_float2(12582912.f, 12582912.f));
    const float2 j = add2(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = add2(x, make_float2(-j.x, -j.y));
    float2 p = fma2(f, make_float2(EX2_C3, EX2_C3), make_float2(EX2_C2, EX2_C2));
    p = fma2(p, f, make_float2(EX2_C1, EX2_C1));
    p = fma2(p, f, make_float2(EX2_C0, EX2_C0));
    y0 = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
    y1 = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
}

// Of every eight key pairs a softmax thread exponentiates, this many take the polynomial
// above and the rest the special-function unit.  Measured on the throughput and long-row
// workloads, 2, 3 or 4 of 8 ran no faster than 0 (the softmax warps are bound by issued
// instructions, not by the special-function unit alone), so the default is 0; the build
// option stays for other shapes.
#ifndef JD_EX2_POLY_OF8
#define JD_EX2_POLY_OF8 0
#endif

// D[tmem] (+)= A[tmem] * B[smem]: A is M x K in TMEM (lane = row, two bf16 per column)
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct AtcItem {
    int h, cs, ce, q0, nt, nx;  // nx: Q tiles in this item (1 or 2)
};

__device__ __forceinline__ AtcItem atc_item(const int *q256, const int *pb_row, const int *cu, int w) {
    AtcItem t;
    const int pb = w / NH;
    t.h = w % NH;
    const int row = pb_row[pb];
    t.cs = cu[row];
    t.ce = cu[row + 1];
    t.q0 = t.cs + (pb - q256[row]) * (2 * TQ);
    t.nt = (t.ce - t.cs + TK - 1) / TK;
    t.nx = t.q0 + TQ < t.ce ? 2 : 1;
    return t;
}

__global__ void __launch_bounds__(ATC_THREADS, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ out, const int *__restrict__ cu,
              const int *__restrict__ qb_off, int n_rows, unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *qfull = bars + 0, *qfree = bars + 2, *kfull = bars + 4, *kfree = kfull + NK, *vfull = kfree + NK,
             *vfree = vfull + NV, *sfull = vfree + NV, *sfree = sfull + 2, *pready = sfree + 2, *pvdone = pready + 2,
             *ofree = pvdone + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);

    const int *q256 = qb_off + n_rows + 1;
    const int *pb_row = q256 + n_rows + 1;
    const int n_items = q256[n_rows] * NH;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            mbar_init(&kfull[i], 1);
            mbar_init(&kfree[i], 1);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(&vfull[i], 1);
            mbar_init(&vfree[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qfree[i], 1);
            mbar_init(&sfull[i], 1);
            mbar_init(&sfree[i], 4);
            mbar_init(&pready[i], 4);
            mbar_init(&pvdone[i], 1);
            mbar_init(&ofree[i], 4);
        }
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tm);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp < 4) {  // warp group 0: the TMA producers and the MMA issue
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(ATC_REGS_LOW));
        if (warp == 0) {
            if (lane == 0) {
                uint32_t J = 0, it = 0;
                for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
                    const AtcItem t = atc_item(q256, pb_row, cu, w);
                    const uint32_t qbuf = it & 1;
                    if (it >= 2) mbar_wait(&qfree[qbuf], ((it - 2) >> 1) & 1, status);
                    mbar_arrive_expect_tx(&qfull[qbuf], t.nx * Q_BYTES);
                    for (int x = 0; x < t.nx; ++x)
                        tma_load_2d(smem + OFF_Q + (qbuf * 2 + x) * Q_BYTES, &tm, &qfull[qbuf], t.h * DH, t.q0 + x * TQ);
                    for (int j = 0; j < t.nt; ++j, ++J) {
                        const uint32_t s = J % NK;
                        if (J >= NK) mbar_wait(&kfree[s], ((J - NK) / NK) & 1, status);
                        mbar_arrive_expect_tx(&kfull[s], KT_BYTES);
                        tma_load_2d(smem + OFF_K + s * KT_BYTES, &tm, &kfull[s], D + t.h * DH, t.cs + j * TK);
                    }
                }
            }
        } else if (warp == V_WARP) {
            if (lane == 0) {
                uint32_t J = 0;
                for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
                    const AtcItem t = atc_item(q256, pb_row, cu, w);
                    for (int j = 0; j < t.nt; ++j, ++J) {
                        const uint32_t s = J % NV;
                        if (J >= NV) mbar_wait(&vfree[s], ((J - NV) / NV) & 1, status);
                        mbar_arrive_expect_tx(&vfull[s], KT_BYTES);
                        tma_load_2d(smem + OFF_V + s * KT_BYTES, &tm, &vfull[s], 2 * D + t.h * DH, t.cs + j * TK);
                    }
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                constexpr uint32_t idesc_s = idesc_bf16_f32(TK);
                constexpr uint32_t idesc_pv = idesc_f16_f32(DH) | (1u << 16);  // P and V FP16; B (V) is MN-major
                uint32_t J = 0, it = 0;
                uint32_t cnt[2] = {0, 0};   // S tiles issued per Q tile, over all items
                uint32_t uses[2] = {0, 0};  // items that used each Q tile
                // O_x += P_x V for the K tile at ring position Jp: cx[x] is that tile's S count of Q tile
                // x, `first` marks an item's first tile (O_x overwritten once the last item's O_x is read
                // out: us[x] items had used it before)
                auto issue_pv = [&](uint32_t Jp, int nx, const uint32_t (&cx)[2], bool first, const uint32_t (&us)[2]) {
                    const uint32_t s = Jp % NV;
                    mbar_wait(&vfull[s], (Jp / NV) & 1, status);
                    const uint32_t v_base = smem_u32(smem + OFF_V + s * KT_BYTES);
                    for (int x = 0; x < nx; ++x) {
                        mbar_wait(&pready[x], cx[x] & 1, status);
                        if (first && us[x] >= 1) mbar_wait(&ofree[x], (us[x] - 1) & 1, status);
                        tc_fence_after();
    #pragma unroll
                        for (int ks = 0; ks < TK / 16; ++ks)
                            tc_mma_bf16_ts(tmem + T_O + 64 * x, tmem + T_P + 64 * x + 8 * ks,
                                           sdesc_sw128(v_base + ks * 16 * 128), idesc_pv, (!first || ks != 0) ? 1u : 0u);
                        tc_commit(&pvdone[x]);
                    }
                    tc_commit(&vfree[s]);
                };
                // The PV products of an item's last K tile are issued after the next item's first S
                // products, so that the softmax groups find their next S tile ready when they finish
                // the item, instead of after both groups' last exponentials.
                bool pend = false;
                uint32_t pJ = 0, pc[2] = {0, 0}, pu[2] = {0, 0};
                int pnx = 0;
                bool pfirst = false;
                for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
                    const AtcItem t = atc_item(q256, pb_row, cu, w);
                    const uint32_t qbuf = it & 1;
                    mbar_wait(&qfull[qbuf], (it >> 1) & 1, status);
                    tc_fence_after();
                    const uint32_t J0 = J, c0[2] = {cnt[0], cnt[1]}, u0[2] = {uses[0], uses[1]};
                    for (int j = 0; j < t.nt; ++j, ++J) {
                        const uint32_t s = J % NK;
                        mbar_wait(&kfull[s], (J / NK) & 1, status);
                        const uint32_t k_base = smem_u32(smem + OFF_K + s * KT_BYTES);
                        for (int x = 0; x < t.nx; ++x) {
                            const uint32_t c = cnt[x]++;
                            if (c >= 1) mbar_wait(&sfree[x], (c - 1) & 1, status);  // S_x read out
                            tc_fence_after();
                            const uint32_t q_base = smem_u32(smem + OFF_Q + (qbuf * 2 + x) * Q_BYTES);
    #pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc_mma_bf16(tmem + T_S + TK * x, sdesc_sw128(q_base + kk * 32),
                                            sdesc_sw128(k_base + kk * 32), idesc_s, kk != 0);
                            tc_commit(&sfull[x]);
                        }
                        tc_commit(&kfree[s]);
                        if (j == t.nt - 1) tc_commit(&qfree[qbuf]);
                        if (j == 0 && pend) {
                            issue_pv(pJ, pnx, pc, pfirst, pu);
                            pend = false;
                        }
                        if (j >= 1) {
                            const uint32_t cx[2] = {c0[0] + j - 1, c0[1] + j - 1};
                            issue_pv(J0 + j - 1, t.nx, cx, j == 1, u0);
                        }
                    }
                    pend = true;
                    pJ = J0 + t.nt - 1;
                    pnx = t.nx;
                    pc[0] = c0[0] + t.nt - 1;
                    pc[1] = c0[1] + t.nt - 1;
                    pfirst = t.nt == 1;
                    pu[0] = u0[0];
                    pu[1] = u0[1];
                    for (int x = 0; x < t.nx; ++x) ++uses[x];
                }
                if (pend) issue_pv(pJ, pnx, pc, pfirst, pu);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(ATC_REGS_HIGH));
        const int x = (warp - 4) >> 2;         // Q tile of this warp group
        const int r = (warp & 3) * 32 + lane;  // query row inside the tile = TMEM lane
        const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float sl2 = 0.125f * 1.4426950408889634f;
        uint32_t c = 0;
        bool prev_pp = false;  // the CTA's previous item had two Q tiles
        // An item's O_x is read out once its last PV product has landed, which this thread waits
        // for anyway before storing the next item's first P tile: the readout follows that store,
        // so the wait for the last product hides behind the next item's first exponentials.
        // rd_dst: the pending row's output (null for a row past the end)
        bool rd_pend = false;
        __nv_bfloat16 *rd_dst = nullptr;
        float rd_inv = 0.f;
        auto readout = [&]() {
            __syncwarp();
            tc_fence_after();
#pragma unroll 1
            for (int hc = 0; hc < 64; hc += 32) {
                uint32_t o[32];
                tmem_ld32(tl + T_O + 64 * x + hc, o);
                tmem_ld_wait();
                if (rd_dst) {  // 32-byte stores: a warp instruction fills whole sectors
                    uint8_t *dst = reinterpret_cast<uint8_t *>(rd_dst + hc);
#pragma unroll
                    for (int k8 = 0; k8 < 2; ++k8) {
                        uint32_t wv[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            wv[e] = pack_bf16x2(__uint_as_float(o[16 * k8 + 2 * e]) * rd_inv,
                                                __uint_as_float(o[16 * k8 + 2 * e + 1]) * rd_inv);
                        st_global_v8(dst + 32 * k8, wv[0], wv[1], wv[2], wv[3], wv[4], wv[5], wv[6], wv[7]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ofree[x]);
            rd_pend = false;
        };
        for (int w = blockIdx.x; w < n_items; w += gridDim.x) {
            const AtcItem t = atc_item(q256, pb_row, cu, w);
            const bool pp = t.nx == 2;  // both groups busy: alternate the exponential phases
            // The hand-off runs on from one two-tile item into the next: group 0 starts an item's
            // exponentials after group 1's last ones of the previous item, group 1 hands over its
            // last tile only when the next item has two tiles too.  Either way every arrival on a
            // hand-off barrier meets exactly one wait.
            const bool g0_wait_first = pp && prev_pp;
            prev_pp = pp;
            if (x >= t.nx) continue;
            const bool g1_hand_last =
                pp && x == 1 && w + (int)gridDim.x < n_items && atc_item(q256, pb_row, cu, w + gridDim.x).nx == 2;
            const int qi = t.q0 + x * TQ + r;
            // A warp whose 32 query rows all lie past the row's end (the tail of a short row's
            // last tile) reads nothing of S, P or O: it keeps every wait and arrival of the
            // pipeline, so the barrier phases stay those of the other warps, and skips the math.
            if (t.q0 + x * TQ + (warp & 3) * 32 >= t.ce) {
                if (rd_pend) {
                    mbar_wait(&pvdone[x], (c - 1) & 1, status);
                    readout();
                }
                for (int j = 0; j < t.nt; ++j, ++c) {
                    mbar_wait(&sfull[x], c & 1, status);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sfree[x]);
                    if (pp) {
                        if (x == 0) {
                            if (j != 0 || g0_wait_first) named_bar_sync(BAR_G1_DONE, 256);
                        } else {
                            named_bar_sync(BAR_G0_DONE, 256);
                        }
                    }
                    if (j != 0) mbar_wait(&pvdone[x], (c - 1) & 1, status);
                    if (pp) {
                        if (x == 0) named_bar_arrive(BAR_G0_DONE, 256);
                        else if (j != t.nt - 1 || g1_hand_last) named_bar_arrive(BAR_G1_DONE, 256);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pready[x]);
                }
                mbar_wait(&pvdone[x], (c - 1) & 1, status);
                __syncwarp();
                if (lane == 0) mbar_arrive(&ofree[x]);
                continue;
            }
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < t.nt; ++j, ++c) {
                const int k0 = t.cs + j * TK;
                mbar_wait(&sfull[x], c & 1, status);
                __syncwarp();
                tc_fence_after();
                uint32_t sv[128];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld32(tl + T_S + TK * x + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * q]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfree[x]);
                // keys past the end of the row do not take part
                if (k0 + TK > t.ce) {
#pragma unroll
                    for (int e = 0; e < TK; ++e)
                        if (k0 + e >= t.ce) sv[e] = __float_as_uint(-INFINITY);
                }
                float m4[4];  // four independent chains over keys 8 i + 2 a, 8 i + 2 a + 1
#pragma unroll
                for (int a = 0; a < 4; ++a) m4[a] = fmaxf(__uint_as_float(sv[2 * a]), __uint_as_float(sv[2 * a + 1]));
#pragma unroll
                for (int e = 8; e < TK; e += 8)
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        m4[a] = fmax3(m4[a], __uint_as_float(sv[e + 2 * a]), __uint_as_float(sv[e + 2 * a + 1]));
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
                if (mx > m + kLazy) {
                    if (m != -INFINITY) {
                        const float alpha = ex2_approx(m - mx);
                        l *= alpha;
                        mbar_wait(&pvdone[x], (c - 1) & 1, status);  // every PV product on O_x has landed
                        __syncwarp();
                        tc_fence_after();
#pragma unroll 1
                        for (int hc = 0; hc < 64; hc += 32) {  // 32 columns at a time: S stays in registers
                            uint32_t o[32];
                            tmem_ld32(tl + T_O + 64 * x + hc, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st32(tl + T_O + 64 * x + hc, o);
                        }
                        tmem_st_wait();
                    }
                    m = mx;
                }
                if (pp) {
                    if (x == 0) {
                        if (j != 0 || g0_wait_first) named_bar_sync(BAR_G1_DONE, 256);
                    } else {
                        named_bar_sync(BAR_G0_DONE, 256);
                    }
                }
                float2 ls[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};  // pair sums: one add.f32x2 per pair
#pragma unroll
                for (int hk = 0; hk < 2; ++hk) {  // 64 keys at a time; the first half's store overlaps the second
                    // P = 2^x in FP32, FP32 row sums, P packed to FP16 pairs (V is FP16).  An FP16 ex2
                    // for two keys measured slower: the special-function unit stayed as busy and the
                    // conversions added instructions.
                    uint32_t pk[32];
#pragma unroll
                    for (int e = 0; e < 64; e += 2) {
                        const float2 xv = fma2(make_float2(__uint_as_float(sv[64 * hk + e]), __uint_as_float(sv[64 * hk + e + 1])),
                                               make_float2(sl2, sl2), make_float2(-m, -m));
                        float p0, p1;
                        if (((e >> 1) & 7) < JD_EX2_POLY_OF8) {
                            ex2_poly2(xv.x, xv.y, p0, p1);
                        } else {
                            p0 = ex2_approx(xv.x);
                            p1 = ex2_approx(xv.y);
                        }
                        ls[(e >> 1) & 3] = add2(ls[(e >> 1) & 3], make_float2(p0, p1));
                        pk[e >> 1] = pack_f16x2(p0, p1);
                    }
                    if (hk == 0) {
                        // P_x consumed by the last product (the previous item's, then also its O_x final)
                        if (j != 0 || rd_pend) mbar_wait(&pvdone[x], (c - 1) & 1, status);
                        __syncwarp();
                        tc_fence_after();
                    }
                    tmem_st32(tl + T_P + 64 * x + 32 * hk, pk);
                }
                if (pp) {
                    if (x == 0) named_bar_arrive(BAR_G0_DONE, 256);
                    else if (j != t.nt - 1 || g1_hand_last) named_bar_arrive(BAR_G1_DONE, 256);
                }
                l += ((ls[0].x + ls[0].y) + (ls[1].x + ls[1].y)) + ((ls[2].x + ls[2].y) + (ls[3].x + ls[3].y));
                if (rd_pend) readout();
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pready[x]);
            }
            // O / l for this item's query rows, read out after the next item's first P store
            rd_pend = true;
            rd_dst = qi < t.ce ? out + (size_t)qi * D + t.h * DH : nullptr;
            rd_inv = 1.0f / l;
        }
        if (rd_pend) {
            mbar_wait(&pvdone[x], (c - 1) & 1, status);
            readout();
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

cudaError_t attn_tc_init_attributes() {
    // The register split above assumes the compiled count: refuse to run on any other, since a
    // softmax warp group asking for more registers than the launch holds would wait forever.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, k_attn_tc);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != ATC_REGS) return cudaErrorInvalidKernelImage;
    return cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, ATC_SMEM);
}

cudaError_t launch_attention_tc(const AttnArgs &a, const CUtensorMap *tm128, int num_sms, cudaStream_t st) {
    if (a.n_rows <= 0 || a.n_tokens <= 0) return cudaSuccess;
    if (a.window >= 0) return cudaErrorInvalidValue;  // global attention only
    // an upper bound of the work items; CTAs beyond the real count exit at once
    const long items = ((long)a.n_tokens / (2 * TQ) + a.n_rows) * NH;
    const int grid = (int)(items < num_sms ? items : num_sms);
    k_attn_tc<<<grid, ATC_THREADS, ATC_SMEM, st>>>(*tm128, (__nv_bfloat16 *)a.o, a.cu_seqlens, a.qb_off, a.n_rows,
                                                   a.status);
    return cudaGetLastError();
}

}  // namespace jd
