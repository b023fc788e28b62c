// Bidirectional attention inside each packed row on the 5th-generation tensor
// cores, global and +-64-window variants.
//
// "Julia-1 MLX", "Performance": every third encoder layer attends globally,
// the others within +-64 tokens; the two head layers attend over the whole row
// ("Julia-1: one score per mask token", "The decision head", step 2).  Rows
// are packed back to back ("julia1 -- Rust runtime for Julia-1", "Why it is
// faster"); a work item is one 128-query block of one row and one head, and a
// persistent CTA per SM walks the item list.  Keys come in 128-key tiles: all
// of the row's tiles (global), or the two tiles of the band [q0 - 64, q0 + 192)
// (window); keys outside the row or the window get probability zero.
//
//   warp 0 lane 0  TMA producer: Q (128 x 64) once per item into one of two
//                  buffers; K and V tiles (128 keys x 64, 128-byte swizzle) into
//                  a three-stage ring
//   warp 1         TMEM allocation; lane 0 issues tcgen05.mma:
//                    S_j = Q K_j^T      (M 128, N 128, K 64) into one of two S buffers
//                    O  += P_j V_j      (M 128, N 64,  K 128; V read MN-major)
//   warps 2..9     softmax: two warps per TMEM lane quarter, each owning one
//                  query row per thread and one half (64 keys) of every tile;
//                  the halves combine row maxima (and, at the end, row sums)
//                  through shared memory.  The running max is kept lazily: O
//                  and the sums are rescaled only when the max grows by more
//                  than 2^8, so P stays below 256.  P is written as bf16 into
//                  shared memory (K-major, 128-byte swizzle; each half writes
//                  its own 64-key block).
// TMEM columns: S buffers 0 and 128, O at 256.

#include "common.cuh"
#include "kernels.h"

namespace jd {

namespace {
constexpr int TQ = 128, TK = 128;
constexpr int Q_BYTES = TQ * 128;          // 128 rows x 64 bf16
constexpr int KT_BYTES = TK * 128;         // 128 keys x 64 bf16
constexpr int KV_STAGE = 2 * KT_BYTES;     // K tile then V tile
constexpr int P_BYTES = TQ * TK * 2;       // two 64-key blocks of 128 x 128 B
constexpr int NKV = 3;                     // K/V ring depth
constexpr int OFF_Q = 0;                   // two Q buffers (work items alternate)
constexpr int OFF_KV = OFF_Q + 2 * Q_BYTES;
constexpr int OFF_P = OFF_KV + NKV * KV_STAGE;
constexpr int OFF_X = OFF_P + 2 * P_BYTES;           // row exchange: max [2][2][128], sum [2][128]
constexpr int X_BYTES = (2 * 2 * 128 + 2 * 128) * 4;
constexpr int OFF_BAR = OFF_X + X_BYTES;
// qfull[2], qfree[2], kvfull[3], kvempty[3], sfull[2], pready[2], pvdone[2], ofree
constexpr int NBAR = 17;
constexpr int ATC_SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
constexpr uint32_t T_O = 256;
constexpr float kLazy = 8.0f;    // log2 headroom before the running max is moved
constexpr int SM_THREADS = 256;  // softmax warps 2..9
}  // namespace

// 2^x with the hardware approximation (ex2.approx.ftz; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct AtcItem {
    int h, cs, ce, q0, ks0, nt;
};

template <bool LOCAL>
__device__ __forceinline__ AtcItem atc_item(const int *q128, const int *qb_row, const int *cu, int w) {
    AtcItem t;
    const int qb = w / NH;
    t.h = w % NH;
    const int row = qb_row[qb];
    t.cs = cu[row];
    t.ce = cu[row + 1];
    t.q0 = t.cs + (qb - q128[row]) * TQ;
    if (LOCAL) {
        t.ks0 = t.q0 - 64;
        t.nt = 2;
    } else {
        t.ks0 = t.cs;
        t.nt = (t.ce - t.cs + TK - 1) / TK;
    }
    return t;
}

template <bool LOCAL>
__global__ void __launch_bounds__(64 + SM_THREADS, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ out, const int *__restrict__ cu,
              const int *__restrict__ qb_off, int n_rows, unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *xmax = reinterpret_cast<float *>(smem + OFF_X);  // [S buffer][half][row]
    float *xsum = xmax + 2 * 2 * 128;                        // [half][row]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *qfull = bars + 0, *qfree = bars + 2, *kvfull = bars + 4, *kvempty = bars + 7, *sfull = bars + 10,
             *pready = bars + 12, *pvdone = bars + 14, *ofree = bars + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);

    const int *q128 = qb_off + n_rows + 1;
    const int *qb_row = q128 + n_rows + 1;
    const int n_items = q128[n_rows] * NH;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NKV; ++i) {
            mbar_init(&kvfull[i], 1);
            mbar_init(&kvempty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qfree[i], 1);
            mbar_init(&sfull[i], 1);
            mbar_init(&pready[i], SM_THREADS / 32);
            mbar_init(&pvdone[i], 1);
        }
        mbar_init(ofree, SM_THREADS / 32);
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

    if (warp == 0) {
        if (lane == 0) {
            uint32_t J = 0, it = 0;
            for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
                const AtcItem t = atc_item<LOCAL>(q128, qb_row, cu, w);
                const uint32_t qbuf = it & 1;
                if (it >= 2) mbar_wait(&qfree[qbuf], ((it - 2) >> 1) & 1, status);
                mbar_arrive_expect_tx(&qfull[qbuf], Q_BYTES);
                tma_load_2d(smem + OFF_Q + qbuf * Q_BYTES, &tm, &qfull[qbuf], t.h * DH, t.q0);
                for (int j = 0; j < t.nt; ++j, ++J) {
                    const uint32_t s = J % NKV;
                    if (J >= NKV) mbar_wait(&kvempty[s], ((J - NKV) / NKV) & 1, status);
                    uint8_t *st = smem + OFF_KV + s * KV_STAGE;
                    mbar_arrive_expect_tx(&kvfull[s], KV_STAGE);
                    tma_load_2d(st, &tm, &kvfull[s], D + t.h * DH, t.ks0 + j * TK);
                    tma_load_2d(st + KT_BYTES, &tm, &kvfull[s], 2 * D + t.h * DH, t.ks0 + j * TK);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(TK);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(DH) | (1u << 16);  // B (V) is MN-major
            uint32_t J = 0, it = 0;
            for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
                const AtcItem t = atc_item<LOCAL>(q128, qb_row, cu, w);
                const uint32_t qbuf = it & 1;
                const uint32_t q_base = smem_u32(smem + OFF_Q + qbuf * Q_BYTES);
                mbar_wait(&qfull[qbuf], (it >> 1) & 1, status);
                tc_fence_after();
                const uint32_t J0 = J;
                auto issue_pv = [&](uint32_t Jp) {
                    const uint32_t b = Jp & 1;
                    mbar_wait(&pready[b], (Jp >> 1) & 1, status);
                    if (Jp == J0 && it >= 1) mbar_wait(ofree, (it - 1) & 1, status);
                    tc_fence_after();
                    const uint32_t p_base = smem_u32(smem + OFF_P + b * P_BYTES);
                    const uint32_t v_base = smem_u32(smem + OFF_KV + (Jp % NKV) * KV_STAGE + KT_BYTES);
#pragma unroll
                    for (int ks = 0; ks < TK / 16; ++ks) {
                        const uint64_t ad = sdesc_sw128(p_base + (ks >> 2) * (TQ * 128) + (ks & 3) * 32);
                        const uint64_t bd = sdesc_sw128(v_base + ks * 16 * 128);
                        tc_mma_bf16(tmem + T_O, ad, bd, idesc_pv, (Jp != J0 || ks != 0) ? 1u : 0u);
                    }
                    tc_commit(&pvdone[b]);
                    tc_commit(&kvempty[Jp % NKV]);
                };
                for (int j = 0; j < t.nt; ++j, ++J) {
                    const uint32_t b = J & 1, s = J % NKV;
                    mbar_wait(&kvfull[s], (J / NKV) & 1, status);
                    if (J >= 2) mbar_wait(&pready[b], ((J - 2) >> 1) & 1, status);  // S buffer b read out
                    tc_fence_after();
                    const uint32_t k_base = smem_u32(smem + OFF_KV + s * KV_STAGE);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem + b * TK, sdesc_sw128(q_base + kk * 32), sdesc_sw128(k_base + kk * 32),
                                    idesc_s, kk != 0);
                    tc_commit(&sfull[b]);
                    if (j == t.nt - 1) tc_commit(&qfree[qbuf]);
                    if (j >= 1) issue_pv(J - 1);
                }
                issue_pv(J - 1);
            }
        }
    } else {
        const int q = warp & 3;            // TMEM lane quarter
        const int hf = (warp - 2) >> 2;    // which 64-key half of each tile
        const int r = q * 32 + lane;       // query row inside the item
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const float sl2 = 0.125f * 1.4426950408889634f;
        uint32_t J = 0, it = 0;
        for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
            const AtcItem t = atc_item<LOCAL>(q128, qb_row, cu, w);
            const int qi = t.q0 + r;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < t.nt; ++j, ++J) {
                const uint32_t b = J & 1;
                const int k0 = t.ks0 + j * TK + hf * 64;  // first key of this thread's half tile
                mbar_wait(&sfull[b], (J >> 1) & 1, status);
                __syncwarp();
                tc_fence_after();
                uint32_t sv[64];
                tmem_ld32(tl + b * TK + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(tl + b * TK + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_ld_wait();
                // keys outside the row (and, windowed, outside |i - j| <= 64) do not take part
                const bool full = LOCAL ? false : (k0 + 64 <= t.ce);
                if (!full) {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const int key = k0 + e;
                        bool ok = key >= t.cs && key < t.ce;
                        if (LOCAL) ok = ok && abs(qi - key) <= 64;
                        if (!ok) sv[e] = __float_as_uint(-INFINITY);
                    }
                }
                float m8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(sv[e]);
#pragma unroll
                for (int e = 8; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(sv[e]));
                const float mh = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                // combine with the other half of the row (per S buffer, so the
                // next tile's write cannot overtake the partner's read)
                xmax[((b * 2) + hf) * 128 + r] = mh;
                named_bar_sync(1, SM_THREADS);
                const float mx = fmaxf(mh, xmax[((b * 2) + (hf ^ 1)) * 128 + r]) * sl2;
                if (mx > m + kLazy) {
                    if (m != -INFINITY) {
                        const float alpha = ex2_approx(m - mx);
                        l *= alpha;
                        mbar_wait(&pvdone[(J - 1) & 1], ((J - 1) >> 1) & 1, status);
                        __syncwarp();
                        tc_fence_after();
                        uint32_t o[32];  // this half rescales O columns [32 hf, 32 hf + 32)
                        tmem_ld32(tl + T_O + hf * 32, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tl + T_O + hf * 32, o);
                        tmem_st_wait();
                    }
                    m = mx;
                }
                if (J >= 2) mbar_wait(&pvdone[b], ((J - 2) >> 1) & 1, status);  // P buffer b read by the MMA
                uint8_t *blk = smem + OFF_P + b * P_BYTES + hf * (TQ * 128);
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 64; c += 32) {
                    uint32_t w16[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[c + e]), sl2, -m));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[c + e + 1]), sl2, -m));
                        ls[(e >> 1) & 3] += p0 + p1;
                        w16[e >> 1] = pack_bf16x2(p0, p1);
                    }
                    const int ch0 = c >> 3;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        *reinterpret_cast<uint4 *>(blk + r * 128 + (((ch0 + k4) ^ (r & 7)) << 4)) =
                            make_uint4(w16[4 * k4], w16[4 * k4 + 1], w16[4 * k4 + 2], w16[4 * k4 + 3]);
                }
                l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pready[b]);
            }
            // O / (l_half0 + l_half1) for this item; this half stores O columns [32 hf, 32 hf + 32)
            xsum[hf * 128 + r] = l;
            named_bar_sync(1, SM_THREADS);
            const float ltot = l + xsum[(hf ^ 1) * 128 + r];
            mbar_wait(&pvdone[(J - 1) & 1], ((J - 1) >> 1) & 1, status);
            __syncwarp();
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32(tl + T_O + hf * 32, o);
            tmem_ld_wait();
            named_bar_sync(1, SM_THREADS);  // both halves have read xsum before the next item writes it
            if (qi < t.ce) {
                const float inv = 1.0f / ltot;
                uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)qi * D + t.h * DH + hf * 32);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    uint32_t wv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(o[8 * k4 + 2 * e]) * inv,
                                            __uint_as_float(o[8 * k4 + 2 * e + 1]) * inv);
                    dst[k4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ofree);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

cudaError_t attn_tc_init_attributes() {
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATC_SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_attn_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATC_SMEM);
}

cudaError_t launch_attention_tc(const AttnArgs &a, const CUtensorMap *tm128, int num_sms, cudaStream_t st) {
    if (a.n_rows <= 0 || a.n_tokens <= 0) return cudaSuccess;
    // an upper bound of the work items; CTAs beyond the real count exit at once
    const long items = ((long)a.n_tokens / TQ + a.n_rows) * NH;
    const int grid = (int)(items < num_sms ? items : num_sms);
    if (a.window >= 0)
        k_attn_tc<true><<<grid, 64 + SM_THREADS, ATC_SMEM, st>>>(*tm128, (__nv_bfloat16 *)a.o, a.cu_seqlens,
                                                                   a.qb_off, a.n_rows, a.status);
    else
        k_attn_tc<false><<<grid, 64 + SM_THREADS, ATC_SMEM, st>>>(*tm128, (__nv_bfloat16 *)a.o, a.cu_seqlens,
                                                                    a.qb_off, a.n_rows, a.status);
    return cudaGetLastError();
}

}  // namespace jd
