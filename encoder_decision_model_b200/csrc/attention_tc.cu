// Global (full-row) bidirectional attention on the 5th-generation tensor cores.
//
// "Julia-1 MLX", "Performance": every third encoder layer attends globally;
// the two head layers attend over the whole row too ("Julia-1: one score per
// mask token", "The decision head", step 2).  Rows are packed back to back
// ("julia1 -- Rust runtime for Julia-1", "Why it is faster"); a work item is
// one 128-query block of one row and one head, and a persistent CTA per SM
// walks the item list.
//
//   warp 0 lane 0  TMA producer: Q (128 x 64) once per item into one of two
//                  buffers; K and V tiles (128 keys x 64, 128-byte swizzle) into
//                  a four-stage ring
//   warp 1         TMEM allocation; lane 0 issues tcgen05.mma:
//                    S_j = Q K_j^T      (M 128, N 128, K 64) into one of two S buffers
//                    O  += P_j V_j      (M 128, N 64,  K 128; V read MN-major)
//   warps 2..5     softmax, one query row per thread: the 128-score row read
//                  from TMEM once into registers, running
//                  max kept lazily (O and the running sum are rescaled only when
//                  the max grows by more than 2^8, so P stays below 256), P
//                  written as bf16 into shared memory (K-major, 128-byte
//                  swizzle), final O / l stored as bf16.
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
constexpr int NKV = 4;                     // K/V ring depth
constexpr int OFF_Q = 0;                   // two Q buffers (work items alternate)
constexpr int OFF_KV = OFF_Q + 2 * Q_BYTES;
constexpr int OFF_P = OFF_KV + NKV * KV_STAGE;
constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
// qfull[2], qfree[2], kvfull[4], kvempty[4], sfull[2], pready[2], pvdone[2], ofree
constexpr int NBAR = 19;
constexpr int ATC_SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
constexpr uint32_t T_O = 256;
constexpr float kLazy = 8.0f;  // log2 headroom before the running max is moved
}  // namespace

// 2^x with the hardware approximation (ex2.approx.ftz; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ int atc_row(const int *q128, int n_rows, int qb) {
    int lo = 0, hi = n_rows - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (q128[mid] <= qb) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(192, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tm, __nv_bfloat16 *__restrict__ out, const int *__restrict__ cu,
              const int *__restrict__ qb_off, int n_rows, unsigned *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
    uint64_t *qfull = bars + 0, *qfree = bars + 2, *kvfull = bars + 4, *kvempty = bars + 8, *sfull = bars + 12,
             *pready = bars + 14, *pvdone = bars + 16, *ofree = bars + 18;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBAR);

    const int *q128 = qb_off + n_rows + 1;
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
            mbar_init(&pready[i], 4);
            mbar_init(&pvdone[i], 1);
        }
        mbar_init(ofree, 4);
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
                const int qb = w / NH, h = w % NH;
                const int row = atc_row(q128, n_rows, qb);
                const int cs = cu[row], ce = cu[row + 1];
                const int q0 = cs + (qb - q128[row]) * TQ;
                const int nt = (ce - cs + TK - 1) / TK;
                const uint32_t qbuf = it & 1;
                if (it >= 2) mbar_wait(&qfree[qbuf], ((it - 2) >> 1) & 1, status);
                mbar_arrive_expect_tx(&qfull[qbuf], Q_BYTES);
                tma_load_2d(smem + OFF_Q + qbuf * Q_BYTES, &tm, &qfull[qbuf], h * DH, q0);
                for (int j = 0; j < nt; ++j, ++J) {
                    const uint32_t s = J % NKV;
                    if (J >= NKV) mbar_wait(&kvempty[s], ((J - NKV) / NKV) & 1, status);
                    uint8_t *st = smem + OFF_KV + s * KV_STAGE;
                    mbar_arrive_expect_tx(&kvfull[s], KV_STAGE);
                    tma_load_2d(st, &tm, &kvfull[s], D + h * DH, cs + j * TK);
                    tma_load_2d(st + KT_BYTES, &tm, &kvfull[s], 2 * D + h * DH, cs + j * TK);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(TK);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(DH) | (1u << 16);  // B (V) is MN-major
            uint32_t J = 0, it = 0;
            for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
                const int qb = w / NH;
                const int row = atc_row(q128, n_rows, qb);
                const int nt = (cu[row + 1] - cu[row] + TK - 1) / TK;
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
                for (int j = 0; j < nt; ++j, ++J) {
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
                    if (j == nt - 1) tc_commit(&qfree[qbuf]);
                    if (j >= 1) issue_pv(J - 1);
                }
                issue_pv(J - 1);
            }
        }
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const float sl2 = 0.125f * 1.4426950408889634f;
        uint32_t J = 0, it = 0;
        for (int w = blockIdx.x; w < n_items; w += gridDim.x, ++it) {
            const int qb = w / NH, h = w % NH;
            const int row = atc_row(q128, n_rows, qb);
            const int cs = cu[row], ce = cu[row + 1];
            const int q0 = cs + (qb - q128[row]) * TQ;
            const int nt = (ce - cs + TK - 1) / TK;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < nt; ++j, ++J) {
                const uint32_t b = J & 1;
                const int nvalid = ce - (cs + j * TK);  // keys of this tile inside the row (>= 1)
                mbar_wait(&sfull[b], (J >> 1) & 1, status);
                __syncwarp();
                tc_fence_after();
                // the whole 128-score row in registers: one TMEM pass
                uint32_t sv[TK];
                tmem_ld32(tl + b * TK, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(tl + b * TK + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_ld32(tl + b * TK + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
                tmem_ld32(tl + b * TK + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
                tmem_ld_wait();
                if (nvalid < TK) {  // last tile of the row: keys past its end do not exist
#pragma unroll
                    for (int e = 0; e < TK; ++e)
                        if (e >= nvalid) sv[e] = __float_as_uint(-INFINITY);
                }
                float m8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(sv[e]);
#pragma unroll
                for (int e = 8; e < TK; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(sv[e]));
                float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                 fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                mx *= sl2;
                if (mx > m + kLazy) {
                    if (j > 0) {
                        const float alpha = ex2_approx(m - mx);
                        l *= alpha;
                        mbar_wait(&pvdone[(J - 1) & 1], ((J - 1) >> 1) & 1, status);
                        tc_fence_after();
                        uint32_t o1[32], o2[32];
                        tmem_ld32(tl + T_O, o1);
                        tmem_ld32(tl + T_O + 32, o2);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            o1[e] = __float_as_uint(__uint_as_float(o1[e]) * alpha);
                            o2[e] = __float_as_uint(__uint_as_float(o2[e]) * alpha);
                        }
                        tmem_st32(tl + T_O, o1);
                        tmem_st32(tl + T_O + 32, o2);
                        tmem_st_wait();
                    }
                    m = mx;
                }
                if (J >= 2) mbar_wait(&pvdone[b], ((J - 2) >> 1) & 1, status);  // P buffer b read by the MMA
                uint8_t *pb = smem + OFF_P + b * P_BYTES;
                // P = exp2(s * scale - m) in bf16, K-major with the 128-byte swizzle
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < TK; c += 32) {
                    uint32_t w16[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const float x0 = fmaf(__uint_as_float(sv[c + e]), sl2, -m);
                        const float x1 = fmaf(__uint_as_float(sv[c + e + 1]), sl2, -m);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        ls[(e >> 1) & 3] += p0 + p1;
                        w16[e >> 1] = pack_bf16x2(p0, p1);
                    }
                    uint8_t *blk = pb + (c >> 6) * (TQ * 128);
                    const int ch0 = (c & 63) >> 3;
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
            // O / l for this item
            mbar_wait(&pvdone[(J - 1) & 1], ((J - 1) >> 1) & 1, status);
            __syncwarp();
            tc_fence_after();
            uint32_t o1[32], o2[32];
            tmem_ld32(tl + T_O, o1);
            tmem_ld32(tl + T_O + 32, o2);
            tmem_ld_wait();
            const int qi = q0 + r;
            if (qi < ce) {
                const float inv = 1.0f / l;
                uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)qi * D + h * DH);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    uint32_t wv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(o1[8 * k4 + 2 * e]) * inv,
                                            __uint_as_float(o1[8 * k4 + 2 * e + 1]) * inv);
                    dst[k4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                }
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    uint32_t wv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(o2[8 * k4 + 2 * e]) * inv,
                                            __uint_as_float(o2[8 * k4 + 2 * e + 1]) * inv);
                    dst[4 + k4] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
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
    return cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, ATC_SMEM);
}

cudaError_t launch_attention_tc(const AttnArgs &a, const CUtensorMap *tm128, int num_sms, cudaStream_t st) {
    if (a.n_rows <= 0 || a.n_tokens <= 0) return cudaSuccess;
    // an upper bound of the work items; CTAs beyond the real count exit at once
    const long items = ((long)a.n_tokens / TQ + a.n_rows) * NH;
    const int grid = (int)(items < num_sms ? items : num_sms);
    k_attn_tc<<<grid, 192, ATC_SMEM, st>>>(*tm128, (__nv_bfloat16 *)a.o, a.cu_seqlens, a.qb_off, a.n_rows, a.status);
    return cudaGetLastError();
}

}  // namespace jd
