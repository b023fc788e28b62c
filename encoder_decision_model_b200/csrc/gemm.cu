// Projection GEMMs with fused epilogues: out = epilogue(A[rows, K] . W[N, K]^T).
//
// BF16 path (sm_100a): one 128 x BN output tile per CTA, 256 threads.
//   warp 0 lane 0  TMA producer: A (128 x 64) and W (BN x 64) bf16 boxes with
//                  128-byte swizzle into a STAGES-deep shared-memory ring;
//   warp 1         allocates TMEM; lane 0 issues tcgen05.mma (M=128, K=16,
//                  N = BN or 2 x 192) into an FP32 TMEM accumulator and
//                  releases ring slots with tcgen05.commit;
//   warps 0..3     drain TMEM (tcgen05.ld 32x32b, one row per thread) into a
//                  row-major FP32 staging tile that reuses the ring's memory;
//   warps 0..7     run the epilogue one row per warp (epilogue.cuh).
// FP32 validation path: the same tile shape and epilogue, with a plain SIMT
// FP32 product filling the staging tile.
//
// "julia1 -- Rust runtime for Julia-1", "Why it is faster": BF16 GEMMs with
// FP32 accumulation and fused epilogues (bias, ReLU, residual add, GEGLU).

#include <algorithm>

#include "epilogue.cuh"
#include "kernels.h"

namespace jd {

template <int BN>
struct TcCfg {
    static constexpr int MMA_N = (BN == 384) ? 192 : BN;
    static constexpr int NMMA = BN / MMA_N;
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN == 384) ? 3 : 4;
    static constexpr int PITCH = BN + 4;
    static constexpr int PIPE = STAGES * STAGE;
    static constexpr int STAGING = 128 * PITCH * 4;
    static constexpr int DATA = PIPE > STAGING ? PIPE : STAGING;
    static constexpr int BAR_BYTES = (2 * STAGES + 1) * 8 + 8;
    static constexpr int SMEM = DATA + BAR_BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = (BN <= 256) ? 256 : 512;
};

template <int EPI, int BN>
__global__ void __launch_bounds__(256, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int K, EpiParams ep) {
    using C = TcCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::DATA);
    uint64_t *empty = full + C::STAGES;
    uint64_t *accf = empty + C::STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accf + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int m0 = blockIdx.y * 128;
    const int KB = K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if constexpr (EPI == EPI_RESID_LN) {
        // the residual rows of this tile are contiguous: pull them into L2 while the MMAs run
        if (warp == 2 && lane == 0) {
            const int nrows = min(128, ep.rows - m0);
            const uint8_t *src = reinterpret_cast<const uint8_t *>(ep.resid + (size_t)m0 * D);
            const uint32_t bytes = nrows > 0 ? (uint32_t)nrows * D * 4 : 0u;
            for (uint32_t off = 0; off < bytes; off += 32768u)
                bulk_prefetch_l2(src + off, min(32768u, bytes - off));
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && lane == 0) {
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % C::STAGES;
            if (kb >= C::STAGES && !mbar_wait(&empty[s], ((kb / C::STAGES) - 1) & 1, ep.status)) break;
            uint8_t *sa = smem + s * C::STAGE;
            mbar_arrive_expect_tx(&full[s], C::STAGE);
            tma_load_2d(sa, &tmA, &full[s], kb * 64, m0);
#pragma unroll
            for (int j = 0; j < C::NMMA; ++j)
                tma_load_2d(sa + C::A_BYTES + j * C::MMA_N * 128, &tmB, &full[s], kb * 64, n0 + j * C::MMA_N);
        }
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(C::MMA_N);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int s = kb % C::STAGES;
            if (!mbar_wait(&full[s], (kb / C::STAGES) & 1, ep.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_base = smem_u32(smem + s * C::STAGE);
            const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
#pragma unroll
                for (int j = 0; j < C::NMMA; ++j) {
                    const uint64_t ad = sdesc_sw128(a_base + k * 32);
                    const uint64_t bd = sdesc_sw128(b_base + j * C::MMA_N * 128 + k * 32);
                    tc_mma_bf16(tmem + j * C::MMA_N, ad, bd, idesc, (kb | k) != 0);
                }
            }
            tc_commit(&empty[s]);
        }
        (void)ok;
        tc_commit(accf);
    }
    __syncwarp();
    const bool have_acc = mbar_wait(accf, 0, ep.status);
    __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the wait
    tc_fence_after();

    float *stg = reinterpret_cast<float *>(smem);
    if (warp < 4) {
        const int r = warp * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c, v);
            tmem_ld_wait();
            float4 *dst = reinterpret_cast<float4 *>(stg + r * C::PITCH + c);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                     __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (!have_acc) return;
    if constexpr (EPI == EPI_RESID_LN) {
        // warp w takes rows w + 8u; four of them in flight at a time
        for (int r = warp; r < 128; r += 32) {
            const int row = m0 + r;
            if (row >= ep.rows) break;
            const int n = min(4, (ep.rows - row + 7) / 8);
            epi_resid_ln_rows<__nv_bfloat16, 4>(stg + r * C::PITCH, C::PITCH, row, 8, n, ep, lane);
        }
    } else {
        for (int r = warp; r < 128; r += 8) {
            const int row = m0 + r;
            if (row >= ep.rows) break;
            epi_row<EPI, __nv_bfloat16, BN>(stg + r * C::PITCH, row, n0, ep, lane);
        }
    }
}

// ---------------------------------------------------------------- persistent BF16 GEMM (N-split epilogues)
//
// One CTA per SM loops over 128 x BN tiles (tile t -> m = t / NB, n = t % NB,
// so the NB column blocks of one row block run side by side and share A in
// L2).  Two TMEM accumulators: the epilogue warps drain tile i while the MMA
// warp fills the other buffer with tile i + 1.
//   warp 0 lane 0  TMA producer (A 128 x 64, W BN x 64 per stage)
//   warp 1         TMEM allocation; lane 0 issues tcgen05.mma
//   warps 2..5     epilogue, one accumulator row per thread (TMEM lane
//                  quarter = warp % 4), results stored straight to global
template <int BN>
struct PcCfg {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN <= 192) ? 5 : 4;
    static constexpr int DATA = STAGES * STAGE;
    static constexpr int BAR_BYTES = (2 * STAGES + 4) * 8 + 8;
    static constexpr int SMEM = DATA + BAR_BYTES + 1024;
    static constexpr uint32_t BUF_COLS = 256;  // column stride of the two accumulators
};

template <int EPI, int BN>
__device__ __forceinline__ void pc_epilogue_row(uint32_t tacc, int row, bool valid, int n0, const EpiParams &ep,
                                                const float2 (&cs)[32], bool have_cs) {
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(ep.out) + (size_t)row * ep.ldo;
    if constexpr (EPI == EPI_GEGLU) {
        constexpr int G = BN / 2;
#pragma unroll 1
        for (int c = 0; c < G; c += 32) {
            uint32_t u[32], g[32];
            tmem_ld32(tacc + c, u);
            tmem_ld32(tacc + G + c, g);
            tmem_ld_wait();
            if (valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(o + n0 / 2 + c);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = q * 8 + e * 2;
                        const float y0 = gelu_erf(__uint_as_float(u[j])) * __uint_as_float(g[j]);
                        const float y1 = gelu_erf(__uint_as_float(u[j + 1])) * __uint_as_float(g[j + 1]);
                        w[e] = pack_bf16x2(y0, y1);
                    }
                    dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    } else if constexpr (EPI == EPI_BIAS_ACT) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
            uint32_t a[32];
            tmem_ld32(tacc + c, a);
            tmem_ld_wait();
            if (valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(o + n0 + c);
                const float *bb = ep.bias + n0 + c;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = q * 8 + e * 2;
                        float y0 = __uint_as_float(a[j]) + (bb ? bb[j] : 0.f);
                        float y1 = __uint_as_float(a[j + 1]) + (bb ? bb[j + 1] : 0.f);
                        if (ep.act == 0) { y0 = fmaxf(y0, 0.f); y1 = fmaxf(y1, 0.f); }
                        else { y0 = gelu_erf(y0); y1 = gelu_erf(y1); }
                        w[e] = pack_bf16x2(y0, y1);
                    }
                    dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    } else {  // EPI_QKV: 64-column heads, rotary pairs (i, i + 32) on columns < rope_cols
#pragma unroll 1
        for (int h = 0; h < BN; h += 64) {
            uint32_t a[32], b[32];
            tmem_ld32(tacc + h, a);
            tmem_ld32(tacc + h + 32, b);
            tmem_ld_wait();
            if (!valid) continue;
            const int n = n0 + h;
            const bool rot = have_cs && n < ep.rope_cols;
            uint4 *d1 = reinterpret_cast<uint4 *>(o + n);
            uint4 *d2 = reinterpret_cast<uint4 *>(o + n + 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t w1[4], w2[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float r[2], s[2];
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int j = q * 8 + e * 2 + t;
                        float x1 = __uint_as_float(a[j]), x2 = __uint_as_float(b[j]);
                        if (ep.bias) { x1 += ep.bias[n + j]; x2 += ep.bias[n + 32 + j]; }
                        if (rot) {
                            const float2 c2 = cs[j];
                            r[t] = x1 * c2.x - x2 * c2.y;
                            s[t] = x2 * c2.x + x1 * c2.y;
                        } else {
                            r[t] = x1;
                            s[t] = x2;
                        }
                    }
                    w1[e] = pack_bf16x2(r[0], r[1]);
                    w2[e] = pack_bf16x2(s[0], s[1]);
                }
                d1[q] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
                d2[q] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
            }
        }
    }
}

template <int EPI, int BN>
__global__ void __launch_bounds__(192, 1)
    k_gemm_pc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int K, int n_tiles,
              int nblk, EpiParams ep) {
    using C = PcCfg<BN>;
    static_assert(BN <= 256, "one MMA per k-step");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::DATA);
    uint64_t *empty = full + C::STAGES;
    uint64_t *accf = empty + C::STAGES;   // [2]
    uint64_t *acce = accf + 2;            // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acce + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&accf[0], 1);
        mbar_init(&accf[1], 1);
        mbar_init(&acce[0], 4);
        mbar_init(&acce[1], 4);
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
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
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const int m0 = (t / nblk) * 128, n0 = (t % nblk) * BN;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES;
                    if (it >= (uint32_t)C::STAGES && !mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, ep.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + s * C::STAGE;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(sa, &tmA, &full[s], kb * 64, m0);
                    tma_load_2d(sa + C::A_BYTES, &tmB, &full[s], kb * 64, n0);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(BN);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
                const uint32_t buf = tc & 1, use = tc >> 1;
                if (tc >= 2 && !mbar_wait(&acce[buf], (use - 1) & 1, ep.status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + buf * C::BUF_COLS;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES;
                    if (!mbar_wait(&full[s], (it / C::STAGES) & 1, ep.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * C::STAGE);
                    const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_bf16(dacc, sdesc_sw128(a_base + k * 32), sdesc_sw128(b_base + k * 32), idesc,
                                    (kb | k) != 0);
                    tc_commit(&empty[s]);
                }
                tc_commit(&accf[buf]);
            }
        }
    } else {
        const int q = warp & 3;  // TMEM lane quarter of this warp
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
            const int m0 = (t / nblk) * 128, n0 = (t % nblk) * BN;
            const int row = m0 + q * 32 + lane;
            const bool valid = row < ep.rows;
            float2 cs[32];
            bool have_cs = false;
            if constexpr (EPI == EPI_QKV) {
                if (ep.rope && n0 < ep.rope_cols) {
                    const int pos = valid ? ep.pos[row] : 0;
                    const float4 *src = reinterpret_cast<const float4 *>(ep.rope + (size_t)pos * 32);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float4 v = src[i];
                        cs[2 * i] = make_float2(v.x, v.y);
                        cs[2 * i + 1] = make_float2(v.z, v.w);
                    }
                    have_cs = true;
                }
            }
            const uint32_t buf = tc & 1;
            if (!mbar_wait(&accf[buf], (tc >> 1) & 1, ep.status)) break;
            __syncwarp();
            tc_fence_after();
            const uint32_t tacc = tmem + buf * C::BUF_COLS + ((uint32_t)(q * 32) << 16);
            pc_epilogue_row<EPI, BN>(tacc, row, valid, n0, ep, cs, have_cs);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[buf]);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- FP32 validation GEMM

template <int BN>
struct F32Cfg {
    static constexpr int PITCH = BN + 4;
    static constexpr int STAGING = 128 * PITCH * 4;
    static constexpr int AS = 32 * 128 * 4;
    static constexpr int WS = 32 * 64 * 4;
    static constexpr int SMEM = STAGING + AS + WS;
};

template <int EPI, int BN>
__global__ void __launch_bounds__(256, 1)
    k_gemm_f32(const float *__restrict__ A, int lda, const float *__restrict__ W, int K, EpiParams ep) {
    using C = F32Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    float *stg = reinterpret_cast<float *>(smem_raw);
    float *As = stg + 128 * C::PITCH;   // [32][128]
    float *Ws = As + 32 * 128;          // [32][64]
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * 128;
    const int warp = tid >> 5, lane = tid & 31;

    for (int nc = 0; nc < BN; nc += 64) {
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        for (int k0 = 0; k0 < K; k0 += 32) {
            __syncthreads();
            for (int e = tid; e < 128 * 32; e += 256) {
                const int r = e >> 5, k = e & 31;
                const int row = m0 + r;
                As[k * 128 + r] = (row < ep.rows) ? A[(size_t)row * lda + k0 + k] : 0.f;
            }
            for (int e = tid; e < 64 * 32; e += 256) {
                const int n = e >> 5, k = e & 31;
                Ws[k * 64 + n] = W[(size_t)(n0 + nc + n) * K + k0 + k];
            }
            __syncthreads();
#pragma unroll 4
            for (int k = 0; k < 32; ++k) {
                float a[8], w[4];
#pragma unroll
                for (int i = 0; i < 8; ++i) a[i] = As[k * 128 + ty * 8 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) w[j] = Ws[k * 64 + tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) stg[(ty * 8 + i) * C::PITCH + nc + tx * 4 + j] = acc[i][j];
    }
    __syncthreads();
    for (int r = warp; r < 128; r += 8) {
        const int row = m0 + r;
        if (row >= ep.rows) break;
        epi_row<EPI, float, BN>(stg + r * C::PITCH, row, n0, ep, lane);
    }
}

// ---------------------------------------------------------------- launchers

template <int EPI, int BN>
static cudaError_t set_attrs() {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<EPI, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<BN>::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_gemm_f32<EPI, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, F32Cfg<BN>::SMEM);
}

static int g_num_sms = 148;

cudaError_t gemm_init_attributes() {
    cudaError_t e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_QKV, 192>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<192>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_GEGLU, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<256>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_BIAS_ACT, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<256>::SMEM)) != cudaSuccess)
        return e;
    if ((e = set_attrs<EPI_QKV, 384>()) != cudaSuccess) return e;
    if ((e = set_attrs<EPI_RESID_LN, 384>()) != cudaSuccess) return e;
    if ((e = set_attrs<EPI_GEGLU, 256>()) != cudaSuccess) return e;
    return set_attrs<EPI_BIAS_ACT, 256>();
}

template <int EPI, int BN>
static cudaError_t launch_tc(const GemmOp &op, cudaStream_t st) {
    using C = TcCfg<BN>;
    dim3 grid(op.N / BN, (op.ep.rows + 127) / 128);
    k_gemm_tc<EPI, BN><<<grid, 256, C::SMEM, st>>>(*op.tmA, *op.tmB, op.K, op.ep);
    return cudaGetLastError();
}

template <int EPI, int BN>
static cudaError_t launch_f32(const GemmOp &op, cudaStream_t st) {
    using C = F32Cfg<BN>;
    dim3 grid(op.N / BN, (op.ep.rows + 127) / 128);
    k_gemm_f32<EPI, BN><<<grid, 256, C::SMEM, st>>>(op.A32, op.lda, op.W32, op.K, op.ep);
    return cudaGetLastError();
}

template <int EPI, int BN>
static cudaError_t launch_pc(const GemmOp &op, cudaStream_t st) {
    if (op.N % BN != 0) return cudaErrorInvalidValue;
    const int nblk = op.N / BN;
    const int n_tiles = nblk * ((op.ep.rows + 127) / 128);
    const int grid = n_tiles < g_num_sms ? n_tiles : g_num_sms;
    k_gemm_pc<EPI, BN><<<grid, 192, PcCfg<BN>::SMEM, st>>>(*op.tmA, *op.tmB, op.K, n_tiles, nblk, op.ep);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmOp &op, bool fp32, cudaStream_t st) {
    if (op.ep.rows <= 0) return cudaSuccess;
    if (op.N % op.bn != 0 || op.K % 64 != 0) return cudaErrorInvalidValue;
    if (!fp32) {  // persistent tcgen05 kernels for the column-split epilogues
        if (op.epi == EPI_QKV) return launch_pc<EPI_QKV, 192>(op, st);
        if (op.epi == EPI_GEGLU) return launch_pc<EPI_GEGLU, 256>(op, st);
        if (op.epi == EPI_BIAS_ACT) return launch_pc<EPI_BIAS_ACT, 256>(op, st);
    }
#define JD_CASE(E, B)                                                  \
    if (op.epi == E && op.bn == B) return fp32 ? launch_f32<E, B>(op, st) : launch_tc<E, B>(op, st);
    JD_CASE(EPI_QKV, 384)
    JD_CASE(EPI_RESID_LN, 384)
    JD_CASE(EPI_GEGLU, 256)
    JD_CASE(EPI_BIAS_ACT, 256)
#undef JD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace jd
