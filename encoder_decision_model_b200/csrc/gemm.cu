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
    for (int r = warp; r < 128; r += 8) {
        const int row = m0 + r;
        if (row >= ep.rows) break;
        epi_row<EPI, __nv_bfloat16, BN>(stg + r * C::PITCH, row, n0, ep, lane);
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

cudaError_t gemm_init_attributes() {
    cudaError_t e;
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

cudaError_t launch_gemm(const GemmOp &op, bool fp32, cudaStream_t st) {
    if (op.ep.rows <= 0) return cudaSuccess;
    if (op.N % op.bn != 0 || op.K % 64 != 0) return cudaErrorInvalidValue;
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
