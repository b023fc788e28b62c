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

// ---------------------------------------------------------------- persistent BF16 GEMM (column-split epilogues)
//
// One CTA per SM loops over 128 x BN tiles (tile t -> m = t / NB, n = t % NB,
// so the NB column blocks of one row block run side by side and share A in
// L2).  Two TMEM accumulators: the epilogue warps drain tile i while the MMA
// warp fills the other buffer with tile i + 1.
//   warp 0 lane 0  TMA producer (A 128 x 64, W BN x 64 per stage)
//   warp 1         TMEM allocation; lane 0 issues tcgen05.mma
//   warps 2..      epilogue, one accumulator row per thread (TMEM lane
//                  quarter = warp % 4; GEGLU runs two warps per quarter, each
//                  on half of the output columns); QKV and bias+activation outputs are
//                  staged per warp as 32 rows x 64 columns (bf16, 128-byte
//                  swizzle) in shared memory and written by one TMA bulk
//                  store each (double-buffered); GEGLU outputs go straight
//                  from registers to global memory.
constexpr int GEGLU_EW = 8;  // GEGLU epilogue warps (16 measured no faster)
#ifndef JD_PC_NBUF
#define JD_PC_NBUF 3
#endif

template <int BN>
struct PcCfg {
    static constexpr int A_BYTES = 128 * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = 4;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int OUT_BOX = 32 * 128;           // 32 rows x 64 bf16
    // staging buffers per epilogue warp: three where the shared memory allows (a 192-wide tile
    // has three boxes per warp, so none waits on the store of the same tile)
    static constexpr int NBUF = BN <= 192 ? JD_PC_NBUF : 2;
    static constexpr int OUT = 4 * NBUF * OUT_BOX;     // 4 warps x NBUF buffers
    static constexpr int DATA = RING + OUT;
    static constexpr int BAR_BYTES = (2 * STAGES + 4) * 8 + 8;
    static constexpr int SMEM = DATA + BAR_BYTES + 1024;
    static constexpr uint32_t BUF_COLS = 256;          // column stride of the two accumulators
};

// Per-warp staging of 32 x 64 bf16 boxes for TMA stores, NB buffers used in turn.
template <int NB>
struct OutStage {
    uint8_t *base;   // this warp's NB 4 KB buffers
    uint32_t count;  // boxes issued so far
    __device__ __forceinline__ uint8_t *begin(int lane) {
        if (count >= NB) {
            if (lane == 0) bulk_wait_read<NB - 1>();  // the store that used this buffer has read it
            __syncwarp();
        }
        return base + (count % NB) * 4096;
    }
    __device__ __forceinline__ void commit(uint8_t *buf, const CUtensorMap *map, int x, int y, int lane) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(map, buf, x, y);
            bulk_commit();
        }
        ++count;
    }
};

// Write 4 x 16 bytes (32 bf16) of row r into 16-byte chunks c0..c0+3 of a swizzled box.
// GELU(u) * g for a pair of columns, FP32, on packed f32x2 FMAs and one ex2 per value.
// GELU(x) = x Phi(x) = max(x, 0) - |x| Phi(-|x|), and the normal tail is written as
// Phi(-a) = 2^(P(a / 6) - a^2 log2(e) / 2), P the degree-7 polynomial of least maximum error
// against log2 Phi(-6 s) + 18 s^2 log2(e) on s in [0, 1] (Remez exchange; |error| <= 4.8e-6 in
// log2, a relative error of 3.3e-6 in the tail, so |GELU error| < 1e-6).  Past |x| = 6 the
// polynomial is held at s = 1 while the Gaussian factor keeps falling; the tail there is below
// 1e-9.  erf's rational form (Abramowitz and Stegun 7.1.26) needs a reciprocal and an ex2 per
// value: the special-function unit then worked as long as the tile's MMAs.
constexpr float GT_C0 = -0.9999952912330627f, GT_C1 = -6.907506465911865f, GT_C2 = 9.46379280090332f,
                GT_C3 = -11.655374526977539f, GT_C4 = 11.026226043701172f, GT_C5 = -7.235760688781738f,
                GT_C6 = 2.873929500579834f, GT_C7 = -0.5136296153068542f;
constexpr float GT_G = -25.968510341644287f;  // -36 log2(e) / 2: the Gaussian factor in s
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 f2c(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 geglu_pair(float2 x, float2 g) {
    const float2 na = make_float2(-fabsf(x.x), -fabsf(x.y));
    const float2 s = f2mul(na, f2c(-1.0f / 6.0f));
    const float2 sc = make_float2(fminf(s.x, 1.0f), fminf(s.y, 1.0f));
    float2 p = f2fma(sc, f2c(GT_C7), f2c(GT_C6));
    p = f2fma(p, sc, f2c(GT_C5));
    p = f2fma(p, sc, f2c(GT_C4));
    p = f2fma(p, sc, f2c(GT_C3));
    p = f2fma(p, sc, f2c(GT_C2));
    p = f2fma(p, sc, f2c(GT_C1));
    p = f2fma(p, sc, f2c(GT_C0));
    const float2 arg = f2fma(f2mul(s, s), f2c(GT_G), p);
    float2 t;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t.x) : "f"(arg.x));
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t.y) : "f"(arg.y));
    const float2 y = f2fma(na, t, make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f)));
    return f2mul(y, g);
}

__device__ __forceinline__ void stage_row32(uint8_t *box, int r, int c0, const uint32_t (&w)[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4 *>(box + r * 128 + (((c0 + q) ^ (r & 7)) << 4)) =
            make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

template <int EPI, int BN, int NPART, bool F8 = false>
__device__ __forceinline__ void pc_epilogue_rows(uint32_t tacc, int r, int row0, int n0, const EpiParams &ep,
                                                 const CUtensorMap *tmO, OutStage<PcCfg<BN>::NBUF> &os, int lane,
                                                 const float2 (&cs)[32], bool have_cs, int part) {
    if constexpr (EPI == EPI_GEGLU) {
        // stored straight from registers: a shared-memory staging pass here
        // competes with the 256-wide MMAs for shared-memory bandwidth; with
        // NPART warps per TMEM lane quarter each takes G / NPART output columns.
        // GELU by geglu_pair (one ex2 per value): with erff, and then with erf's rational
        // form, this epilogue kept the special-function unit as busy as the tile's MMAs.
        constexpr int G = BN / 2;
        constexpr int GP = G / NPART;
        static_assert(GP == 64, "two 32-column chunks per warp");
        const int row = row0 + r;
        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(ep.out) + (size_t)row * ep.ldo + n0 / 2;
        auto emit = [&](const uint32_t (&u)[32], const uint32_t (&g)[32], int c) {
            if (row < ep.rows) {  // 32-byte stores: a warp instruction fills whole sectors
                uint8_t *dst = reinterpret_cast<uint8_t *>(o + c);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int j = q * 16 + e * 2;
                        const float2 y = geglu_pair(make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1])),
                                                    make_float2(__uint_as_float(g[j]), __uint_as_float(g[j + 1])));
                        w[e] = pack_bf16x2(y.x, y.y);
                    }
                    st_global_v8(dst + 32 * q, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                }
            }
        };
        // the second chunk's TMEM loads are in flight while the first chunk computes
        const int c0 = part * GP;
        uint32_t u0[32], g0[32], u1[32], g1[32];
        tmem_ld32(tacc + c0, u0);
        tmem_ld32(tacc + G + c0, g0);
        tmem_ld_wait();
        tmem_ld32(tacc + c0 + 32, u1);
        tmem_ld32(tacc + G + c0 + 32, g1);
        emit(u0, g0, c0);
        tmem_ld_wait();
        emit(u1, g1, c0 + 32);
    } else if constexpr (EPI == EPI_BIAS_ACT) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 64) {
            uint8_t *box = os.begin(lane);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t a[32], w[16];
                tmem_ld32(tacc + c + 32 * hh, a);
                tmem_ld_wait();
                const float4 *bb = reinterpret_cast<const float4 *>(ep.bias + n0 + c + 32 * hh);
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 b = ep.bias ? bb[j4] : make_float4(0.f, 0.f, 0.f, 0.f);
                    float y[4] = {__uint_as_float(a[4 * j4]) + b.x, __uint_as_float(a[4 * j4 + 1]) + b.y,
                                  __uint_as_float(a[4 * j4 + 2]) + b.z, __uint_as_float(a[4 * j4 + 3]) + b.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) y[e] = ep.act == 0 ? fmaxf(y[e], 0.f) : gelu_erf(y[e]);
                    w[2 * j4] = pack_bf16x2(y[0], y[1]);
                    w[2 * j4 + 1] = pack_bf16x2(y[2], y[3]);
                }
                stage_row32(box, r, 4 * hh, w);
            }
            os.commit(box, tmO, ep.out_col0 + n0 + c, row0, lane);
        }
    } else {  // EPI_QKV: 64-column heads, rotary pairs (i, i + 32) on columns < rope_cols
#pragma unroll 1
        for (int h = 0; h < BN; h += 64) {
            uint8_t *box = os.begin(lane);
            uint32_t a[32], b[32], w1[16], w2[16];
            tmem_ld32(tacc + h, a);
            tmem_ld32(tacc + h + 32, b);
            tmem_ld_wait();
            const int n = n0 + h;
            const bool rot = have_cs && n < ep.rope_cols;
            const bool vcol = ep.out_col0 + n >= 2 * D;  // v: FP16 (the attention's P V products are FP16)
            float ba[32], bb[32];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
                if (ep.bias) {
                    x = reinterpret_cast<const float4 *>(ep.bias + n)[j4];
                    y = reinterpret_cast<const float4 *>(ep.bias + n + 32)[j4];
                }
                ba[4 * j4] = x.x; ba[4 * j4 + 1] = x.y; ba[4 * j4 + 2] = x.z; ba[4 * j4 + 3] = x.w;
                bb[4 * j4] = y.x; bb[4 * j4 + 1] = y.y; bb[4 * j4 + 2] = y.z; bb[4 * j4 + 3] = y.w;
            }
            float sa[32], sb[32];  // FP8: per-column scales of the E4M3 product (activation x weight row)
            if constexpr (F8) {
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 x = reinterpret_cast<const float4 *>(ep.col_scale + n)[j4];
                    const float4 y = reinterpret_cast<const float4 *>(ep.col_scale + n + 32)[j4];
                    sa[4 * j4] = x.x; sa[4 * j4 + 1] = x.y; sa[4 * j4 + 2] = x.z; sa[4 * j4 + 3] = x.w;
                    sb[4 * j4] = y.x; sb[4 * j4 + 1] = y.y; sb[4 * j4 + 2] = y.z; sb[4 * j4 + 3] = y.w;
                }
            }
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float r2[2], s2[2];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int jj = j + t;
                    const float x1 = F8 ? fmaf(__uint_as_float(a[jj]), sa[jj], ba[jj]) : __uint_as_float(a[jj]) + ba[jj];
                    const float x2 = F8 ? fmaf(__uint_as_float(b[jj]), sb[jj], bb[jj]) : __uint_as_float(b[jj]) + bb[jj];
                    if (rot) {
                        r2[t] = x1 * cs[jj].x - x2 * cs[jj].y;
                        s2[t] = x2 * cs[jj].x + x1 * cs[jj].y;
                    } else {
                        r2[t] = x1;
                        s2[t] = x2;
                    }
                }
                w1[j >> 1] = vcol ? pack_f16x2(r2[0], r2[1]) : pack_bf16x2(r2[0], r2[1]);
                w2[j >> 1] = vcol ? pack_f16x2(s2[0], s2[1]) : pack_bf16x2(s2[0], s2[1]);
            }
            stage_row32(box, r, 0, w1);
            stage_row32(box, r, 4, w2);
            os.commit(box, tmO, ep.out_col0 + n, row0, lane);
        }
    }
}

// F8: A and W are E4M3 (128-element k-blocks of 128 bytes, the same swizzled layout as 64
// bf16), the MMAs kind::f8f6f4 with K = 32, and the epilogue multiplies each column by
// ep.col_scale before its bias / RoPE.
template <int EPI, int BN, int EW, bool F8 = false>
__global__ void __launch_bounds__(64 + 32 * EW, 1)
    k_gemm_pc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmO, int K, int n_tiles, int nblk, EpiParams ep) {
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
    constexpr int KBW = F8 ? 128 : 64;  // elements per 128-byte k-block row
    const int KB = K / KBW;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&accf[0], 1);
        mbar_init(&accf[1], 1);
        mbar_init(&acce[0], EW);
        mbar_init(&acce[1], EW);
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmO);
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
                    tma_load_2d(sa, &tmA, &full[s], kb * KBW, m0);
                    tma_load_2d(sa + C::A_BYTES, &tmB, &full[s], kb * KBW, n0);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(BN) : idesc_bf16_f32(BN);
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
                    for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction: 16 bf16 or 32 E4M3
                        if constexpr (F8)
                            tc_mma_e4m3(dacc, sdesc_sw128(a_base + k * 32), sdesc_sw128(b_base + k * 32), idesc,
                                        (kb | k) != 0);
                        else
                            tc_mma_bf16(dacc, sdesc_sw128(a_base + k * 32), sdesc_sw128(b_base + k * 32), idesc,
                                        (kb | k) != 0);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(&accf[buf]);
            }
        }
    } else {
        const int q = warp & 3;           // TMEM lane quarter of this warp
        const int part = (warp - 2) >> 2;  // which share of the tile's columns (EW / 4 shares)
        OutStage<C::NBUF> os{smem + C::RING + ((warp - 2) & 3) * C::NBUF * C::OUT_BOX, 0u};
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
            const int m0 = (t / nblk) * 128, n0 = (t % nblk) * BN;
            const int row0 = m0 + q * 32;
            float2 cs[32];
            bool have_cs = false;
            if constexpr (EPI == EPI_QKV) {
                if (ep.rope && n0 < ep.rope_cols) {
                    const int row = row0 + lane;
                    // position-minor planes: consecutive rows (positions) of a warp read one contiguous span
                    const float4 *src = ep.rope + (row < ep.rows ? ep.pos[row] : 0);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float4 v = src[(size_t)i * MAX_POS];
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
            pc_epilogue_rows<EPI, BN, EW / 4, F8>(tacc, lane, row0, n0, ep, &tmO, os, lane, cs, have_cs, part);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[buf]);
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- persistent residual + LayerNorm GEMM
//
// x[rows, 384] += A . W^T (+ bias);  xn = LN(x) * g (+ b), one CTA per SM
// looping over 128-row tiles; the 384 accumulator columns stay in one TMEM
// buffer, so the overlap comes from the producer running ahead (the next
// tile's A / W stages load while this tile's epilogue streams the residual).
//   warp 0 lane 0  TMA producer: per 32-wide k-block, A box 128 x 32 and W as two 192 x 32
//                  boxes (64-byte swizzle) into a STAGES-deep ring; 32-wide k-blocks give
//                  twice the stages of 64-wide ones in the same memory, so more of the
//                  operand loads are in flight (the K = 1152 mainloop waited on them)
//   warp 1         TMEM allocation; lane 0 issues the N = 2 x 192 MMAs
//   warps 2..5     epilogue, one row per thread:
//     pass 1  per 32-column chunk: the residual chunk (128 x 32 FP32, 128-byte
//             swizzle) arrives by TMA (NXB buffers, prefetched across tiles,
//             so NXB - 1 chunk loads are in flight while one is processed);
//             v = x + acc (+ bias) is written back in place, stored to x by
//             TMA and parked in TMEM; row mean and M2 are merged chunk by
//             chunk (Chan's pairwise update), so one pass yields the moments;
//     pass 2  xn = LN(v) from TMEM, stored from registers with 32-byte stores
//             (the shared memory goes to the operand ring and the residual
//             buffers instead of output staging).
// The residual stream is the HBM traffic of this kernel.  Measured splits of the
// 224 KB between operand stages and residual buffers (32 KB / 16 KB each): five
// stages and four buffers beat 4 + 6, 3 + 8 and 6 + 2.
template <int STAGES_, int NXB_>
struct RlCfg {
    static constexpr int A_BYTES = 128 * 64;   // 128 rows x 32 bf16
    static constexpr int B_BYTES = 384 * 64;   // 384 rows x 32 bf16
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = STAGES_;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int XCH = 128 * 32 * 4;   // residual chunk: 128 rows x 32 FP32
    static constexpr int NXB = NXB_;
    static constexpr int DATA = RING + NXB * XCH;
    static constexpr int BAR_BYTES = (2 * STAGES + 2 + NXB) * 8 + 8;
    static constexpr int SMEM = DATA + BAR_BYTES + 1024;
    static_assert(NXB >= 2 && NXB <= 12 && SMEM <= 227 * 1024, "residual GEMM shared memory");
};
#ifndef JD_RL_STAGES
#define JD_RL_STAGES 5
#endif
#ifndef JD_RL_NXB
#define JD_RL_NXB 4
#endif
constexpr int RL_STAGES = JD_RL_STAGES, RL_NXB = JD_RL_NXB;
using RlCur = RlCfg<RL_STAGES, RL_NXB>;
// The persistent split kernel measured faster than k_gemm_rl for K = 1152 (Wo2: 20.7 against
// 21.6 ms per step at 1024 rows) and slower for K = 384 (Wo: 17.5 against 14.7 ms): with a short
// K the extra A reads of the second CTA outweigh the overlap.
#ifndef JD_RL_SPLIT_MIN_K
#define JD_RL_SPLIT_MIN_K 768
#endif
// CTAs per row tile of the split residual GEMM: six (64 columns each) when the grid fits the SMs,
// else three (128 columns each)
constexpr int RP_NS = 2;  // CTAs per row tile of the persistent split residual GEMM (192 columns each)

// OUT8: the LayerNorm output goes out as E4M3 bytes, y * ep.out8_inv_scale, rows of 384 bytes
// (the operand of the FP8 QKV GEMM).
template <int STAGES_, int NXB_, bool OUT8 = false>
__global__ void __launch_bounds__(192, 1)
    k_gemm_rl(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmXN, int K, int n_tiles,
              EpiParams ep) {
    using C = RlCfg<STAGES_, NXB_>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xbuf = smem + C::RING;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::DATA);
    uint64_t *empty = full + C::STAGES;
    uint64_t *accf = empty + C::STAGES;
    uint64_t *acce = accf + 1;
    uint64_t *xfull = acce + 1;  // [NXB]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(xfull + C::NXB);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KB = K / 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        mbar_init(acce, 4);
        for (int b = 0; b < C::NXB; ++b) mbar_init(&xfull[b], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmXN);
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
                const int m0 = t * 128;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES;
                    if (it >= (uint32_t)C::STAGES && !mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, ep.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + s * C::STAGE;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(sa, &tmA, &full[s], kb * 32, m0);
                    tma_load_2d(sa + C::A_BYTES, &tmB, &full[s], kb * 32, 0);
                    tma_load_2d(sa + C::A_BYTES + 192 * 64, &tmB, &full[s], kb * 32, 192);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(192);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
                if (tc >= 1 && !mbar_wait(acce, (tc - 1) & 1, ep.status)) break;
                tc_fence_after();
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES;
                    if (!mbar_wait(&full[s], (it / C::STAGES) & 1, ep.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * C::STAGE);
                    const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        tc_mma_bf16(tmem, sdesc_sw64(a_base + k * 32), sdesc_sw64(b_base + k * 32), idesc,
                                    (kb | k) != 0);
                        tc_mma_bf16(tmem + 192, sdesc_sw64(a_base + k * 32),
                                    sdesc_sw64(b_base + 192 * 64 + k * 32), idesc, (kb | k) != 0);
                    }
                    tc_commit(&empty[s]);
                }
                tc_commit(accf);
            }
        }
    } else {
        const int q = warp & 3;             // TMEM lane quarter
        const int r = q * 32 + lane;        // row inside the tile
        const bool leader = threadIdx.x == 64;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const int first = blockIdx.x;
        // residual chunk loads: chunk index g = (local tile) * 12 + c into buffer g % NXB
        if (leader && first < n_tiles) {
            for (int c = 0; c < C::NXB; ++c) {
                mbar_arrive_expect_tx(&xfull[c], C::XCH);
                tma_load_2d(xbuf + c * C::XCH, &tmX, &xfull[c], c * 32, first * 128);
            }
        }
        // every epilogue thread runs the same sequence of named barriers: a wait
        // that gives up does not leave the loop (later waits then return at once)
        uint32_t tc = 0;
        for (int t = first; t < n_tiles; t += gridDim.x, ++tc) {
            const int m0 = t * 128;
            mbar_wait(accf, tc & 1, ep.status);
            __syncwarp();
            tc_fence_after();
            float cnt = 0.f, mean = 0.f, m2 = 0.f;
            // ---- pass 1
#pragma unroll 1
            for (int c = 0; c < 12; ++c) {
                const uint32_t g = tc * 12 + c, b = g % C::NXB;
                uint32_t a[32];
                tmem_ld32(tl + c * 32, a);
                mbar_wait(&xfull[b], (g / C::NXB) & 1, ep.status);
                tmem_ld_wait();
                uint8_t *xb = xbuf + b * C::XCH;
                float v[32];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 x = *reinterpret_cast<const float4 *>(xb + r * 128 + ((j4 ^ (r & 7)) << 4));
                    float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (ep.bias) bb = reinterpret_cast<const float4 *>(ep.bias + c * 32)[j4];
                    v[4 * j4 + 0] = x.x + __uint_as_float(a[4 * j4 + 0]) + bb.x;
                    v[4 * j4 + 1] = x.y + __uint_as_float(a[4 * j4 + 1]) + bb.y;
                    v[4 * j4 + 2] = x.z + __uint_as_float(a[4 * j4 + 2]) + bb.z;
                    v[4 * j4 + 3] = x.w + __uint_as_float(a[4 * j4 + 3]) + bb.w;
                }
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) s += v[j];
                const float cm = s * (1.0f / 32.f);
                float cq = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) cq += (v[j] - cm) * (v[j] - cm);
                if (c == 0) {
                    mean = cm;
                    m2 = cq;
                    cnt = 32.f;
                } else {
                    const float tot = cnt + 32.f, dl = cm - mean;
                    mean += dl * (32.f / tot);
                    m2 += cq + dl * dl * (cnt * 32.f / tot);
                    cnt = tot;
                }
                uint32_t w[32];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    *reinterpret_cast<float4 *>(xb + r * 128 + ((j4 ^ (r & 7)) << 4)) =
                        make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[j]);
                tmem_st32(tl + c * 32, w);
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (leader) {
                    tma_store_2d(&tmX, xb, c * 32, m0);
                    bulk_commit();
                    // refill the previous chunk's buffer (its store has read it once at most
                    // this chunk's store is pending) with chunk g - 1 + NXB
                    if (g >= 1) {
                        const uint32_t h = g - 1 + C::NXB;
                        const int th = first + (int)(h / 12) * (int)gridDim.x;
                        if (th < n_tiles) {
                            const uint32_t bp = (g - 1) % C::NXB;
                            bulk_wait_read<1>();
                            mbar_arrive_expect_tx(&xfull[bp], C::XCH);
                            tma_load_2d(xbuf + bp * C::XCH, &tmX, &xfull[bp], (int)(h % 12) * 32, th * 128);
                        }
                    }
                }
            }
            tmem_st_wait();
            const float rstd = 1.0f / sqrtf(m2 * (1.0f / D) + ep.eps);
            // ---- pass 2: xn = LN(v) from TMEM, written straight from registers
            const int row = m0 + r;
            __nv_bfloat16 *xo = reinterpret_cast<__nv_bfloat16 *>(ep.out) + (size_t)row * ep.ldo;
            if constexpr (OUT8) {
                uint8_t *xo8 = reinterpret_cast<uint8_t *>(ep.out) + (size_t)row * ep.ldo;
#pragma unroll 1
                for (int j = 0; j < 6; ++j) {
                    uint32_t a[32], b2[32];
                    tmem_ld32(tl + j * 64, a);
                    tmem_ld32(tl + j * 64 + 32, b2);
                    tmem_ld_wait();
                    uint32_t w[16];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const int col = j * 64 + h * 32 + j4 * 4;
                            const float4 gg = *reinterpret_cast<const float4 *>(ep.ln_g + col);
                            const uint32_t *src = h ? b2 : a;
                            const float sc = rstd * ep.out8_inv_scale;
                            const float y0 = (__uint_as_float(src[4 * j4 + 0]) - mean) * sc * gg.x;
                            const float y1 = (__uint_as_float(src[4 * j4 + 1]) - mean) * sc * gg.y;
                            const float y2 = (__uint_as_float(src[4 * j4 + 2]) - mean) * sc * gg.z;
                            const float y3 = (__uint_as_float(src[4 * j4 + 3]) - mean) * sc * gg.w;
                            w[h * 8 + j4] = pack_e4m3x2(y0, y1) | (pack_e4m3x2(y2, y3) << 16);
                        }
                    }
                    if (row < ep.rows) {  // 64 bytes of the row: two 32-byte stores
                        uint8_t *dst = xo8 + j * 64;
                        st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                        st_global_v8(dst + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
                    }
                }
            } else {
#pragma unroll 1
            for (int j = 0; j < 6; ++j) {
                uint32_t a[32], b2[32];
                tmem_ld32(tl + j * 64, a);
                tmem_ld32(tl + j * 64 + 32, b2);
                tmem_ld_wait();
                uint32_t w[32];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const int col = j * 64 + h * 32 + j4 * 4;
                        const float4 gg = *reinterpret_cast<const float4 *>(ep.ln_g + col);
                        float4 be = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (ep.ln_b) be = *reinterpret_cast<const float4 *>(ep.ln_b + col);
                        const uint32_t *src = h ? b2 : a;
                        const float y0 = (__uint_as_float(src[4 * j4 + 0]) - mean) * rstd * gg.x + be.x;
                        const float y1 = (__uint_as_float(src[4 * j4 + 1]) - mean) * rstd * gg.y + be.y;
                        const float y2 = (__uint_as_float(src[4 * j4 + 2]) - mean) * rstd * gg.z + be.z;
                        const float y3 = (__uint_as_float(src[4 * j4 + 3]) - mean) * rstd * gg.w + be.w;
                        w[h * 16 + 2 * j4] = pack_bf16x2(y0, y1);
                        w[h * 16 + 2 * j4 + 1] = pack_bf16x2(y2, y3);
                    }
                }
                if (row < ep.rows) {  // 32-byte stores: a warp instruction fills whole sectors
                    uint8_t *dst = reinterpret_cast<uint8_t *>(xo + j * 64);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        st_global_v8(dst + 32 * cc, w[8 * cc], w[8 * cc + 1], w[8 * cc + 2], w[8 * cc + 3], w[8 * cc + 4],
                                     w[8 * cc + 5], w[8 * cc + 6], w[8 * cc + 7]);
                }
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce);
        }
        if (leader) bulk_wait_all();
        __syncwarp();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait with cluster-scope acquire (the arrivals come from the other CTAs of the cluster).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, unsigned *status) {
    const uint32_t addr = smem_u32(bar);
    uint64_t t0 = 0;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(addr, parity)) return true;
        if ((it & 255u) == 0) {
            if (status && (*reinterpret_cast<volatile unsigned *>(status) & ST_WAIT_TIMEOUT)) return false;
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > 2000000000ull) {
                if (status) atomicOr(status, ST_WAIT_TIMEOUT);
                return false;
            }
        }
    }
}
// Arrive on the barrier at the address of `local_bar` in CTA `rank` of this cluster.
__device__ __forceinline__ void mbar_arrive_remote(const uint64_t *local_bar, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local_bar)), "r"(rank));
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

// ---------------------------------------------------------------- residual + LayerNorm GEMM, split over a cluster
//
// For batches of a few row tiles (a single request of some hundred tokens makes
// seven), the persistent residual GEMM keeps one SM per tile busy: each loads
// the whole weight (884 KB for Wo2) and streams the tile's whole residual.  Here
// a cluster of NS CTAs shares a 128-row tile: CTA r computes the NC = 384 / NS
// output columns [NC r, NC r + NC) (an N = NC accumulator, the weight rows of
// its columns only), adds the residual of its columns, stores them, and sends
// each row's mean and M2 over its columns to every CTA of the cluster through
// distributed shared memory; after a cluster barrier each CTA merges the NS
// partial moments in rank order (equal counts: the mean of the means, M2 plus
// the spread of the means) and writes the LayerNorm output of its columns.
//   warp 0 lane 0  TMA producer: A box 128 x 64 and NC / 64 W boxes of 64 x 64 (128-byte swizzle)
//                  per stage
//   warp 1         TMEM allocation; lane 0 issues the N = NC MMAs
//   warps 2..5     epilogue, one row per thread; the NC / 32 residual chunks (FP32,
//                  128 x 32) are loaded by TMA at the start, under the mainloop
template <int NS>
struct RsCfg {
    static constexpr int NC = D / NS;            // output columns per CTA
    static constexpr int A_BYTES = 128 * 128;    // 128 rows x 64 bf16
    static constexpr int B_BYTES = NC * 128;     // NC rows x 64 bf16
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = NS >= 6 ? 6 : 4;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int NWL = NC / 64;          // W boxes of 64 rows per stage
    static constexpr int XCH = 128 * 32 * 4;     // residual chunk: 128 rows x 32 FP32
    static constexpr int NX = NC / 32;
    static constexpr int MOM = 12 * 128 * 8;     // (mean, M2) of every row's twelve 32-column chunks
    static constexpr int DATA = RING + NX * XCH + MOM;
    static constexpr int BAR_BYTES = (2 * STAGES + 2 + NX) * 8 + 8;
    static constexpr int SMEM = DATA + BAR_BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = NC <= 64 ? 64 : (NC <= 128 ? 128 : 256);
    static_assert(NC % 64 == 0 && NC <= 256, "column share: whole 64-row W boxes");
    static_assert(SMEM <= 227 * 1024, "split residual GEMM shared memory");
};

__device__ __forceinline__ uint32_t rs_cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void rs_cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int NS, bool OUT8>
__global__ void __cluster_dims__(NS, 1, 1) __launch_bounds__(192, 1)
    k_gemm_rls(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmX, int K, EpiParams ep) {
    using C = RsCfg<NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xbuf = smem + C::RING;
    float2 *mom = reinterpret_cast<float2 *>(smem + C::RING + C::NX * C::XCH);  // [12 chunks][128 rows]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::DATA);
    uint64_t *empty = full + C::STAGES;
    uint64_t *accf = empty + C::STAGES;
    uint64_t *xfull = accf + 1;  // [NX]
    uint64_t *momf = xfull + C::NX;  // every CTA's moments of this CTA's rows have arrived
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(momf + 1);

    const uint32_t rank = rs_cluster_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = (int)(blockIdx.x / NS) * 128;
    const int c0 = (int)rank * C::NC;
    const int KB = K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        for (int c = 0; c < C::NX; ++c) mbar_init(&xfull[c], 1);
        mbar_init(momf, 1);  // one arrival with the expected moment bytes
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    rs_cluster_sync();  // every CTA's moment barrier exists before the first remote store
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool leader = threadIdx.x == 64;

    if (warp == 0) {
        if (lane == 0) {
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % C::STAGES;
                if (kb >= C::STAGES && !mbar_wait(&empty[s], ((kb / C::STAGES) - 1) & 1, ep.status)) break;
                uint8_t *sa = smem + s * C::STAGE;
                mbar_arrive_expect_tx(&full[s], C::STAGE);
                tma_load_2d(sa, &tmA, &full[s], kb * 64, m0);
#pragma unroll
                for (int w = 0; w < C::NWL; ++w)
                    tma_load_2d(sa + C::A_BYTES + w * 64 * 128, &tmB, &full[s], kb * 64, c0 + 64 * w);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(C::NC);
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % C::STAGES;
                if (!mbar_wait(&full[s], (kb / C::STAGES) & 1, ep.status)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + s * C::STAGE);
                const uint32_t b_base = a_base + C::A_BYTES;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    tc_mma_bf16(tmem, sdesc_sw128(a_base + k * 32), sdesc_sw128(b_base + k * 32), idesc, (kb | k) != 0);
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
        }
    } else if (leader) {  // the residual of this CTA's columns, under the mainloop
        for (int c = 0; c < C::NX; ++c) {
            mbar_arrive_expect_tx(&xfull[c], C::XCH);
            tma_load_2d(xbuf + c * C::XCH, &tmX, &xfull[c], c0 + c * 32, m0);
        }
    }

    const int q = warp & 3;
    const int r = q * 32 + lane;  // row inside the tile (epilogue warps)
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    float mean = 0.f, m2 = 0.f;
    if (warp >= 2) {
        if (leader) mbar_arrive_expect_tx(momf, NS * C::NX * 128 * 8);
        mbar_wait(accf, 0, ep.status);
        __syncwarp();
        tc_fence_after();
        // ---- pass 1: v = x + acc (+ bias) for this CTA's columns; each 32-column chunk's
        //      (mean, M2) goes to slot [global chunk][row] of every CTA of the cluster
#pragma unroll 1
        for (int c = 0; c < C::NX; ++c) {
            uint32_t a[32];
            tmem_ld32(tl + c * 32, a);
            mbar_wait(&xfull[c], 0, ep.status);
            tmem_ld_wait();
            uint8_t *xb = xbuf + c * C::XCH;
            float v[32];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                const float4 x = *reinterpret_cast<const float4 *>(xb + r * 128 + ((j4 ^ (r & 7)) << 4));
                float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ep.bias) bb = reinterpret_cast<const float4 *>(ep.bias + c0 + c * 32)[j4];
                v[4 * j4 + 0] = x.x + __uint_as_float(a[4 * j4 + 0]) + bb.x;
                v[4 * j4 + 1] = x.y + __uint_as_float(a[4 * j4 + 1]) + bb.y;
                v[4 * j4 + 2] = x.z + __uint_as_float(a[4 * j4 + 2]) + bb.z;
                v[4 * j4 + 3] = x.w + __uint_as_float(a[4 * j4 + 3]) + bb.w;
            }
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) s += v[j];
            const float cm = s * (1.0f / 32.f);
            float cq = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) cq += (v[j] - cm) * (v[j] - cm);
            {
                // asynchronous stores that complete their bytes on each receiving CTA's moment barrier
                const uint32_t local = smem_u32(&mom[((int)rank * C::NX + c) * 128 + r]);
                const uint32_t lbar = smem_u32(momf);
#pragma unroll
                for (int j = 0; j < NS; ++j) {
                    uint32_t remote, rbar;
                    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(j));
                    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(lbar), "r"(j));
                    asm volatile(
                        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(remote),
                        "f"(cm), "f"(cq), "r"(rbar)
                        : "memory");
                }
            }
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4)
                *reinterpret_cast<float4 *>(xb + r * 128 + ((j4 ^ (r & 7)) << 4)) =
                    make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
            uint32_t w[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[j]);
            tmem_st32(tl + c * 32, w);
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (leader) {
                tma_store_2d(&tmX, xb, c0 + c * 32, m0);
                bulk_commit();
            }
        }
        tmem_st_wait();
        // every CTA's moments of these rows; a CTA leaves only after all stores into it landed
        mbar_wait_cluster(momf, 0, ep.status);
    }
    if (warp >= 2) {
        // ---- the twelve chunks' moments merged in column order with k_gemm_rl's update, so the
        //      row's mean and M2 -- and the outputs -- are bit-identical to the unsplit kernel's
        float cnt = 0.f;
#pragma unroll 1
        for (int c = 0; c < 12; ++c) {
            const float2 p = mom[c * 128 + r];
            if (c == 0) {
                mean = p.x;
                m2 = p.y;
                cnt = 32.f;
            } else {
                const float tot = cnt + 32.f, dl = p.x - mean;
                mean += dl * (32.f / tot);
                m2 += p.y + dl * dl * (cnt * 32.f / tot);
                cnt = tot;
            }
        }
        const float mu = mean;
        const float rstd = 1.0f / sqrtf(m2 * (1.0f / D) + ep.eps);
        // ---- pass 2: LayerNorm of this CTA's columns from TMEM, stored from registers
        const int row = m0 + r;
#pragma unroll 1
        for (int c = 0; c < C::NX; ++c) {
            uint32_t a[32];
            tmem_ld32(tl + c * 32, a);
            tmem_ld_wait();
            const int col0 = c0 + c * 32;
            uint32_t w[16];
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
                const int col = col0 + j4 * 4;
                const float4 gg = *reinterpret_cast<const float4 *>(ep.ln_g + col);
                float4 be = make_float4(0.f, 0.f, 0.f, 0.f);
                if (!OUT8 && ep.ln_b) be = *reinterpret_cast<const float4 *>(ep.ln_b + col);
                const float sc = OUT8 ? rstd * ep.out8_inv_scale : rstd;
                const float y0 = (__uint_as_float(a[4 * j4 + 0]) - mu) * sc * gg.x + be.x;
                const float y1 = (__uint_as_float(a[4 * j4 + 1]) - mu) * sc * gg.y + be.y;
                const float y2 = (__uint_as_float(a[4 * j4 + 2]) - mu) * sc * gg.z + be.z;
                const float y3 = (__uint_as_float(a[4 * j4 + 3]) - mu) * sc * gg.w + be.w;
                if (OUT8) {
                    if (j4 < 8) w[j4] = pack_e4m3x2(y0, y1) | (pack_e4m3x2(y2, y3) << 16);
                } else {
                    w[2 * j4] = pack_bf16x2(y0, y1);
                    w[2 * j4 + 1] = pack_bf16x2(y2, y3);
                }
            }
            if (row < ep.rows) {
                if (OUT8) {
                    uint8_t *dst = reinterpret_cast<uint8_t *>(ep.out) + (size_t)row * ep.ldo + col0;
                    st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                } else {
                    uint8_t *dst = reinterpret_cast<uint8_t *>(reinterpret_cast<__nv_bfloat16 *>(ep.out) +
                                                               (size_t)row * ep.ldo + col0);
                    st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                    st_global_v8(dst + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
                }
            }
        }
        if (leader) bulk_wait_all();
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- persistent residual + LayerNorm GEMM split over a cluster
//
// The same product as k_gemm_rl for batches of many row tiles, with the 384 output
// columns of every tile split over a cluster of NS = 2 CTAs (CTA r: columns [192 r,
// 192 r + 192)).  With 192 columns per CTA, two accumulators fit in TMEM, so the
// epilogue of one tile overlaps the MMAs of the next (with 384 columns per CTA the next
// tile's MMAs wait for the whole epilogue).  The clusters walk the row tiles (cluster c:
// tiles c, c + C, ...); the two CTAs of a cluster take the same tiles.  Per tile each CTA
// sends its rows' (mean, M2) over its columns into both CTAs' shared memory (slots
// double-buffered by tile parity; every epilogue thread arrives on both CTAs' moment
// barriers after its stores); a CTA merges the two halves in rank order once all have
// arrived.  A slot is rewritten two tiles later only after the other CTA has sent the
// next tile's moments, which it does after merging this one.
//   warp 0 lane 0  TMA producer: A box 128 x 64 and W box 192 x 64 (128-byte swizzle)
//   warp 1         TMEM allocation (two accumulators); lane 0 issues the N = 192 MMAs
//   warps 2..5     epilogue, one row per thread: residual chunks (128 x 32 FP32) through a
//                  ring of NXB buffers refilled across tiles, as in k_gemm_rl
template <int NS>
struct RpCfg {
    static constexpr int NC = D / NS;              // output columns per CTA
    static constexpr int A_BYTES = 128 * 128;      // 128 rows x 64 bf16
    static constexpr int B_BYTES = NC * 128;       // NC rows x 64 bf16
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = 3;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int XCH = 128 * 32 * 4;       // residual chunk: 128 rows x 32 FP32
    static constexpr int NX = NC / 32;             // residual chunks per tile
    static constexpr int NXB = 4;                  // residual buffers
    static constexpr int MOM = 2 * 12 * 128 * 8;   // (mean, M2): [tile parity][32-column chunk][row]
    static constexpr int DATA = RING + NXB * XCH + MOM;
    static constexpr int NBAR = 2 * STAGES + 2 + 2 + NXB + 2;
    static constexpr int SMEM = DATA + NBAR * 8 + 8 + 1024;
    static constexpr uint32_t ACC_STRIDE = 256;    // TMEM columns between the two accumulators
    static_assert(NC % 32 == 0 && NC <= 256 && SMEM <= 227 * 1024, "persistent split residual GEMM");
};

template <int NS, bool OUT8>
__global__ void __cluster_dims__(NS, 1, 1) __launch_bounds__(192, 1)
    k_gemm_rlp(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmX, int K, int n_tiles, EpiParams ep) {
    using C = RpCfg<NS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xbuf = smem + C::RING;
    float2 *mom = reinterpret_cast<float2 *>(smem + C::RING + C::NXB * C::XCH);  // [2][12][128]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::DATA);
    uint64_t *empty = full + C::STAGES;
    uint64_t *accf = empty + C::STAGES;  // [2]
    uint64_t *acce = accf + 2;           // [2]
    uint64_t *xfull = acce + 2;          // [NXB]
    uint64_t *momf = xfull + C::NXB;     // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(momf + 2);

    const uint32_t rank = rs_cluster_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cid = (int)(blockIdx.x / NS), ncl = (int)(gridDim.x / NS);
    const int c0 = (int)rank * C::NC;
    const int KB = K / 64;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 4);
            mbar_init(&momf[b], 1);  // the leader's arrival with the tile's expected moment bytes
        }
        for (int b = 0; b < C::NXB; ++b) mbar_init(&xfull[b], 1);
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    rs_cluster_sync();  // both CTAs' barriers exist before the first remote arrival
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int t = cid; t < n_tiles && ok; t += ncl) {
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const uint32_t s = it % C::STAGES;
                    if (it >= (uint32_t)C::STAGES && !mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1, ep.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + s * C::STAGE;
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    tma_load_2d(sa, &tmA, &full[s], kb * 64, t * 128);
                    tma_load_2d(sa + C::A_BYTES, &tmB, &full[s], kb * 64, c0);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(C::NC);
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int t = cid; t < n_tiles && ok; t += ncl, ++tc) {
                const uint32_t b = tc & 1;
                if (tc >= 2 && !mbar_wait(&acce[b], ((tc >> 1) - 1) & 1, ep.status)) break;
                tc_fence_after();
                const uint32_t dacc = tmem + b * C::ACC_STRIDE;
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
                tc_commit(&accf[b]);
            }
        }
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const bool leader = threadIdx.x == 64;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        // residual chunk g (local tile g / NX, chunk g % NX) goes into buffer g % NXB
        if (leader && cid < n_tiles) {
            for (int g = 0; g < C::NXB; ++g) {
                const int th = cid + (g / C::NX) * ncl;
                if (th >= n_tiles) break;
                mbar_arrive_expect_tx(&xfull[g], C::XCH);
                tma_load_2d(xbuf + g * C::XCH, &tmX, &xfull[g], c0 + (g % C::NX) * 32, th * 128);
            }
        }
        uint32_t tc = 0;
        for (int t = cid; t < n_tiles; t += ncl, ++tc) {
            const int m0 = t * 128;
            const uint32_t b = tc & 1;
            const uint32_t tacc = tl + b * C::ACC_STRIDE;
            mbar_wait(&accf[b], (tc >> 1) & 1, ep.status);
            __syncwarp();
            tc_fence_after();
            // the moments of this tile arrive as NS x NX x 128 asynchronous 8-byte stores
            if (leader) mbar_arrive_expect_tx(&momf[b], NS * C::NX * 128 * 8);
            // ---- pass 1: v = x + acc (+ bias) for this CTA's columns; each 32-column chunk's
            //      (mean, M2) goes to slot [tile parity][global chunk][row] of both CTAs
#pragma unroll 1
            for (int c = 0; c < C::NX; ++c) {
                const uint32_t g = tc * C::NX + c, xb_i = g % C::NXB;
                uint32_t a[32];
                tmem_ld32(tacc + c * 32, a);
                mbar_wait(&xfull[xb_i], (g / C::NXB) & 1, ep.status);
                tmem_ld_wait();
                uint8_t *xb = xbuf + xb_i * C::XCH;
                float v[32];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 x = *reinterpret_cast<const float4 *>(xb + r * 128 + ((j4 ^ (r & 7)) << 4));
                    float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (ep.bias) bb = reinterpret_cast<const float4 *>(ep.bias + c0 + c * 32)[j4];
                    v[4 * j4 + 0] = x.x + __uint_as_float(a[4 * j4 + 0]) + bb.x;
                    v[4 * j4 + 1] = x.y + __uint_as_float(a[4 * j4 + 1]) + bb.y;
                    v[4 * j4 + 2] = x.z + __uint_as_float(a[4 * j4 + 2]) + bb.z;
                    v[4 * j4 + 3] = x.w + __uint_as_float(a[4 * j4 + 3]) + bb.w;
                }
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) s += v[j];
                const float cm = s * (1.0f / 32.f);
                float cq = 0.f;
#pragma unroll
                for (int j = 0; j < 32; ++j) cq += (v[j] - cm) * (v[j] - cm);
                {
                    // asynchronous stores that complete their bytes on the receiving CTA's moment
                    // barrier: no release of this thread's other (global) stores is waited for
                    const uint32_t local = smem_u32(&mom[((int)b * 12 + (int)rank * C::NX + c) * 128 + r]);
                    const uint32_t lbar = smem_u32(&momf[b]);
#pragma unroll
                    for (int j = 0; j < NS; ++j) {
                        uint32_t remote, rbar;
                        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(j));
                        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(lbar), "r"(j));
                        asm volatile(
                            "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
                                remote),
                            "f"(cm), "f"(cq), "r"(rbar)
                            : "memory");
                    }
                }
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4)
                    *reinterpret_cast<float4 *>(xb + r * 128 + ((j4 ^ (r & 7)) << 4)) =
                        make_float4(v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2], v[4 * j4 + 3]);
                uint32_t w[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[j]);
                tmem_st32(tacc + c * 32, w);
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (leader) {
                    tma_store_2d(&tmX, xb, c0 + c * 32, m0);
                    bulk_commit();
                    // refill the previous chunk's buffer (its store has read it once at most this
                    // chunk's store is pending) with chunk g - 1 + NXB
                    if (g >= 1) {
                        const uint32_t h = g - 1 + C::NXB;
                        const int th = cid + (int)(h / C::NX) * ncl;
                        if (th < n_tiles) {
                            const uint32_t bp = (g - 1) % C::NXB;
                            bulk_wait_read<1>();
                            mbar_arrive_expect_tx(&xfull[bp], C::XCH);
                            tma_load_2d(xbuf + bp * C::XCH, &tmX, &xfull[bp], c0 + (int)(h % C::NX) * 32, th * 128);
                        }
                    }
                }
            }
            tmem_st_wait();
            mbar_wait_cluster(&momf[b], (tc >> 1) & 1, ep.status);
            // ---- the twelve chunks' moments merged in column order with k_gemm_rl's update, so the
            //      row's mean and M2 -- and the outputs -- are bit-identical to the unsplit kernel's
            float cnt = 0.f, mean = 0.f, m2 = 0.f;
#pragma unroll 1
            for (int c = 0; c < 12; ++c) {
                const float2 p = mom[((int)b * 12 + c) * 128 + r];
                if (c == 0) {
                    mean = p.x;
                    m2 = p.y;
                    cnt = 32.f;
                } else {
                    const float tot = cnt + 32.f, dl = p.x - mean;
                    mean += dl * (32.f / tot);
                    m2 += p.y + dl * dl * (cnt * 32.f / tot);
                    cnt = tot;
                }
            }
            const float mu = mean;
            const float rstd = 1.0f / sqrtf(m2 * (1.0f / D) + ep.eps);
            // ---- pass 2: LayerNorm of this CTA's columns from TMEM
            const int row = m0 + r;
#pragma unroll 1
            for (int c = 0; c < C::NX; ++c) {
                uint32_t a[32];
                tmem_ld32(tacc + c * 32, a);
                tmem_ld_wait();
                const int col0 = c0 + c * 32;
                uint32_t w[16];
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const int col = col0 + j4 * 4;
                    const float4 gg = *reinterpret_cast<const float4 *>(ep.ln_g + col);
                    float4 be = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (!OUT8 && ep.ln_b) be = *reinterpret_cast<const float4 *>(ep.ln_b + col);
                    const float sc = OUT8 ? rstd * ep.out8_inv_scale : rstd;
                    const float y0 = (__uint_as_float(a[4 * j4 + 0]) - mu) * sc * gg.x + be.x;
                    const float y1 = (__uint_as_float(a[4 * j4 + 1]) - mu) * sc * gg.y + be.y;
                    const float y2 = (__uint_as_float(a[4 * j4 + 2]) - mu) * sc * gg.z + be.z;
                    const float y3 = (__uint_as_float(a[4 * j4 + 3]) - mu) * sc * gg.w + be.w;
                    if (OUT8) {
                        w[j4] = pack_e4m3x2(y0, y1) | (pack_e4m3x2(y2, y3) << 16);
                    } else {
                        w[2 * j4] = pack_bf16x2(y0, y1);
                        w[2 * j4 + 1] = pack_bf16x2(y2, y3);
                    }
                }
                if (row < ep.rows) {
                    if (OUT8) {
                        uint8_t *dst = reinterpret_cast<uint8_t *>(ep.out) + (size_t)row * ep.ldo + col0;
                        st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                    } else {
                        uint8_t *dst = reinterpret_cast<uint8_t *>(reinterpret_cast<__nv_bfloat16 *>(ep.out) +
                                                                   (size_t)row * ep.ldo + col0);
                        st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
                        st_global_v8(dst + 32, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[b]);
        }
        if (leader) bulk_wait_all();
        __syncwarp();
    }
    __syncwarp();
    rs_cluster_sync();  // no CTA leaves while the other may still write into it
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
int num_sms() { return g_num_sms; }

cudaError_t gemm_init_attributes() {
    cudaError_t e;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rl<RL_STAGES, RL_NXB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RlCur::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rl<RL_STAGES, RL_NXB, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RlCur::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rlp<RP_NS, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RpCfg<RP_NS>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rlp<RP_NS, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RpCfg<RP_NS>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rls<3, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RsCfg<3>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rls<3, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RsCfg<3>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rls<6, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RsCfg<6>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_rls<6, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  RsCfg<6>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_QKV, 192, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<192>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_QKV, 192, 4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<192>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_QKV, 64, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<64>::SMEM)) != cudaSuccess)
        return e;

    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_GEGLU, 256, GEGLU_EW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  PcCfg<256>::SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_gemm_pc<EPI_BIAS_ACT, 256, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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

template <int EPI, int BN, bool F8 = false>
static cudaError_t launch_pc(const GemmOp &op, cudaStream_t st) {
    if (op.N % BN != 0 || (F8 && (op.K % 128 != 0 || !op.ep.col_scale))) return cudaErrorInvalidValue;
    const int nblk = op.N / BN;
    const int n_tiles = nblk * ((op.ep.rows + 127) / 128);
    const int grid = n_tiles < g_num_sms ? n_tiles : g_num_sms;
    if (!op.tmO) return cudaErrorInvalidValue;
    constexpr int EW = EPI == EPI_GEGLU ? GEGLU_EW : 4;  // epilogue warps
    k_gemm_pc<EPI, BN, EW, F8><<<grid, 64 + 32 * EW, PcCfg<BN>::SMEM, st>>>(*op.tmA, *op.tmB, *op.tmO, op.K,
                                                                             n_tiles, nblk, op.ep);
    return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmOp &op, bool fp32, cudaStream_t st) {
    if (op.ep.rows <= 0) return cudaSuccess;
    if (op.N % op.bn != 0 || op.K % 64 != 0) return cudaErrorInvalidValue;
    if (!fp32 && op.epi == EPI_RESID_LN && op.tmX && op.tmXN && op.tmA64 && op.tmB64 && op.ep.ln_g && !op.ep.fin_g &&
        op.N == D && op.K % 32 == 0) {
        const int n_tiles = (op.ep.rows + 127) / 128;
        const int grid = n_tiles < g_num_sms ? n_tiles : g_num_sms;
        if (op.tmA && op.tmBs && op.K % 64 == 0 && 3 * n_tiles <= g_num_sms) {
            // few row tiles: split each tile's columns over a cluster, so six or three SMs share it
            if (op.out8 && (op.ep.ln_b || op.ep.out8_inv_scale <= 0.f)) return cudaErrorInvalidValue;
            if (6 * n_tiles <= g_num_sms) {
                if (op.out8)
                    k_gemm_rls<6, true><<<6 * n_tiles, 192, RsCfg<6>::SMEM, st>>>(*op.tmA, *op.tmBs, *op.tmX, op.K, op.ep);
                else
                    k_gemm_rls<6, false><<<6 * n_tiles, 192, RsCfg<6>::SMEM, st>>>(*op.tmA, *op.tmBs, *op.tmX, op.K, op.ep);
            } else {
                if (op.out8)
                    k_gemm_rls<3, true><<<3 * n_tiles, 192, RsCfg<3>::SMEM, st>>>(*op.tmA, *op.tmBs, *op.tmX, op.K, op.ep);
                else
                    k_gemm_rls<3, false><<<3 * n_tiles, 192, RsCfg<3>::SMEM, st>>>(*op.tmA, *op.tmBs, *op.tmX, op.K, op.ep);
            }
            return cudaGetLastError();
        }
        if (op.tmA && op.tmBp && op.K % 64 == 0 && op.K >= JD_RL_SPLIT_MIN_K) {
            // many row tiles and a long K (Wo2, the head's second feed-forward GEMM): persistent,
            // the columns split over 2 CTAs so that one tile's epilogue overlaps the next one's MMAs
            if (op.out8 && (op.ep.ln_b || op.ep.out8_inv_scale <= 0.f)) return cudaErrorInvalidValue;
            const int ncl = std::min(n_tiles, g_num_sms / RP_NS);
            if (op.out8)
                k_gemm_rlp<RP_NS, true><<<RP_NS * ncl, 192, RpCfg<RP_NS>::SMEM, st>>>(*op.tmA, *op.tmBp, *op.tmX, op.K,
                                                                                       n_tiles, op.ep);
            else
                k_gemm_rlp<RP_NS, false><<<RP_NS * ncl, 192, RpCfg<RP_NS>::SMEM, st>>>(*op.tmA, *op.tmBp, *op.tmX, op.K,
                                                                                        n_tiles, op.ep);
            return cudaGetLastError();
        }
        if (op.out8) {
            if (op.ep.ln_b || op.ep.out8_inv_scale <= 0.f) return cudaErrorInvalidValue;
            k_gemm_rl<RL_STAGES, RL_NXB, true><<<grid, 192, RlCur::SMEM, st>>>(*op.tmA64, *op.tmB64, *op.tmX,
                                                                               *op.tmXN, op.K, n_tiles, op.ep);
        } else {
            k_gemm_rl<RL_STAGES, RL_NXB><<<grid, 192, RlCur::SMEM, st>>>(*op.tmA64, *op.tmB64, *op.tmX, *op.tmXN,
                                                                         op.K, n_tiles, op.ep);
        }
        return cudaGetLastError();
    }
    if (op.out8 || (op.f8 && (fp32 || op.epi != EPI_QKV))) return cudaErrorInvalidValue;
    if (!fp32) {  // persistent tcgen05 kernels for the column-split epilogues
        if (op.epi == EPI_QKV) {
            if (op.f8) return launch_pc<EPI_QKV, 192, true>(op, st);
            // few row tiles: one 64-column head per tile, so up to three times as many SMs share the product
            const int row_tiles = (op.ep.rows + 127) / 128;
            if (op.tmBs && op.N % 64 == 0 && row_tiles * (op.N / 64) <= g_num_sms) {
                GemmOp o = op;
                o.tmB = op.tmBs;
                return launch_pc<EPI_QKV, 64>(o, st);
            }
            return launch_pc<EPI_QKV, 192>(op, st);
        }
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
