// Fused GEMM epilogues, applied one output row at a time by one warp.
//
// A GEMM tile (128 rows x BN columns of FP32 accumulators) is first staged
// row-major in shared memory; each warp then takes whole rows so that every
// global load and store of the epilogue is coalesced and a LayerNorm over the
// full 384-wide row can be computed in registers with warp reductions.
//
//  EPI_QKV      q|k|v projection (+ bias); rotary embedding on the q and k
//               columns ("julia1 -- Rust runtime", "Why it is faster": RoPE
//               applied on load; here in the producing GEMM instead).
//  EPI_RESID_LN residual add into the FP32 stream x (+ bias), then optionally
//               (a) the final encoder norm + type-table row ("The decision
//               head", step 1) and (b) the next pre-norm LayerNorm, written as
//               the next GEMM's operand ("Why it is faster": residual adds
//               fused into the following LayerNorm).
//  EPI_GEGLU    y = GELU(u) * g from interleaved [u | g] column blocks
//               ("Why it is faster": the [T, 2304] intermediate is never
//               materialised).
//  EPI_BIAS_ACT y = act(acc + bias), ReLU or GELU (head feed-forward).
#pragma once

#include "common.cuh"

namespace jd {

enum EpiKind { EPI_QKV = 0, EPI_RESID_LN = 1, EPI_GEGLU = 2, EPI_BIAS_ACT = 3 };

struct EpiParams {
    int rows;                // valid output rows
    void *out;               // [rows, ldo] of OutT (unused by a RESID_LN without ln_g)
    int ldo;
    const float *bias;       // [N] by weight row, or null
    const float4 *rope;      // [16][MAX_POS]: plane k holds (cos, sin) of pairs 2k, 2k + 1 per position, or null
    int out_col0;            // column offset of this launch's output inside the tensor map (BF16 path)
    const int *pos;          // [rows] position within the request row
    int rope_cols;           // output columns [0, rope_cols) are rotated
    float *resid;            // [rows, 384] FP32 residual stream (RESID_LN)
    const float *ln_g;       // LayerNorm after the add (null: none)
    const float *ln_b;       // its bias (null: none)
    const float *fin_g;      // final encoder norm gain (null: none)
    const float *type_tab;   // [3, 384]
    const int *tok_row;      // [rows] request row of each token
    const int *row_type;     // [B]
    float *tap;              // optional [rows, 384] copy of the final-norm output
    int act;                 // 0 ReLU, 1 GELU
    float eps;
    unsigned *status;
    const float *col_scale;  // FP8 QKV GEMM: [N] per output column, activation scale x weight row scale
    float out8_inv_scale;    // FP8 LayerNorm output of the residual GEMM: E4M3(y * out8_inv_scale) into out
};

// LayerNorm of the 384 values held 12 per lane (columns j*128 + lane*4 + e).
__device__ __forceinline__ void ln_regs(float (&v)[12], const float *g, const float *b, int lane, float eps) {
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 12; ++e) s += v[e];
    const float mean = warp_sum(s) * (1.0f / D);
    float q = 0.f;
#pragma unroll
    for (int e = 0; e < 12; ++e) {
        v[e] -= mean;
        q += v[e] * v[e];
    }
    const float rstd = 1.0f / sqrtf(warp_sum(q) * (1.0f / D) + eps);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int c = j * 128 + lane * 4;
        const float4 gg = *reinterpret_cast<const float4 *>(g + c);
        float4 bb = make_float4(0.f, 0.f, 0.f, 0.f);
        if (b) bb = *reinterpret_cast<const float4 *>(b + c);
        v[4 * j + 0] = v[4 * j + 0] * rstd * gg.x + bb.x;
        v[4 * j + 1] = v[4 * j + 1] * rstd * gg.y + bb.y;
        v[4 * j + 2] = v[4 * j + 2] * rstd * gg.z + bb.z;
        v[4 * j + 3] = v[4 * j + 3] * rstd * gg.w + bb.w;
    }
}

// Second half of the residual epilogue for one row whose sum v = x + acc (+ bias) is in registers.
template <typename OutT>
__device__ __forceinline__ void epi_resid_ln_finish(float (&v)[12], int row, const EpiParams &ep, int lane);

template <typename OutT>
__device__ __forceinline__ void epi_resid_ln_row(const float *acc, int row, const EpiParams &ep, int lane) {
    float v[12];
    float *xr = ep.resid + (size_t)row * D;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int c = j * 128 + lane * 4;
        const float4 a = *reinterpret_cast<const float4 *>(acc + c);
        const float4 x = *reinterpret_cast<const float4 *>(xr + c);
        float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ep.bias) b = *reinterpret_cast<const float4 *>(ep.bias + c);
        v[4 * j + 0] = x.x + a.x + b.x;
        v[4 * j + 1] = x.y + a.y + b.y;
        v[4 * j + 2] = x.z + a.z + b.z;
        v[4 * j + 3] = x.w + a.w + b.w;
    }
    epi_resid_ln_finish<OutT>(v, row, ep, lane);
}

// R rows (row0 + u * rstep, u < n) per warp with every global load issued
// before the first use, so that a warp keeps R residual rows in flight.
template <typename OutT, int R>
__device__ __forceinline__ void epi_resid_ln_rows(const float *acc0, int pitch, int row0, int rstep, int n,
                                                  const EpiParams &ep, int lane) {
    float v[R][12];
    float4 b[3];
#pragma unroll
    for (int j = 0; j < 3; ++j)
        b[j] = ep.bias ? *reinterpret_cast<const float4 *>(ep.bias + j * 128 + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < R; ++u) {
        if (u < n) {
            const float *xr = ep.resid + (size_t)(row0 + u * rstep) * D;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const float4 x = *reinterpret_cast<const float4 *>(xr + j * 128 + lane * 4);
                v[u][4 * j + 0] = x.x; v[u][4 * j + 1] = x.y; v[u][4 * j + 2] = x.z; v[u][4 * j + 3] = x.w;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < R; ++u) {
        if (u < n) {
            const float *acc = acc0 + (size_t)u * rstep * pitch;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const float4 a = *reinterpret_cast<const float4 *>(acc + j * 128 + lane * 4);
                v[u][4 * j + 0] += a.x + b[j].x;
                v[u][4 * j + 1] += a.y + b[j].y;
                v[u][4 * j + 2] += a.z + b[j].z;
                v[u][4 * j + 3] += a.w + b[j].w;
            }
            epi_resid_ln_finish<OutT>(v[u], row0 + u * rstep, ep, lane);
        }
    }
}

template <typename OutT>
__device__ __forceinline__ void epi_resid_ln_finish(float (&v)[12], int row, const EpiParams &ep, int lane) {
    float *xr = ep.resid + (size_t)row * D;
    if (ep.fin_g) {
        ln_regs(v, ep.fin_g, nullptr, lane, ep.eps);
        const int t = ep.row_type[ep.tok_row[row]];
        const float *tt = ep.type_tab + t * D;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int c = j * 128 + lane * 4;
            if (ep.tap)
                *reinterpret_cast<float4 *>(ep.tap + (size_t)row * D + c) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            const float4 ty = *reinterpret_cast<const float4 *>(tt + c);
            v[4 * j + 0] += ty.x;
            v[4 * j + 1] += ty.y;
            v[4 * j + 2] += ty.z;
            v[4 * j + 3] += ty.w;
        }
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int c = j * 128 + lane * 4;
        *reinterpret_cast<float4 *>(xr + c) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
    if (ep.ln_g) {
        ln_regs(v, ep.ln_g, ep.ln_b, lane, ep.eps);
        OutT *o = reinterpret_cast<OutT *>(ep.out) + (size_t)row * ep.ldo;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int c = j * 128 + lane * 4;
            store4<OutT>(o + c, v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
    }
}

// acc covers global output columns [n0, n0 + BN); BN a multiple of 128.
template <typename OutT, int BN>
__device__ __forceinline__ void epi_qkv_row(const float *acc, int row, int n0, const EpiParams &ep, int lane) {
    OutT *o = reinterpret_cast<OutT *>(ep.out) + (size_t)row * ep.ldo;
    const int i = (lane & 15) * 2;
    int pos = 0;
    if (ep.rope) pos = ep.pos[row];
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 128) {
        const int seg = c0 + (lane >> 4) * 64;
        float a0 = acc[seg + i], a1 = acc[seg + i + 1];
        float b0 = acc[seg + 32 + i], b1 = acc[seg + 33 + i];
        const int n = n0 + seg;
        if (ep.bias) {
            a0 += ep.bias[n + i];
            a1 += ep.bias[n + i + 1];
            b0 += ep.bias[n + 32 + i];
            b1 += ep.bias[n + 33 + i];
        }
        if (ep.rope && n < ep.rope_cols) {
            const float4 cs = ep.rope[(size_t)(i >> 1) * MAX_POS + pos];
            const float r0 = a0 * cs.x - b0 * cs.y, s0 = b0 * cs.x + a0 * cs.y;
            const float r1 = a1 * cs.z - b1 * cs.w, s1 = b1 * cs.z + a1 * cs.w;
            a0 = r0; b0 = s0; a1 = r1; b1 = s1;
        }
        store2<OutT>(o + n + i, a0, a1);
        store2<OutT>(o + n + 32 + i, b0, b1);
    }
}

// Interleaved GEGLU tile: acc columns [0, G) are u, [G, 2G) the matching gate
// columns; output columns [n0 / 2, n0 / 2 + G).
template <typename OutT, int BN>
__device__ __forceinline__ void epi_geglu_row(const float *acc, int row, int n0, const EpiParams &ep, int lane) {
    constexpr int G = BN / 2;
    OutT *o = reinterpret_cast<OutT *>(ep.out) + (size_t)row * ep.ldo + n0 / 2;
#pragma unroll
    for (int c = lane * 4; c < G; c += 128) {
        const float4 u = *reinterpret_cast<const float4 *>(acc + c);
        const float4 g = *reinterpret_cast<const float4 *>(acc + G + c);
        store4<OutT>(o + c, gelu_erf(u.x) * g.x, gelu_erf(u.y) * g.y, gelu_erf(u.z) * g.z, gelu_erf(u.w) * g.w);
    }
}

template <typename OutT, int BN>
__device__ __forceinline__ void epi_bias_act_row(const float *acc, int row, int n0, const EpiParams &ep, int lane) {
    OutT *o = reinterpret_cast<OutT *>(ep.out) + (size_t)row * ep.ldo + n0;
#pragma unroll
    for (int c = lane * 4; c < BN; c += 128) {
        float4 a = *reinterpret_cast<const float4 *>(acc + c);
        if (ep.bias) {
            const float4 b = *reinterpret_cast<const float4 *>(ep.bias + n0 + c);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        if (ep.act == 0) {
            a.x = fmaxf(a.x, 0.f); a.y = fmaxf(a.y, 0.f); a.z = fmaxf(a.z, 0.f); a.w = fmaxf(a.w, 0.f);
        } else {
            a.x = gelu_erf(a.x); a.y = gelu_erf(a.y); a.z = gelu_erf(a.z); a.w = gelu_erf(a.w);
        }
        store4<OutT>(o + c, a.x, a.y, a.z, a.w);
    }
}

template <int EPI, typename OutT, int BN>
__device__ __forceinline__ void epi_row(const float *acc, int row, int n0, const EpiParams &ep, int lane) {
    if constexpr (EPI == EPI_QKV) epi_qkv_row<OutT, BN>(acc, row, n0, ep, lane);
    else if constexpr (EPI == EPI_RESID_LN) epi_resid_ln_row<OutT>(acc, row, ep, lane);
    else if constexpr (EPI == EPI_GEGLU) epi_geglu_row<OutT, BN>(acc, row, n0, ep, lane);
    else epi_bias_act_row<OutT, BN>(acc, row, n0, ep, lane);
}

}  // namespace jd
