// Bandwidth-bound kernels around the projections and attention: batch
// metadata, embedding gather + LayerNorm, marker gather, the scorer and the
// per-question read-outs.

#include "common.cuh"
#include "kernels.h"

namespace jd {

// ------------------------------------------------------------------ metadata

__global__ void k_token_meta(const int *__restrict__ cu, int n_rows, int *__restrict__ tok_row, int *__restrict__ pos) {
    for (int r = blockIdx.x; r < n_rows; r += gridDim.x) {
        const int cs = cu[r], ce = cu[r + 1];
        for (int t = cs + threadIdx.x; t < ce; t += blockDim.x) {
            tok_row[t] = r;
            pos[t] = t - cs;
        }
    }
}

// Attention work-unit offsets, one CTA of 1024 threads:
//   qb_off[r]             = sum over rows < r of ceil(len / 64)   (64-query blocks)
//   qb_off[n_rows + 1 + r] = sum over rows < r of ceil(len / 256)  (256-query blocks)
__global__ void __launch_bounds__(1024) k_qblock_offsets(const int *__restrict__ cu, int n_rows, int *__restrict__ qb_off) {
    __shared__ int part[2][1024];
    const int tid = threadIdx.x;
    const int per = (n_rows + 1023) / 1024;
    const int r0 = tid * per, r1 = min(n_rows, r0 + per);
    int s64 = 0, s256 = 0;
    for (int r = r0; r < r1; ++r) {
        const int len = cu[r + 1] - cu[r];
        s64 += (len + 63) / 64;
        s256 += (len + 255) / 256;
    }
    part[0][tid] = s64;
    part[1][tid] = s256;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive scans
        const int v0 = tid >= off ? part[0][tid - off] : 0;
        const int v1 = tid >= off ? part[1][tid - off] : 0;
        __syncthreads();
        part[0][tid] += v0;
        part[1][tid] += v1;
        __syncthreads();
    }
    int run64 = tid ? part[0][tid - 1] : 0, run256 = tid ? part[1][tid - 1] : 0;
    int *q256 = qb_off + n_rows + 1;
    for (int r = r0; r < r1; ++r) {
        const int len = cu[r + 1] - cu[r];
        qb_off[r] = run64;
        q256[r] = run256;
        run64 += (len + 63) / 64;
        run256 += (len + 255) / 256;
    }
    if (tid == 1023) {
        qb_off[n_rows] = part[0][1023];
        q256[n_rows] = part[1][1023];
    }
}

// row of every 256-query block: pb_row[q256[r] .. q256[r + 1]) = r
__global__ void k_qblock_rows(const int *__restrict__ qb_off, int n_rows, int *__restrict__ pb_row) {
    const int *q256 = qb_off + n_rows + 1;
    for (int r = blockIdx.x * blockDim.y + threadIdx.y; r < n_rows; r += gridDim.x * blockDim.y)
        for (int pb = q256[r] + threadIdx.x; pb < q256[r + 1]; pb += blockDim.x) pb_row[pb] = r;
}

cudaError_t launch_prep(const int *cu_seqlens, int n_rows, int n_tokens, int *tok_row, int *pos, int *qb_off,
                        cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    (void)n_tokens;
    k_token_meta<<<min(n_rows, 4096), 256, 0, st>>>(cu_seqlens, n_rows, tok_row, pos);
    k_qblock_offsets<<<1, 1024, 0, st>>>(cu_seqlens, n_rows, qb_off);
    k_qblock_rows<<<min((n_rows + 7) / 8, 1024), dim3(32, 8), 0, st>>>(qb_off, n_rows, qb_off + 2 * (n_rows + 1));
    return cudaGetLastError();
}

// ------------------------------------------------------------------ embedding gather + LayerNorm

// One warp per token: x = LN(E[id]) with the embedding norm's gain ("Julia-1
// MLX", "Performance": a request reads only the embedding rows of its own
// tokens).  Layer 0 has no pre-attention norm, so x is also its operand.
template <typename OutT>
__global__ void __launch_bounds__(256)
    k_embed_ln(const int *__restrict__ tokens, int n_tokens, const float *__restrict__ E, int vocab,
               const float *__restrict__ g, float eps, float *__restrict__ x, OutT *__restrict__ xn, unsigned *status) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= n_tokens) return;
    int id = tokens[t];
    if (id < 0 || id >= vocab) {
        if (lane == 0) atomicOr(status, ST_TOKEN_RANGE);
        id = 0;
    }
    const float *e = E + (size_t)id * D;
    float v[12];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(e + j * 128 + lane * 4));
        v[4 * j] = a.x; v[4 * j + 1] = a.y; v[4 * j + 2] = a.z; v[4 * j + 3] = a.w;
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 12; ++k) s += v[k];
    const float mean = warp_sum(s) * (1.0f / D);
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < 12; ++k) {
        v[k] -= mean;
        q += v[k] * v[k];
    }
    const float rstd = 1.0f / sqrtf(warp_sum(q) * (1.0f / D) + eps);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int c = j * 128 + lane * 4;
        const float4 gg = *reinterpret_cast<const float4 *>(g + c);
        const float a0 = v[4 * j] * rstd * gg.x, a1 = v[4 * j + 1] * rstd * gg.y;
        const float a2 = v[4 * j + 2] * rstd * gg.z, a3 = v[4 * j + 3] * rstd * gg.w;
        *reinterpret_cast<float4 *>(x + (size_t)t * D + c) = make_float4(a0, a1, a2, a3);
        store4<OutT>(xn + (size_t)t * D + c, a0, a1, a2, a3);
    }
}

cudaError_t launch_embed_ln(const int *tokens, int n_tokens, const float *E, int vocab, const float *g, float eps,
                            float *x, void *xn, bool fp32, unsigned *status, cudaStream_t st) {
    if (n_tokens <= 0) return cudaSuccess;
    const int blocks = (n_tokens + 7) / 8;
    if (fp32)
        k_embed_ln<float><<<blocks, 256, 0, st>>>(tokens, n_tokens, E, vocab, g, eps, x, (float *)xn, status);
    else
        k_embed_ln<__nv_bfloat16><<<blocks, 256, 0, st>>>(tokens, n_tokens, E, vocab, g, eps, x,
                                                          (__nv_bfloat16 *)xn, status);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ marker gather

template <typename T>
__global__ void __launch_bounds__(256)
    k_gather_markers(const int *__restrict__ mask_pos, int n_markers, int n_tokens, const float *__restrict__ h,
                     const T *__restrict__ xn, float *__restrict__ hm, T *__restrict__ xm, unsigned *status) {
    const int m = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (m >= n_markers) return;
    int p = mask_pos[m];
    if (p < 0 || p >= n_tokens) {
        if (lane == 0) atomicOr(status, ST_BAD_INDEX);
        p = 0;
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int c = j * 128 + lane * 4;
        *reinterpret_cast<float4 *>(hm + (size_t)m * D + c) = *reinterpret_cast<const float4 *>(h + (size_t)p * D + c);
        const float4 a = load4f<T>(xn + (size_t)p * D + c);
        store4<T>(xm + (size_t)m * D + c, a.x, a.y, a.z, a.w);
    }
}

cudaError_t launch_gather_markers(const int *mask_pos, int n_markers, int n_tokens, const float *h, const void *xn,
                                  float *hm, void *xm, bool fp32, unsigned *status, cudaStream_t st) {
    if (n_markers <= 0) return cudaSuccess;
    const int blocks = (n_markers + 7) / 8;
    if (fp32)
        k_gather_markers<float><<<blocks, 256, 0, st>>>(mask_pos, n_markers, n_tokens, h, (const float *)xn, hm,
                                                        (float *)xm, status);
    else
        k_gather_markers<__nv_bfloat16><<<blocks, 256, 0, st>>>(mask_pos, n_markers, n_tokens, h,
                                                                (const __nv_bfloat16 *)xn, hm, (__nv_bfloat16 *)xm,
                                                                status);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ scorer

// "Julia-1: one score per mask token", "The decision head", step 4: LayerNorm
// -> Linear(384, 384) -> GELU -> Linear(384, 1) per option (FP32).  One CTA
// scores 32 markers; the hidden layer keeps W1 reads coalesced (W1 stored
// transposed) and the marker vectors in shared memory.
constexpr int SC_M = 32;

__global__ void __launch_bounds__(256) k_scorer(ScorerArgs a) {
    extern __shared__ float sn[];  // [SC_M][D]
    const int m0 = blockIdx.x * SC_M;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nm = min(SC_M, a.n_markers - m0);
    for (int mi = warp; mi < SC_M; mi += 8) {
        float v[12];
        if (mi < nm) {
            const float *src = a.hm + (size_t)(m0 + mi) * D;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const float4 x = *reinterpret_cast<const float4 *>(src + j * 128 + lane * 4);
                v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                if (a.tap) *reinterpret_cast<float4 *>(a.tap + (size_t)(m0 + mi) * D + j * 128 + lane * 4) = x;
            }
            float s = 0.f;
#pragma unroll
            for (int k = 0; k < 12; ++k) s += v[k];
            const float mean = warp_sum(s) * (1.0f / D);
            float q = 0.f;
#pragma unroll
            for (int k = 0; k < 12; ++k) {
                v[k] -= mean;
                q += v[k] * v[k];
            }
            const float rstd = 1.0f / sqrtf(warp_sum(q) * (1.0f / D) + a.eps);
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const int c = j * 128 + lane * 4;
#pragma unroll
                for (int e = 0; e < 4; ++e) v[4 * j + e] = v[4 * j + e] * rstd * a.ln_g[c + e] + a.ln_b[c + e];
            }
        } else {
#pragma unroll
            for (int k = 0; k < 12; ++k) v[k] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) sn[mi * D + j * 128 + lane * 4 + e] = v[4 * j + e];
    }
    __syncthreads();
    if (a.linear) {
        for (int mi = warp; mi < nm; mi += 8) {
            float s = 0.f;
            for (int c = lane; c < D; c += 32) s = fmaf(sn[mi * D + c], a.w2[c], s);
            s = warp_sum(s);
            if (lane == 0) a.logits[m0 + mi] = s + a.b2[0];
        }
        return;
    }
    float acc0[SC_M], acc1[SC_M];
    const int o0 = tid, o1 = tid + 256;  // output features; o1 valid when < 384
#pragma unroll
    for (int mi = 0; mi < SC_M; ++mi) acc0[mi] = acc1[mi] = 0.f;
    for (int k = 0; k < D; ++k) {
        const float w0 = a.w1t[k * D + o0];
        const float w1 = o1 < D ? a.w1t[k * D + o1] : 0.f;
#pragma unroll
        for (int mi = 0; mi < SC_M; ++mi) {
            const float xv = sn[mi * D + k];
            acc0[mi] = fmaf(xv, w0, acc0[mi]);
            acc1[mi] = fmaf(xv, w1, acc1[mi]);
        }
    }
    __syncthreads();
    const float bb0 = a.b1[o0], bb1 = o1 < D ? a.b1[o1] : 0.f;
#pragma unroll
    for (int mi = 0; mi < SC_M; ++mi) {
        sn[mi * D + o0] = gelu_erf(acc0[mi] + bb0);
        if (o1 < D) sn[mi * D + o1] = gelu_erf(acc1[mi] + bb1);
    }
    __syncthreads();
    for (int mi = warp; mi < nm; mi += 8) {
        float s = 0.f;
        for (int c = lane; c < D; c += 32) s = fmaf(sn[mi * D + c], a.w2[c], s);
        s = warp_sum(s);
        if (lane == 0) a.logits[m0 + mi] = s + a.b2[0];
    }
}

cudaError_t gemm_init_attributes();
cudaError_t attn_init_attributes();

cudaError_t init_kernel_attributes() {
    cudaError_t e = cudaFuncSetAttribute(k_scorer, cudaFuncAttributeMaxDynamicSharedMemorySize, SC_M * D * 4);
    if (e != cudaSuccess) return e;
    if ((e = attn_init_attributes()) != cudaSuccess) return e;
    return gemm_init_attributes();
}

cudaError_t launch_scorer(const ScorerArgs &a, cudaStream_t st) {
    if (a.n_markers <= 0) return cudaSuccess;
    const int smem = SC_M * D * 4;
    k_scorer<<<(a.n_markers + SC_M - 1) / SC_M, 256, smem, st>>>(a);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ read-outs

// "Three modes through one head": softmax across the options at temperature
// 1; choice = argmax (lowest index on ties), score = sum_i i p_i, noul =
// p(true) = p_1 for noul rows (NaN otherwise), max_p.  One warp per row.
__global__ void __launch_bounds__(256)
    k_readout(const float *__restrict__ z, const int *__restrict__ opt_off, const int *__restrict__ row_type, int n_rows,
              float *__restrict__ probs, int *__restrict__ choice, float *__restrict__ score, float *__restrict__ noul,
              float *__restrict__ max_p) {
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (r >= n_rows) return;
    const int b = opt_off[r], k = opt_off[r + 1] - b;
    float mx = -INFINITY;
    int arg = 0x7fffffff;
    for (int i = lane; i < k; i += 32) {
        const float v = z[b + i];
        if (v > mx) { mx = v; arg = i; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, mx, o);
        const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
        if (om > mx || (om == mx && oa < arg)) { mx = om; arg = oa; }
    }
    float s = 0.f;
    for (int i = lane; i < k; i += 32) s += expf(z[b + i] - mx);
    s = warp_sum(s);
    const float inv = 1.0f / s;
    float sc = 0.f, p1 = 0.f;
    for (int i = lane; i < k; i += 32) {
        const float p = expf(z[b + i] - mx) * inv;
        probs[b + i] = p;
        sc += (float)i * p;
        if (i == 1) p1 = p;
    }
    sc = warp_sum(sc);
    p1 = warp_sum(p1);
    if (lane == 0) {
        choice[r] = arg;
        score[r] = sc;
        noul[r] = row_type[r] == 2 ? p1 : __int_as_float(0x7fc00000);
        max_p[r] = inv;  // exp(max - max) / sum
    }
}

cudaError_t launch_readout(const float *logits, const int *opt_off, const int *row_type, int n_rows, float *probs,
                           int *choice, float *score, float *noul, float *max_p, cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    k_readout<<<(n_rows + 7) / 8, 256, 0, st>>>(logits, opt_off, row_type, n_rows, probs, choice, score, noul, max_p);
    return cudaGetLastError();
}

}  // namespace jd
