// Bandwidth-bound kernels around the projections and attention: batch
// metadata, embedding gather + LayerNorm, marker gather.

#include "common.cuh"
#include "kernels.h"
#include "batch_pad.h"

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

// Attention work units, one CTA of 1024 threads:
//   qb_off[r]              = sum over rows < r of ceil(len / 64)   (64-query blocks)
//   qb_off[n_rows + 1 + r] = sum over rows < r of ceil(len / 256)  (256-query blocks)
// then, by the thread that owns row r, the row of each of its 256-query blocks (pb_row) and
// each of its 64-query blocks' row start, row end and first query (span[3 b .. 3 b + 2]).
__global__ void __launch_bounds__(1024) k_qblock_meta(const int *__restrict__ cu, int n_rows, int *__restrict__ qb_off,
                                                      int *__restrict__ pb_row, int *__restrict__ span) {
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
        const int cs = cu[r], ce = cu[r + 1], len = ce - cs;
        const int n64 = (len + 63) / 64, n256 = (len + 255) / 256;
        qb_off[r] = run64;
        q256[r] = run256;
        for (int b = 0; b < n256; ++b) pb_row[run256 + b] = r;
        for (int b = 0; b < n64; ++b) {
            int *sp = span + 3 * (run64 + b);
            sp[0] = cs;
            sp[1] = ce;
            sp[2] = cs + b * 64;
        }
        run64 += n64;
        run256 += n256;
    }
    if (tid == 1023) {
        qb_off[n_rows] = part[0][1023];
        q256[n_rows] = part[1][1023];
    }
}

cudaError_t launch_prep(const int *cu_seqlens, int n_rows, int n_tokens, int *tok_row, int *pos, int *qb_off,
                        cudaStream_t st) {
    if (n_rows <= 0) return cudaSuccess;
    k_token_meta<<<min(n_rows, 4096), 256, 0, st>>>(cu_seqlens, n_rows, tok_row, pos);
    k_qblock_meta<<<1, 1024, 0, st>>>(cu_seqlens, n_rows, qb_off, qb_off + 2 * (n_rows + 1),
                                      qb_off + qb_span_offset(n_rows, n_tokens));
    return cudaGetLastError();
}

// ------------------------------------------------------------------ embedding gather + LayerNorm

// One warp per token: x = LN(E[id]) with the embedding norm's gain ("Julia-1
// MLX", "Performance": a request reads only the embedding rows of its own
// tokens).  Layer 0 has no pre-attention norm, so x is also its operand.
// OutT uint8_t: xn as E4M3 bytes of y * inv8 (the operand of the FP8 QKV GEMM).
template <typename OutT>
__global__ void __launch_bounds__(256)
    k_embed_ln(const int *__restrict__ tokens, int n_tokens, const float *__restrict__ E, int vocab,
               const float *__restrict__ g, float eps, float *__restrict__ x, OutT *__restrict__ xn, float inv8,
               unsigned *status) {
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
        if constexpr (sizeof(OutT) == 1)
            *reinterpret_cast<uint32_t *>(xn + (size_t)t * D + c) =
                pack_e4m3x2(a0 * inv8, a1 * inv8) | (pack_e4m3x2(a2 * inv8, a3 * inv8) << 16);
        else
            store4<OutT>(xn + (size_t)t * D + c, a0, a1, a2, a3);
    }
}

cudaError_t launch_embed_ln(const int *tokens, int n_tokens, const float *E, int vocab, const float *g, float eps,
                            float *x, void *xn, bool fp32, unsigned *status, cudaStream_t st, float inv8) {
    if (n_tokens <= 0) return cudaSuccess;
    const int blocks = (n_tokens + 7) / 8;
    if (fp32)
        k_embed_ln<float><<<blocks, 256, 0, st>>>(tokens, n_tokens, E, vocab, g, eps, x, (float *)xn, 0.f, status);
    else if (inv8 > 0.f)
        k_embed_ln<uint8_t><<<blocks, 256, 0, st>>>(tokens, n_tokens, E, vocab, g, eps, x, (uint8_t *)xn, inv8,
                                                    status);
    else
        k_embed_ln<__nv_bfloat16><<<blocks, 256, 0, st>>>(tokens, n_tokens, E, vocab, g, eps, x,
                                                          (__nv_bfloat16 *)xn, 0.f, status);
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

// ------------------------------------------------------------------ bucket padding

__global__ void __launch_bounds__(256)
    k_pad_batch(PadShape s, const int *tokens, const int *cu, const int *mask, const int *opt, const int *type,
                int *dtokens, int *dcu, int *dmask, int *dopt, int *dtype) {
    const int stride = gridDim.x * blockDim.x;
    const int n = max(s.Tb, max(s.Mb, s.Bb + 1));
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        if (i < s.Tb) dtokens[i] = pad_token_at(s, tokens, i);
        if (i < s.Mb) dmask[i] = pad_mask_at(s, mask, i);
        if (i <= s.Bb) {
            dcu[i] = pad_cu_at(s, cu, i);
            dopt[i] = pad_opt_at(s, opt, i);
        }
        if (i < s.Bb) dtype[i] = pad_type_at(s, type, i);
    }
}

cudaError_t launch_pad_batch(const PadShape &s, const int *tokens, const int *cu, const int *mask, const int *opt,
                             const int *type, int *dtokens, int *dcu, int *dmask, int *dopt, int *dtype,
                             cudaStream_t st) {
    const int n = max(s.Tb, max(s.Mb, s.Bb + 1));
    k_pad_batch<<<min((n + 255) / 256, 1184), 256, 0, st>>>(s, tokens, cu, mask, opt, type, dtokens, dcu, dmask,
                                                             dopt, dtype);
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256)
    k_unpad_outputs(int M, int B, const float *logits, const float *probs, const int *choice, const float *score,
                    const float *noul, const float *max_p, float *o_logits, float *o_probs, int *o_choice,
                    float *o_score, float *o_noul, float *o_max_p) {
    const int stride = gridDim.x * blockDim.x;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < max(M, B); i += stride) {
        if (i < M) {
            o_logits[i] = logits[i];
            o_probs[i] = probs[i];
        }
        if (i < B) {
            o_choice[i] = choice[i];
            o_score[i] = score[i];
            o_noul[i] = noul[i];
            o_max_p[i] = max_p[i];
        }
    }
}

cudaError_t launch_unpad_outputs(int M, int B, const float *logits, const float *probs, const int *choice,
                                 const float *score, const float *noul, const float *max_p, float *o_logits,
                                 float *o_probs, int *o_choice, float *o_score, float *o_noul, float *o_max_p,
                                 cudaStream_t st) {
    const int n = max(M, B);
    if (n <= 0) return cudaSuccess;
    k_unpad_outputs<<<min((n + 255) / 256, 148), 256, 0, st>>>(M, B, logits, probs, choice, score, noul, max_p,
                                                              o_logits, o_probs, o_choice, o_score, o_noul, o_max_p);
    return cudaGetLastError();
}

cudaError_t gemm_init_attributes();
cudaError_t attn_init_attributes();
cudaError_t head_init_attributes();

cudaError_t init_kernel_attributes() {
    cudaError_t e = head_init_attributes();
    if (e != cudaSuccess) return e;
    if ((e = attn_init_attributes()) != cudaSuccess) return e;
    return gemm_init_attributes();
}

}  // namespace jd
