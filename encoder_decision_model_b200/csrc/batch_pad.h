// Padding of a batch to its CUDA-graph bucket (host and device).
#pragma once

#include <cuda_runtime.h>

namespace jd {

// Bucketed CUDA graphs.  A batch of T tokens, B rows and M markers runs as the batch of its
// bucket: Tb tokens, B + 1 rows and Mb markers (pad_shape).  The added last row, the pad row,
// holds tokens T .. Tb - 1 (token id 0), markers M .. Mb - 1 on its first Mb - M tokens, and type
// 0.  Every kernel treats it as one more row, and no row's result depends on the other rows of
// its batch, so the real rows come out as they do from the unpadded batch.  The pad row has at
// least 8 tokens and at most 8 markers.
struct PadShape {
    int T, B, M;     // the batch
    int Tb, Bb, Mb;  // its bucket
};
inline PadShape pad_shape(int T, int B, int M) {
    return PadShape{T, B, M, (T + 8 + 127) / 128 * 128, B + 1, (M + 1 + 7) / 8 * 8};
}
// Entry i of each padded array, from the batch's own arrays (read only below T, B + 1, M).
__host__ __device__ inline int pad_token_at(const PadShape &s, const int *tokens, int i) {
    return i < s.T ? tokens[i] : 0;
}
__host__ __device__ inline int pad_cu_at(const PadShape &s, const int *cu, int i) { return i <= s.B ? cu[i] : s.Tb; }
__host__ __device__ inline int pad_opt_at(const PadShape &s, const int *opt, int i) { return i <= s.B ? opt[i] : s.Mb; }
__host__ __device__ inline int pad_mask_at(const PadShape &s, const int *mask, int i) {
    return i < s.M ? mask[i] : s.T + (i - s.M);
}
__host__ __device__ inline int pad_type_at(const PadShape &s, const int *type, int i) { return i < s.B ? type[i] : 0; }

// Writes the padded batch into d* (Tb, Bb + 1, Mb, Bb + 1, Bb ints); a source may be its own
// destination.
cudaError_t launch_pad_batch(const PadShape &s, const int *tokens, const int *cu, const int *mask, const int *opt,
                             const int *type, int *dtokens, int *dcu, int *dmask, int *dopt, int *dtype,
                             cudaStream_t st);
// Copies the real rows' outputs (M logits and probabilities, B read-outs of each kind) out of
// the padded batch's output arrays.
cudaError_t launch_unpad_outputs(int M, int B, const float *logits, const float *probs, const int *choice,
                                 const float *score, const float *noul, const float *max_p, float *o_logits,
                                 float *o_probs, int *o_choice, float *o_score, float *o_noul, float *o_max_p,
                                 cudaStream_t st);

}  // namespace jd
