// Launchers of the library's kernels (host side).  Every launcher queues work
// on the given stream and returns the launch status; none allocates memory.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "epilogue.cuh"

namespace jd {

// Opt-in shared-memory sizes of every kernel that needs more than 48 KB; call
// once per device before the first launch (not during stream capture).
cudaError_t init_kernel_attributes();

// One projection: out = epilogue(A[rows, K] . W[N, K]^T).
struct GemmOp {
    int epi;                  // EpiKind
    int bn;                   // tile width: 384 (QKV, RESID_LN) or 256 (GEGLU, BIAS_ACT)
    int K, N;
    const CUtensorMap *tmA;   // BF16 path: A box 64 x 128
    const CUtensorMap *tmB;   // BF16 path: W box 64 x (bn == 384 ? 192 : 256)
    const CUtensorMap *tmO;   // BF16 column-split epilogues: output, box 64 x 32, 128-byte swizzle
    const CUtensorMap *tmX;   // BF16 residual epilogue: FP32 residual, box 32 x 128, 128-byte swizzle
    const CUtensorMap *tmXN;  // BF16 residual epilogue: LayerNorm output, box 64 x 128, 128-byte swizzle
    const CUtensorMap *tmA64; // BF16 residual GEMM: A box 32 x 128, 64-byte swizzle
    const CUtensorMap *tmB64; // BF16 residual GEMM: W box 32 x 192, 64-byte swizzle
    const CUtensorMap *tmBs;  // BF16 residual GEMM split over a cluster: W box 64 x 64, 128-byte swizzle
    const CUtensorMap *tmBp;  // BF16 persistent split residual GEMM: W box 64 x 192, 128-byte swizzle
    const float *A32;         // FP32 path: A [rows, lda]
    int lda;
    const float *W32;         // FP32 path: W [N, K]
    EpiParams ep;
    bool f8 = false;          // QKV on E4M3 operands (tmA, tmB: byte maps, box 128 x rows); needs ep.col_scale
    bool out8 = false;        // residual GEMM: LayerNorm output as E4M3 bytes (ep.out8_inv_scale); no ln_b
};
cudaError_t launch_gemm(const GemmOp &op, bool fp32, cudaStream_t st);

// Per-token row index / position and per-row attention work-unit offsets
// (qb_off holds 2 * (n_rows + 1) ints: 64-query then 256-query block offsets,
// followed by the row of every 256-query block (n_tokens / 256 + n_rows ints)
// and, for every 64-query block, its row's first and end token and its first
// query (3 ints each, (n_tokens + 63) / 64 + n_rows blocks: as many as the
// sliding-window attention's grid), in all qb_ints(n_rows, n_tokens) ints).
constexpr int qb_span_offset(int n_rows, int n_tokens) { return 2 * (n_rows + 1) + n_tokens / 256 + n_rows; }
constexpr size_t qb_ints(int n_rows, int n_tokens) {
    return (size_t)qb_span_offset(n_rows, n_tokens) + 3 * ((size_t)(n_tokens + 63) / 64 + n_rows);
}
cudaError_t launch_prep(const int *cu_seqlens, int n_rows, int n_tokens, int *tok_row, int *pos, int *qb_off,
                        cudaStream_t st);

// x = LN(E[token]) (gain only); xn = x in the activation type (inv8 > 0, BF16 models: xn holds
// the E4M3 bytes of x * inv8 instead).
cudaError_t launch_embed_ln(const int *tokens, int n_tokens, const float *E, int vocab, const float *g, float eps,
                            float *x, void *xn, bool fp32, unsigned *status, cudaStream_t st, float inv8 = 0.f);

// Varlen bidirectional attention inside each row.  qkv [T, 1152] holds
// q | k | v per token (head h at column h * 64 of each part); window < 0
// means global.  o [T, 384].
struct AttnArgs {
    const void *qkv;
    void *o;
    const int *cu_seqlens;
    const int *qb_off;        // the prep kernel's block offsets and block rows
    int n_rows, n_tokens;
    int window;
    const CUtensorMap *tm_qkv; // BF16 path: box 64 x 64 over [T_cap, 1152]
    const CUtensorMap *tm_qkv128; // BF16 global layers on tcgen05: box 64 x 128 (null: mma.sync kernel)
    unsigned *status;
};
cudaError_t launch_attention(const AttnArgs &a, bool fp32, cudaStream_t st);
cudaError_t launch_attention_tc(const AttnArgs &a, const CUtensorMap *tm128, int num_sms, cudaStream_t st);
int num_sms();

// Gather the marker rows: hm[m] = h[mask_pos[m]] (FP32), xm[m] = xn[mask_pos[m]].
cudaError_t launch_gather_markers(const int *mask_pos, int n_markers, int n_tokens, const float *h, const void *xn,
                                  float *hm, void *xm, bool fp32, unsigned *status, cudaStream_t st);

// Marker-only attention of the last head layer: the queries of each row's
// markers qm [M, 384] against all keys / values of that row (qkv columns 384..).
// Rows longer than 1024 keys split their keys over up to 8 CTAs per (row, head),
// with partial results in `part` (part_entries x 6 heads x 66 floats; null: no split)
// merged by a second kernel.
// BF16 with both maps (tm_q: marker queries, box 64 x 32; tm_kv: q|k|v, box 64 x 64) runs on
// the tensor cores (mma.sync); otherwise a SIMT kernel.
cudaError_t launch_marker_attention(const void *qm, const void *qkv, void *om, const int *cu_seqlens,
                                    const int *opt_off, int n_rows, int n_markers, int max_row_len, float *part,
                                    int part_entries, bool fp32, const CUtensorMap *tm_q, const CUtensorMap *tm_kv,
                                    unsigned *status, cudaStream_t st);
constexpr int MARKER_PART_ENTRIES_MIN = 4096;  // scratch entries: max(marker capacity, this)
int marker_attention_splits(int n_markers, int max_row_len, const float *part, int part_entries);

// The decision head after the last head layer, one launch: LayerNorm and scorer of every marker
// state hm [M, 384] (FP32), logits, per-row softmax and read-outs.
struct HeadArgs {
    const float *hm;
    int n_markers, n_rows;
    const int *opt_off;        // [n_rows + 1] markers of each row
    const int *row_type;       // [n_rows]
    const float *ln_g, *ln_b;
    const float *w1t, *b1;     // MLP: W1 transposed [384 in][384 out], bias [384]
    const float *w2, *b2;      // MLP: [384], [1]; linear variant: W [384], b [1]
    int linear;
    float eps;
    float *logits, *probs;     // [M]
    int *choice;               // [n_rows]
    float *score, *noul, *max_p;
    float *tap;                // optional copy of hm
    unsigned *status;
};
cudaError_t launch_head(const HeadArgs &a, cudaStream_t st);

}  // namespace jd
