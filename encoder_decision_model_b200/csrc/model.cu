// jd_model: device weights, workspace and the launch sequence of the forward
// pass ("Julia-1: one score per mask token", "The decision head").
//
// Per encoder layer l (global iff l % 3 == 0; "Julia-1 MLX", "Performance"):
//   QKV GEMM + RoPE      xn -> qkv                 (theta 160000 global / 10000 local)
//   attention            qkv -> o                  (global, or keys with |i - j| <= 64)
//   Wo GEMM + residual   x += o Wo^T; xn = LN_mlp(x)
//   Wi GEMM + GEGLU      y = GELU(u) * g
//   Wo2 GEMM + residual  x += y Wo2^T; xn = LN_attn(l+1)(x)
//     (last layer: h = LN_final(x) + type row, xn = LN1 of head layer 0)
// Head layer 0 (all tokens) and head layer 1 (keys / values for all tokens,
// everything else only at the markers), scorer, read-outs.
//
// Weights file: .jdw (see workloads/gen.py for the writer), FP32.  The
// library keeps the embedding table, norms, biases, type table and scorer in
// FP32 and stores projection weights as BF16 (BF16 mode) or FP32 (validation
// mode).  Wi rows are interleaved in blocks of 128 ([u_j | g_j]) so that one
// 256-wide GEMM tile holds both halves of 128 GEGLU outputs.

#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "e4m3.h"
#include "host_common.h"
#include "kernels.h"
#include "batch_pad.h"
#include "route_kernels.h"

using namespace jd;

namespace {

constexpr int NL = 22;
constexpr int VOCAB = 256000;
constexpr float EPS = 1e-5f;

#define CK(call)                                                                                       \
    do {                                                                                               \
        cudaError_t e_ = (call);                                                                       \
        if (e_ != cudaSuccess) return jd::fail(JD_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

// ---------------------------------------------------------------- weights file

struct TensorRec {
    std::vector<uint32_t> shape;
    uint64_t offset;  // absolute
    uint64_t count;
};

struct WeightFile {
    std::map<std::string, TensorRec> idx;
    FILE *fh = nullptr;
    ~WeightFile() {
        if (fh) fclose(fh);
    }
};

jd_status open_weights(const char *path, WeightFile &wf) {
    wf.fh = fopen(path, "rb");
    if (!wf.fh) return fail(JD_ERR_IO, "cannot open weights file %s", path);
    char magic[8];
    uint32_t n = 0;
    if (fread(magic, 1, 8, wf.fh) != 8 || memcmp(magic, "JDWGT001", 8) != 0 || fread(&n, 4, 1, wf.fh) != 1)
        return fail(JD_ERR_IO, "%s is not a .jdw weights file", path);
    const uint64_t header = 12ull + 96ull * n;
    const uint64_t data0 = (header + 255) / 256 * 256;
    for (uint32_t i = 0; i < n; ++i) {
        unsigned char rec[96];
        if (fread(rec, 1, 96, wf.fh) != 96) return fail(JD_ERR_IO, "truncated weights header");
        char name[65];
        memcpy(name, rec, 64);
        name[64] = 0;
        uint32_t ndim, dims[4];
        uint64_t off;
        memcpy(&ndim, rec + 64, 4);
        memcpy(dims, rec + 68, 16);
        memcpy(&off, rec + 84, 8);
        TensorRec t;
        t.count = 1;
        for (uint32_t d = 0; d < ndim && d < 4; ++d) {
            t.shape.push_back(dims[d]);
            t.count *= dims[d];
        }
        t.offset = data0 + off;
        wf.idx[name] = t;
    }
    return JD_OK;
}

jd_status read_tensor(WeightFile &wf, const std::string &name, std::vector<uint32_t> shape, std::vector<float> &out) {
    auto it = wf.idx.find(name);
    if (it == wf.idx.end()) return fail(JD_ERR_IO, "weights file has no tensor %s", name.c_str());
    if (it->second.shape != shape) return fail(JD_ERR_IO, "tensor %s has an unexpected shape", name.c_str());
    out.resize(it->second.count);
    if (fseeko(wf.fh, (off_t)it->second.offset, SEEK_SET) != 0 ||
        fread(out.data(), 4, out.size(), wf.fh) != out.size())
        return fail(JD_ERR_IO, "cannot read tensor %s", name.c_str());
    return JD_OK;
}

// FP32 -> BF16, round to nearest even (NaN kept quiet).
uint16_t to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over [rows, cols] with row stride ld (elements); box = box_cols x box_rows, 128-byte
// swizzle unless sw64 (64-byte swizzle, for boxes of 32 bf16 columns).  Elements are bf16,
// FP32 (fp32) or bytes (u8: the E4M3 operands of the FP8 QKV GEMM).
jd_status make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t ld, uint32_t box_cols,
                   uint32_t box_rows, bool fp32 = false, bool sw64 = false, bool u8 = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(JD_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * (fp32 ? 4 : (u8 ? 1 : 2))};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    const CUtensorMapDataType dt = fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                        : (u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(JD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return JD_OK;
}

struct ProjW {            // one projection weight [N, K]
    void *w = nullptr;    // bf16 or f32 on device
    CUtensorMap tm{};     // BF16 mode only
    CUtensorMap tm64{};   // BF16 mode, 384-wide tiles: box 32 x 192, 64-byte swizzle (residual GEMM)
    CUtensorMap tms{};    // BF16 mode, 384-wide tiles: box 64 x 64 (split residual GEMM, one-head QKV tiles)
    bool has_tms = false;
    int N = 0, K = 0;
    // FP8 mode, encoder QKV: E4M3 codes of W[n, :] / s_n (s_n = max_k |W[n, k]| / 448), box 128 x 192,
    // and per output column the product of the input's activation scale and s_n
    void *w8 = nullptr;
    CUtensorMap tm8{};
    float *col_scale = nullptr;
};

}  // namespace

struct jd_model {
    jd_model_config cfg{};
    int device = 0;
    bool fp32 = false;
    bool fp8 = false;           // JD_PREC_FP8: the encoder QKV projections on E4M3 operands
    float inv8[22] = {};        // FP8 mode: 1 / activation scale of each encoder layer's QKV input
    int T_cap = 0, B_cap = 0, M_cap = 0;
    size_t bytes = 0;
    std::vector<void *> allocs;

    // weights
    float *E = nullptr, *emb_g = nullptr, *fin_g = nullptr, *type_tab = nullptr;
    float *attn_g[NL] = {}, *mlp_g[NL] = {};
    ProjW Wqkv[NL], Wo[NL], Wi[NL], Wo2[NL];
    float *n1g[2] = {}, *n1b[2] = {}, *n2g[2] = {}, *n2b[2] = {};
    ProjW in_full[2], in_q[2], in_kv[2], out_p[2], lin1[2], lin2[2];
    float *in_b[2] = {}, *out_b[2] = {}, *l1_b[2] = {}, *l2_b[2] = {};
    float *sc_g = nullptr, *sc_b = nullptr, *sc_w1t = nullptr, *sc_b1 = nullptr, *sc_w2 = nullptr, *sc_b2 = nullptr;
    float *lin_w = nullptr, *lin_b = nullptr;
    float4 *rope_g = nullptr, *rope_l = nullptr;  // [16][MAX_POS] (cos, sin) of pairs 2k, 2k + 1

    // workspace
    float *x = nullptr;
    void *xn = nullptr, *qkv = nullptr, *o = nullptr, *y = nullptr;
    int *tok_row = nullptr, *pos = nullptr, *qb_off = nullptr;
    float *hm = nullptr;
    float *mk_part = nullptr;  // key-split partials of the marker attention
    int mk_part_entries = 0;
    void *xm = nullptr, *qm = nullptr, *om = nullptr, *xnm = nullptr, *ym = nullptr;
    unsigned *status = nullptr;
    uint8_t *xn8 = nullptr;     // FP8 mode: E4M3 QKV input [T, 384]
    CUtensorMap tm_xn8{};       // box 128 x 128 bytes
    CUtensorMap tm_xn{}, tm_o{}, tm_y_enc{}, tm_y_head{}, tm_qkv{}, tm_xm{}, tm_om{}, tm_xnm{}, tm_ym{};
    CUtensorMap tm_o64{}, tm_y_enc64{}, tm_y_head64{};  // residual GEMM A operands: box 32 x 128, 64-byte swizzle
    // output maps of the column-split epilogues (box 64 x 32)
    CUtensorMap to_qkv{}, to_y_enc{}, to_y_head{}, to_qm{}, to_ym{};
    CUtensorMap tm_x32{};  // FP32 residual stream, box 32 x 128
    CUtensorMap tm_qkv128{};  // q|k|v, box 64 x 128 (tensor-core attention)

    // internal outputs (jd_forward, host entry points) and device batch staging
    float *i_logits = nullptr, *i_probs = nullptr, *i_score = nullptr, *i_noul = nullptr, *i_maxp = nullptr;
    int *i_choice = nullptr;
    int *d_tokens = nullptr, *d_cu = nullptr, *d_mask = nullptr, *d_opt = nullptr, *d_type = nullptr;
    // pinned host staging
    // pinned host staging of the host entry points: two slots, so that one call can be prepared
    // while the previous one runs (jd_decide_host_submit / jd_decide_host_collect); slot 1 is
    // allocated on first use
    struct HostSlot {
        int *h_tokens = nullptr, *h_cu = nullptr, *h_mask = nullptr, *h_opt = nullptr, *h_type = nullptr;
        float *h_logits = nullptr, *h_probs = nullptr, *h_score = nullptr, *h_noul = nullptr, *h_maxp = nullptr;
        int *h_choice = nullptr;
        unsigned *h_status = nullptr;
        cudaEvent_t done = nullptr;  // recorded after the slot's outputs are copied back
        int B = 0, M = 0;
    };
    HostSlot hs[2];
    int64_t submitted = 0, collected = 0;

    cudaStream_t last_stream = nullptr;

    // device-side router (jd_route_device): workspace grown on demand, pinned read-back slots
    void *route_buf = nullptr;
    size_t route_bytes = 0;
    int *h_route = nullptr;  // [16]: the round's counters, then the status word
    int launches = 0;

    // per-kernel event timing (profiling mode)
    bool prof = false;
    std::vector<cudaEvent_t> ev;
    std::vector<const char *> ev_name;
    int n_ev = 0;
    std::map<std::string, std::pair<long, double>> prof_acc;

    // CUDA graphs: one per bucket of padded batch shapes (tokens, rows, markers, longest row),
    // least recently used dropped beyond GRAPH_BUCKETS_MAX, plus one exact-shape entry for the
    // calls that no bucket serves (taps requested, or a bucket beyond the capacity)
    bool graph_mode = false;
    struct Bucket {
        cudaGraphExec_t exec = nullptr;
        int launches = 0;
        long last_use = 0;
    };
    std::map<std::array<int, 4>, Bucket> gbuckets;
    long gclock = 0;
    long g_captures = 0, g_replays = 0;
    cudaGraphExec_t gexec = nullptr;
    int gexec_launches = 0;
    std::vector<uintptr_t> gkey;

    template <class T>
    jd_status dalloc(T **p, size_t n) {
        void *q = nullptr;
        size_t b = std::max<size_t>(n, 1) * sizeof(T);
        cudaError_t e = cudaMalloc(&q, b);
        if (e != cudaSuccess) return fail(JD_ERR_CUDA, "cudaMalloc(%zu): %s", b, cudaGetErrorString(e));
        e = cudaMemset(q, 0, b);
        if (e != cudaSuccess) return fail(JD_ERR_CUDA, "cudaMemset: %s", cudaGetErrorString(e));
        allocs.push_back(q);
        bytes += b;
        *p = static_cast<T *>(q);
        return JD_OK;
    }
    template <class T>
    jd_status halloc(T **p, size_t n) {
        void *q = nullptr;
        cudaError_t e = cudaHostAlloc(&q, std::max<size_t>(n, 1) * sizeof(T), cudaHostAllocDefault);
        if (e != cudaSuccess) return fail(JD_ERR_CUDA, "cudaHostAlloc: %s", cudaGetErrorString(e));
        hallocs.push_back(q);
        *p = static_cast<T *>(q);
        return JD_OK;
    }
    std::vector<void *> hallocs;
};

namespace {

#define TRY(call)                    \
    do {                             \
        jd_status s_ = (call);       \
        if (s_ != JD_OK) return s_;  \
    } while (0)

jd_status upload_f32(jd_model *m, WeightFile &wf, const std::string &name, std::vector<uint32_t> shape, float **dst) {
    std::vector<float> h;
    TRY(read_tensor(wf, name, shape, h));
    TRY(m->dalloc(dst, h.size()));
    CK(cudaMemcpy(*dst, h.data(), h.size() * 4, cudaMemcpyHostToDevice));
    return JD_OK;
}

// Upload rows [r0, r0 + N) of a host [*, K] matrix as a projection weight.
jd_status upload_proj(jd_model *m, const std::vector<float> &h, int r0, int N, int K, int bn, ProjW &p) {
    p.N = N;
    p.K = K;
    const float *src = h.data() + (size_t)r0 * K;
    if (m->fp32) {
        float *d = nullptr;
        TRY(m->dalloc(&d, (size_t)N * K));
        CK(cudaMemcpy(d, src, (size_t)N * K * 4, cudaMemcpyHostToDevice));
        p.w = d;
    } else {
        std::vector<uint16_t> b((size_t)N * K);
        for (size_t i = 0; i < b.size(); ++i) b[i] = to_bf16(src[i]);
        uint16_t *d = nullptr;
        TRY(m->dalloc(&d, b.size()));
        CK(cudaMemcpy(d, b.data(), b.size() * 2, cudaMemcpyHostToDevice));
        p.w = d;
        // one TMA box per MMA: 192 rows for 384-wide tiles (two N=192 MMAs), else the tile width
        const uint32_t box_rows = bn == 384 ? 192 : (uint32_t)bn;
        TRY(make_map(&p.tm, d, K, N, K, 64, box_rows));
        if (bn == 384) {
            TRY(make_map(&p.tm64, d, K, N, K, 32, 192, false, true));
            TRY(make_map(&p.tms, d, K, N, K, 64, 64));
            p.has_tms = true;
        }
    }
    return JD_OK;
}

// FP8 mode: E4M3 copy of a [N, K] projection with one scale per output row, the row scales
// multiplied by the scale of its input's activations (act_scale) into col_scale.
jd_status upload_proj_e4m3(jd_model *m, const std::vector<float> &h, int N, int K, float act_scale, ProjW &p) {
    p.N = N;
    p.K = K;
    std::vector<uint8_t> q((size_t)N * K);
    std::vector<float> cs(N);
    for (int n = 0; n < N; ++n) {
        const float *row = h.data() + (size_t)n * K;
        float amax = 0.f;
        for (int k = 0; k < K; ++k) amax = std::max(amax, std::fabs(row[k]));
        const float sn = amax > 0.f ? amax / 448.0f : 1.0f;
        for (int k = 0; k < K; ++k) q[(size_t)n * K + k] = e4m3_encode(row[k] / sn);
        cs[n] = act_scale * sn;
    }
    uint8_t *d = nullptr;
    TRY(m->dalloc(&d, q.size()));
    CK(cudaMemcpy(d, q.data(), q.size(), cudaMemcpyHostToDevice));
    p.w8 = d;
    TRY(make_map(&p.tm8, d, K, N, K, 128, 192, false, false, true));
    TRY(m->dalloc(&p.col_scale, N));
    CK(cudaMemcpy(p.col_scale, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice));
    return JD_OK;
}

// Scale of an E4M3 LayerNorm output with gain g (no bias): every |y_k| <= sqrt(384) * max |g|
// (a row's whole variance in one channel), so y / scale never saturates at 448.
float ln_e4m3_scale(const std::vector<float> &g) {
    float gm = 0.f;
    for (float v : g) gm = std::max(gm, std::fabs(v));
    return std::sqrt((float)D) * (gm > 0.f ? gm : 1.0f) / 448.0f;
}

jd_status load_proj(jd_model *m, WeightFile &wf, const std::string &name, int N, int K, int bn, ProjW &p) {
    std::vector<float> h;
    TRY(read_tensor(wf, name, {(uint32_t)N, (uint32_t)K}, h));
    return upload_proj(m, h, 0, N, K, bn, p);
}

// RoPE angles p * theta^(-2i/64) in double, stored as 16 position-minor planes:
// plane k, position p = (cos, sin) of frequency 2k, then of 2k + 1.
jd_status make_rope_table(jd_model *m, double theta, float4 **dst) {
    std::vector<float4> h((size_t)16 * MAX_POS);
    for (int k = 0; k < 16; ++k)
        for (int p = 0; p < MAX_POS; ++p) {
            const double a0 = (double)p * std::pow(theta, -2.0 * (2 * k) / 64.0);
            const double a1 = (double)p * std::pow(theta, -2.0 * (2 * k + 1) / 64.0);
            h[(size_t)k * MAX_POS + p] =
                make_float4((float)std::cos(a0), (float)std::sin(a0), (float)std::cos(a1), (float)std::sin(a1));
        }
    TRY(m->dalloc(dst, h.size()));
    CK(cudaMemcpy(*dst, h.data(), h.size() * sizeof(float4), cudaMemcpyHostToDevice));
    return JD_OK;
}

// Copy the weight pointers and their tensor maps of m into v (no device memory is allocated).
void share_weights(jd_model &v, const jd_model *m) {
    v.E = m->E; v.emb_g = m->emb_g; v.fin_g = m->fin_g; v.type_tab = m->type_tab;
    for (int l = 0; l < NL; ++l) {
        v.attn_g[l] = m->attn_g[l]; v.mlp_g[l] = m->mlp_g[l];
        v.Wqkv[l] = m->Wqkv[l]; v.Wo[l] = m->Wo[l]; v.Wi[l] = m->Wi[l]; v.Wo2[l] = m->Wo2[l];
    }
    for (int i = 0; i < 2; ++i) {
        v.n1g[i] = m->n1g[i]; v.n1b[i] = m->n1b[i]; v.n2g[i] = m->n2g[i]; v.n2b[i] = m->n2b[i];
        v.in_full[i] = m->in_full[i]; v.in_q[i] = m->in_q[i]; v.in_kv[i] = m->in_kv[i];
        v.out_p[i] = m->out_p[i]; v.lin1[i] = m->lin1[i]; v.lin2[i] = m->lin2[i];
        v.in_b[i] = m->in_b[i]; v.out_b[i] = m->out_b[i]; v.l1_b[i] = m->l1_b[i]; v.l2_b[i] = m->l2_b[i];
    }
    v.sc_g = m->sc_g; v.sc_b = m->sc_b; v.sc_w1t = m->sc_w1t; v.sc_b1 = m->sc_b1; v.sc_w2 = m->sc_w2;
    v.sc_b2 = m->sc_b2; v.lin_w = m->lin_w; v.lin_b = m->lin_b; v.rope_g = m->rope_g; v.rope_l = m->rope_l;
    for (int l = 0; l < NL; ++l) v.inv8[l] = m->inv8[l];
}

jd_status load_weights(jd_model *m, const char *path) {
    WeightFile wf;
    TRY(open_weights(path, wf));
    const uint32_t d = D;
    TRY(upload_f32(m, wf, "embed.E", {VOCAB, d}, &m->E));
    TRY(upload_f32(m, wf, "embed.norm.g", {d}, &m->emb_g));
    for (int l = 0; l < NL; ++l) {
        const std::string p = "enc." + std::to_string(l) + ".";
        if (l != 0) TRY(upload_f32(m, wf, p + "attn_norm.g", {d}, &m->attn_g[l]));
        TRY(upload_f32(m, wf, p + "mlp_norm.g", {d}, &m->mlp_g[l]));
        if (m->fp8) {  // the QKV input is the embedding norm's output (layer 0) or this layer's attention norm's
            std::vector<float> g, w;
            TRY(read_tensor(wf, l == 0 ? std::string("embed.norm.g") : p + "attn_norm.g", {d}, g));
            const float sa = ln_e4m3_scale(g);
            m->inv8[l] = 1.0f / sa;
            TRY(read_tensor(wf, p + "Wqkv", {(uint32_t)QKV, d}, w));
            TRY(upload_proj_e4m3(m, w, QKV, D, sa, m->Wqkv[l]));
        } else {
            TRY(load_proj(m, wf, p + "Wqkv", QKV, D, 384, m->Wqkv[l]));
        }
        TRY(load_proj(m, wf, p + "Wo", D, D, 384, m->Wo[l]));
        TRY(load_proj(m, wf, p + "Wo2", D, FF, 384, m->Wo2[l]));
        std::vector<float> wi, il((size_t)2 * FF * D);
        TRY(read_tensor(wf, p + "Wi", {2 * FF, d}, wi));
        for (int j = 0; j < FF / 128; ++j) {  // [u_j (128 rows) | g_j (128 rows)]
            memcpy(&il[(size_t)(j * 256) * D], &wi[(size_t)(j * 128) * D], sizeof(float) * 128 * D);
            memcpy(&il[(size_t)(j * 256 + 128) * D], &wi[(size_t)(FF + j * 128) * D], sizeof(float) * 128 * D);
        }
        TRY(upload_proj(m, il, 0, 2 * FF, D, 256, m->Wi[l]));
    }
    TRY(upload_f32(m, wf, "enc.final_norm.g", {d}, &m->fin_g));
    TRY(upload_f32(m, wf, "head.type_table", {3, d}, &m->type_tab));
    for (int i = 0; i < 2; ++i) {
        const std::string p = "head." + std::to_string(i) + ".";
        TRY(upload_f32(m, wf, p + "norm1.g", {d}, &m->n1g[i]));
        TRY(upload_f32(m, wf, p + "norm1.b", {d}, &m->n1b[i]));
        TRY(upload_f32(m, wf, p + "norm2.g", {d}, &m->n2g[i]));
        TRY(upload_f32(m, wf, p + "norm2.b", {d}, &m->n2b[i]));
        std::vector<float> win;
        TRY(read_tensor(wf, p + "in_proj.W", {QKV, d}, win));
        if (i == 0) {
            TRY(upload_proj(m, win, 0, QKV, D, 384, m->in_full[i]));
        } else {
            TRY(upload_proj(m, win, 0, D, D, 384, m->in_q[i]));
            TRY(upload_proj(m, win, D, 2 * D, D, 384, m->in_kv[i]));
        }
        TRY(upload_f32(m, wf, p + "in_proj.b", {QKV}, &m->in_b[i]));
        TRY(load_proj(m, wf, p + "out_proj.W", D, D, 384, m->out_p[i]));
        TRY(upload_f32(m, wf, p + "out_proj.b", {d}, &m->out_b[i]));
        TRY(load_proj(m, wf, p + "linear1.W", HFF, D, 256, m->lin1[i]));
        TRY(upload_f32(m, wf, p + "linear1.b", {HFF}, &m->l1_b[i]));
        TRY(load_proj(m, wf, p + "linear2.W", D, HFF, 384, m->lin2[i]));
        TRY(upload_f32(m, wf, p + "linear2.b", {d}, &m->l2_b[i]));
    }
    TRY(upload_f32(m, wf, "scorer.norm.g", {d}, &m->sc_g));
    TRY(upload_f32(m, wf, "scorer.norm.b", {d}, &m->sc_b));
    {
        std::vector<float> w1, w1t((size_t)D * D);
        TRY(read_tensor(wf, "scorer.linear1.W", {d, d}, w1));
        for (int o = 0; o < D; ++o)
            for (int k = 0; k < D; ++k) w1t[(size_t)k * D + o] = w1[(size_t)o * D + k];
        TRY(m->dalloc(&m->sc_w1t, w1t.size()));
        CK(cudaMemcpy(m->sc_w1t, w1t.data(), w1t.size() * 4, cudaMemcpyHostToDevice));
    }
    TRY(upload_f32(m, wf, "scorer.linear1.b", {d}, &m->sc_b1));
    TRY(upload_f32(m, wf, "scorer.linear2.W", {1, d}, &m->sc_w2));
    TRY(upload_f32(m, wf, "scorer.linear2.b", {1}, &m->sc_b2));
    TRY(upload_f32(m, wf, "scorer_lin.W", {1, d}, &m->lin_w));
    TRY(upload_f32(m, wf, "scorer_lin.b", {1}, &m->lin_b));
    TRY(make_rope_table(m, 160000.0, &m->rope_g));
    TRY(make_rope_table(m, 10000.0, &m->rope_l));
    return JD_OK;
}

jd_status alloc_host_slot(jd_model *m, jd_model::HostSlot &h) {
    const size_t T = m->T_cap, M = m->M_cap, B = m->B_cap;
    TRY(m->halloc(&h.h_tokens, T));
    TRY(m->halloc(&h.h_cu, B + 1));
    TRY(m->halloc(&h.h_mask, M));
    TRY(m->halloc(&h.h_opt, B + 1));
    TRY(m->halloc(&h.h_type, B));
    TRY(m->halloc(&h.h_logits, M));
    TRY(m->halloc(&h.h_probs, M));
    TRY(m->halloc(&h.h_choice, B));
    TRY(m->halloc(&h.h_score, B));
    TRY(m->halloc(&h.h_noul, B));
    TRY(m->halloc(&h.h_maxp, B));
    TRY(m->halloc(&h.h_status, 1));
    CK(cudaEventCreateWithFlags(&h.done, cudaEventDisableTiming));
    return JD_OK;
}

jd_status alloc_workspace(jd_model *m) {
    const size_t T = m->T_cap, M = m->M_cap, B = m->B_cap;
    const size_t es = m->fp32 ? 4 : 2;
    TRY(m->dalloc(&m->x, T * D));
    uint8_t *p = nullptr;
    TRY(m->dalloc(&p, T * D * es)); m->xn = p;
    TRY(m->dalloc(&p, T * QKV * es)); m->qkv = p;
    TRY(m->dalloc(&p, T * D * es)); m->o = p;
    TRY(m->dalloc(&p, T * HFF * es)); m->y = p;
    TRY(m->dalloc(&m->tok_row, T));
    TRY(m->dalloc(&m->pos, T));
    TRY(m->dalloc(&m->qb_off, qb_ints((int)B, (int)T)));
    TRY(m->dalloc(&m->hm, M * D));
    m->mk_part_entries = std::max((int)M, MARKER_PART_ENTRIES_MIN);
    TRY(m->dalloc(&m->mk_part, (size_t)m->mk_part_entries * NH * (DH + 2)));
    TRY(m->dalloc(&p, M * D * es)); m->xm = p;
    TRY(m->dalloc(&p, M * D * es)); m->qm = p;
    TRY(m->dalloc(&p, M * D * es)); m->om = p;
    TRY(m->dalloc(&p, M * D * es)); m->xnm = p;
    TRY(m->dalloc(&p, M * HFF * es)); m->ym = p;
    TRY(m->dalloc(&m->status, 1));
    if (m->fp8) {
        TRY(m->dalloc(&m->xn8, T * D));
        TRY(make_map(&m->tm_xn8, m->xn8, D, T, D, 128, 128, false, false, true));
    }
    TRY(m->dalloc(&m->i_logits, M));
    TRY(m->dalloc(&m->i_probs, M));
    TRY(m->dalloc(&m->i_choice, B));
    TRY(m->dalloc(&m->i_score, B));
    TRY(m->dalloc(&m->i_noul, B));
    TRY(m->dalloc(&m->i_maxp, B));
    TRY(m->dalloc(&m->d_tokens, T));
    TRY(m->dalloc(&m->d_cu, B + 1));
    TRY(m->dalloc(&m->d_mask, M));
    TRY(m->dalloc(&m->d_opt, B + 1));
    TRY(m->dalloc(&m->d_type, B));
    TRY(alloc_host_slot(m, m->hs[0]));
    TRY(m->halloc(&m->h_route, 16));
    if (!m->fp32) {
        TRY(make_map(&m->tm_xn, m->xn, D, T, D, 64, 128));
        TRY(make_map(&m->tm_o, m->o, D, T, D, 64, 128));
        TRY(make_map(&m->tm_y_enc, m->y, FF, T, FF, 64, 128));
        TRY(make_map(&m->tm_y_head, m->y, HFF, T, HFF, 64, 128));
        TRY(make_map(&m->tm_o64, m->o, D, T, D, 32, 128, false, true));
        TRY(make_map(&m->tm_y_enc64, m->y, FF, T, FF, 32, 128, false, true));
        TRY(make_map(&m->tm_y_head64, m->y, HFF, T, HFF, 32, 128, false, true));
        TRY(make_map(&m->tm_qkv, m->qkv, QKV, T, QKV, 64, 64));
        TRY(make_map(&m->tm_xm, m->xm, D, M, D, 64, 128));
        TRY(make_map(&m->tm_om, m->om, D, M, D, 64, 128));
        TRY(make_map(&m->tm_xnm, m->xnm, D, M, D, 64, 128));
        TRY(make_map(&m->tm_ym, m->ym, HFF, M, HFF, 64, 128));
        TRY(make_map(&m->to_qkv, m->qkv, QKV, T, QKV, 64, 32));
        TRY(make_map(&m->tm_x32, m->x, D, T, D, 32, 128, true));
        TRY(make_map(&m->tm_qkv128, m->qkv, QKV, T, QKV, 64, 128));
        TRY(make_map(&m->to_y_enc, m->y, FF, T, FF, 64, 32));
        TRY(make_map(&m->to_y_head, m->y, HFF, T, HFF, 64, 32));
        TRY(make_map(&m->to_qm, m->qm, D, M, D, 64, 32));
        TRY(make_map(&m->to_ym, m->ym, HFF, M, HFF, 64, 32));
    }
    return JD_OK;
}

EpiParams base_ep(jd_model *m, int rows) {
    EpiParams e;
    memset(&e, 0, sizeof(e));
    e.rows = rows;
    e.eps = EPS;
    e.status = m->status;
    e.act = m->cfg.head_act;
    return e;
}

GemmOp make_op(int epi, int bn, const ProjW &w, const CUtensorMap *tmA, const void *A, int lda, const EpiParams &ep,
               const CUtensorMap *tmO = nullptr, const CUtensorMap *tmX = nullptr, const CUtensorMap *tmXN = nullptr,
               const CUtensorMap *tmA64 = nullptr) {
    GemmOp op;
    op.tmO = tmO;
    op.tmX = tmX;
    op.tmXN = tmXN;
    op.tmA64 = tmA64;
    op.tmB64 = tmA64 ? &w.tm64 : nullptr;
    op.tmBs = w.N % 64 == 0 && w.has_tms ? &w.tms : nullptr;  // W box 64 x 64 (split residual, small-batch QKV)
    op.tmBp = tmA64 ? &w.tm : nullptr;  // box 64 x 192 of the 384-wide weights
    op.epi = epi;
    op.bn = bn;
    op.K = w.K;
    op.N = w.N;
    op.tmA = tmA;
    op.tmB = &w.tm;
    op.A32 = static_cast<const float *>(A);
    op.lda = lda;
    op.W32 = static_cast<const float *>(w.w);
    op.ep = ep;
    return op;
}

template <class T>
T *offset(void *p, size_t elems, bool fp32) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(p) + elems * (fp32 ? 4 : 2));
}

#define LK(call)                                                                                  \
    do {                                                                                          \
        cudaError_t e_ = (call);                                                                  \
        if (e_ != cudaSuccess) return fail(JD_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

// Launch with optional per-kernel event timing and a launch count.
#define KL(name, nk, call)                                                     \
    do {                                                                       \
        if (m->prof && m->n_ev < (int)m->ev.size()) {                          \
            LK(cudaEventRecord(m->ev[m->n_ev], st));                           \
            m->ev_name[m->n_ev++] = (name);                                    \
        }                                                                      \
        LK(call);                                                              \
        m->launches += (nk);                                                   \
    } while (0)

// The whole launch sequence (no allocation, no synchronisation).
jd_status enqueue_forward(jd_model *m, const jd_batch *b, const jd_outputs *out, const jd_taps *taps,
                          cudaStream_t st) {
    const bool f32 = m->fp32;
    m->launches = 0;
    m->n_ev = 0;
    const int T = b->n_tokens, B = b->n_rows, M = b->n_markers;
    LK(cudaMemsetAsync(m->status, 0, sizeof(unsigned), st));
    KL("prep", 2, launch_prep(b->cu_seqlens, B, T, m->tok_row, m->pos, m->qb_off, st));
    const bool f8 = m->fp8;
    KL("embed_ln", 1, launch_embed_ln(b->tokens, T, m->E, VOCAB, m->emb_g, EPS, m->x, f8 ? (void *)m->xn8 : m->xn, f32,
                                      m->status, st, f8 ? m->inv8[0] : 0.f));

    AttnArgs aa;
    aa.qkv = m->qkv;
    aa.o = m->o;
    aa.cu_seqlens = b->cu_seqlens;
    aa.qb_off = m->qb_off;
    aa.n_rows = B;
    aa.n_tokens = T;
    aa.tm_qkv = &m->tm_qkv;
    aa.tm_qkv128 = &m->tm_qkv128;
    aa.status = m->status;

    for (int l = 0; l < NL; ++l) {
        const bool glob = (l % 3) == 0;
        EpiParams e = base_ep(m, T);
        e.out = m->qkv;
        e.ldo = QKV;
        e.rope = glob ? m->rope_g : m->rope_l;
        e.pos = m->pos;
        e.rope_cols = 2 * D;
        if (f8) {
            e.col_scale = m->Wqkv[l].col_scale;
            GemmOp op = make_op(EPI_QKV, 384, m->Wqkv[l], &m->tm_xn8, m->xn8, D, e, &m->to_qkv);
            op.tmB = &m->Wqkv[l].tm8;
            op.f8 = true;
            KL("gemm_qkv_rope", 1, launch_gemm(op, false, st));
        } else {
            KL("gemm_qkv_rope", 1, launch_gemm(make_op(EPI_QKV, 384, m->Wqkv[l], &m->tm_xn, m->xn, D, e, &m->to_qkv), f32, st));
        }

        aa.window = glob ? -1 : 64;
        KL(glob ? "attn_global" : "attn_local", 1, launch_attention(aa, f32, st));

        e = base_ep(m, T);
        e.out = m->xn;
        e.ldo = D;
        e.resid = m->x;
        e.ln_g = m->mlp_g[l];
        KL("gemm_wo_res_ln", 1, launch_gemm(make_op(EPI_RESID_LN, 384, m->Wo[l], &m->tm_o, m->o, D, e, nullptr, &m->tm_x32, &m->tm_xn, &m->tm_o64), f32, st));

        e = base_ep(m, T);
        e.out = m->y;
        e.ldo = FF;
        KL("gemm_wi_geglu", 1, launch_gemm(make_op(EPI_GEGLU, 256, m->Wi[l], &m->tm_xn, m->xn, D, e, &m->to_y_enc), f32, st));

        e = base_ep(m, T);
        e.out = m->xn;
        e.ldo = D;
        e.resid = m->x;
        if (l + 1 < NL) {
            e.ln_g = m->attn_g[l + 1];
        } else {
            e.fin_g = m->fin_g;
            e.type_tab = m->type_tab;
            e.tok_row = m->tok_row;
            e.row_type = b->row_type;
            e.tap = taps ? taps->encoder_out : nullptr;
            e.ln_g = m->n1g[0];
            e.ln_b = m->n1b[0];
        }
        GemmOp o2 = make_op(EPI_RESID_LN, 384, m->Wo2[l], &m->tm_y_enc, m->y, FF, e, nullptr, &m->tm_x32, &m->tm_xn,
                            &m->tm_y_enc64);
        if (f8 && l + 1 < NL) {  // the next layer's QKV input, as E4M3
            o2.ep.out = m->xn8;
            o2.ep.out8_inv_scale = m->inv8[l + 1];
            o2.out8 = true;
        }
        KL("gemm_wo2_res_ln", 1, launch_gemm(o2, f32, st));
    }

    // ---- head layer 0 (all tokens)
    {
        EpiParams e = base_ep(m, T);
        e.out = m->qkv;
        e.ldo = QKV;
        e.bias = m->in_b[0];
        KL("head0_gemm_in", 1, launch_gemm(make_op(EPI_QKV, 384, m->in_full[0], &m->tm_xn, m->xn, D, e, &m->to_qkv), f32, st));
        aa.window = -1;
        KL("head0_attn", 1, launch_attention(aa, f32, st));
        e = base_ep(m, T);
        e.out = m->xn;
        e.ldo = D;
        e.bias = m->out_b[0];
        e.resid = m->x;
        e.ln_g = m->n2g[0];
        e.ln_b = m->n2b[0];
        KL("head0_gemm_out", 1, launch_gemm(make_op(EPI_RESID_LN, 384, m->out_p[0], &m->tm_o, m->o, D, e, nullptr, &m->tm_x32, &m->tm_xn, &m->tm_o64), f32, st));
        e = base_ep(m, T);
        e.out = m->y;
        e.ldo = HFF;
        e.bias = m->l1_b[0];
        KL("head0_gemm_ffn1", 1, launch_gemm(make_op(EPI_BIAS_ACT, 256, m->lin1[0], &m->tm_xn, m->xn, D, e, &m->to_y_head), f32, st));
        e = base_ep(m, T);
        e.out = m->xn;
        e.ldo = D;
        e.bias = m->l2_b[0];
        e.resid = m->x;
        e.ln_g = m->n1g[1];
        e.ln_b = m->n1b[1];
        KL("head0_gemm_ffn2", 1, launch_gemm(make_op(EPI_RESID_LN, 384, m->lin2[0], &m->tm_y_head, m->y, HFF, e, nullptr, &m->tm_x32, &m->tm_xn, &m->tm_y_head64), f32, st));
    }
    // ---- head layer 1: keys / values for every token, the rest at the markers only
    {
        EpiParams e = base_ep(m, T);
        e.out = offset<uint8_t>(m->qkv, D, f32);
        e.ldo = QKV;
        e.bias = m->in_b[1] + D;
        e.out_col0 = D;  // keys / values land in columns 384..1151 of qkv
        KL("head1_gemm_kv", 1, launch_gemm(make_op(EPI_QKV, 384, m->in_kv[1], &m->tm_xn, m->xn, D, e, &m->to_qkv), f32, st));
        KL("head1_gather", 1, launch_gather_markers(b->mask_pos, M, T, m->x, m->xn, m->hm, m->xm, f32, m->status, st));
        e = base_ep(m, M);
        e.out = m->qm;
        e.ldo = D;
        e.bias = m->in_b[1];
        KL("head1_gemm_q", 1, launch_gemm(make_op(EPI_QKV, 384, m->in_q[1], &m->tm_xm, m->xm, D, e, &m->to_qm), f32, st));
        KL("head1_marker_attn", marker_attention_splits(M, b->max_row_len, m->mk_part, m->mk_part_entries) > 1 ? 2 : 1,
           launch_marker_attention(m->qm, m->qkv, m->om, b->cu_seqlens, b->opt_off, B, M, b->max_row_len, m->mk_part,
                                   m->mk_part_entries, f32, f32 ? nullptr : &m->to_qm, f32 ? nullptr : &m->tm_qkv,
                                   m->status, st));
        e = base_ep(m, M);
        e.out = m->xnm;
        e.ldo = D;
        e.bias = m->out_b[1];
        e.resid = m->hm;
        e.ln_g = m->n2g[1];
        e.ln_b = m->n2b[1];
        KL("head1_gemm_out", 1, launch_gemm(make_op(EPI_RESID_LN, 384, m->out_p[1], &m->tm_om, m->om, D, e), f32, st));
        e = base_ep(m, M);
        e.out = m->ym;
        e.ldo = HFF;
        e.bias = m->l1_b[1];
        KL("head1_gemm_ffn1", 1, launch_gemm(make_op(EPI_BIAS_ACT, 256, m->lin1[1], &m->tm_xnm, m->xnm, D, e, &m->to_ym), f32, st));
        e = base_ep(m, M);
        e.bias = m->l2_b[1];
        e.resid = m->hm;
        KL("head1_gemm_ffn2", 1, launch_gemm(make_op(EPI_RESID_LN, 384, m->lin2[1], &m->tm_ym, m->ym, HFF, e), f32, st));
    }
    // ---- scorer, softmax and read-outs in one launch
    HeadArgs ha;
    ha.hm = m->hm;
    ha.n_markers = M;
    ha.n_rows = B;
    ha.opt_off = b->opt_off;
    ha.row_type = b->row_type;
    ha.ln_g = m->sc_g;
    ha.ln_b = m->sc_b;
    ha.w1t = m->sc_w1t;
    ha.b1 = m->sc_b1;
    ha.linear = m->cfg.scorer == JD_SCORER_LINEAR;
    ha.w2 = ha.linear ? m->lin_w : m->sc_w2;
    ha.b2 = ha.linear ? m->lin_b : m->sc_b2;
    ha.eps = EPS;
    ha.logits = out->logits;
    ha.probs = out->probs;
    ha.choice = out->choice;
    ha.score = out->score;
    ha.noul = out->noul;
    ha.max_p = out->max_p;
    ha.tap = taps ? taps->marker_state : nullptr;
    ha.status = m->status;
    KL("head", 1, launch_head(ha, st));
    if (m->prof && m->n_ev < (int)m->ev.size()) {
        LK(cudaEventRecord(m->ev[m->n_ev], st));
        m->ev_name[m->n_ev++] = nullptr;
    }
    return JD_OK;
}

// Fold the events of the last profiled call into the per-kernel totals.
jd_status collect_profile(jd_model *m, cudaStream_t st) {
    CK(cudaStreamSynchronize(st));
    for (int i = 0; i + 1 < m->n_ev; ++i) {
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, m->ev[i], m->ev[i + 1]));
        auto &acc = m->prof_acc[m->ev_name[i]];
        acc.first += 1;
        acc.second += ms;
    }
    return JD_OK;
}

jd_status check_batch(jd_model *m, const jd_batch *b) {
    if (!b) return fail(JD_ERR_INVALID_ARG, "batch is NULL");
    if (b->n_rows < 1 || b->n_tokens < 1 || b->n_markers < 1)
        return fail(JD_ERR_INVALID_ARG, "empty batch (rows %d, tokens %d, markers %d)", b->n_rows, b->n_tokens,
                    b->n_markers);
    if (b->n_tokens > m->cfg.max_tokens || b->n_rows > m->cfg.max_rows || b->n_markers > m->cfg.max_markers)
        return fail(JD_ERR_CAPACITY, "batch (%d tokens, %d rows, %d markers) exceeds capacity (%d, %d, %d)",
                    b->n_tokens, b->n_rows, b->n_markers, m->cfg.max_tokens, m->cfg.max_rows, m->cfg.max_markers);
    if (b->max_row_len > MAX_POS) return fail(JD_ERR_INVALID_ARG, "a row is longer than 8192 tokens");
    if (!b->tokens || !b->cu_seqlens || !b->mask_pos || !b->opt_off || !b->row_type)
        return fail(JD_ERR_INVALID_ARG, "batch has a NULL array");
    return JD_OK;
}

// Capture the launch sequence of one call on `st` (a private stream when st is the legacy
// stream, which cannot be captured) and instantiate it.
jd_status capture_forward(jd_model *m, const jd_batch *b, const jd_outputs *out, const jd_taps *taps,
                          cudaStream_t st, cudaGraphExec_t *exec) {
    cudaStream_t cap = st;
    bool own = false;
    if (cap == nullptr) {
        CK(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
        own = true;
    }
    CK(cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal));
    jd_status s = enqueue_forward(m, b, out, taps, cap);
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(cap, &g);
    if (own) cudaStreamDestroy(cap);
    if (s != JD_OK) {
        if (g) cudaGraphDestroy(g);
        return s;
    }
    if (e != cudaSuccess) return fail(JD_ERR_CUDA, "graph capture: %s", cudaGetErrorString(e));
    e = cudaGraphInstantiate(exec, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return fail(JD_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(e));
    ++m->g_captures;
    return JD_OK;
}

constexpr size_t GRAPH_BUCKETS_MAX = 64;

// The bucket of a batch in graph mode: its padded shape (pad_shape) and the longest row of the
// padded batch as the graph sees it.  That is 1024 for batches whose rows all fit in 1024 tokens,
// else the longest row rounded up to a multiple of 1024, so that the marker attention splits the
// keys of every row as it does for the unpadded batch.  False when the padded batch exceeds the
// model's capacity.
bool graph_bucket(const jd_model *m, const jd_batch *b, PadShape *s, int *Lb) {
    *s = pad_shape(b->n_tokens, b->n_rows, b->n_markers);
    const int L = std::max(b->max_row_len, s->Tb - s->T);
    *Lb = L <= 1024 ? 1024 : std::min(MAX_POS, (L + 1023) / 1024 * 1024);
    return s->Tb <= m->T_cap && s->Bb <= m->B_cap && s->Mb <= m->M_cap;
}

// Replay (capturing on first use) the graph of a bucket.  Its batch is the padded one in the
// model's device staging (d_tokens ...), its outputs the model's internal output arrays.
jd_status bucket_replay(jd_model *m, const PadShape &s, int Lb, cudaStream_t st) {
    const std::array<int, 4> key{s.Tb, s.Bb, s.Mb, Lb};
    auto it = m->gbuckets.find(key);
    if (it == m->gbuckets.end()) {
        if (m->gbuckets.size() >= GRAPH_BUCKETS_MAX) {
            auto lru = m->gbuckets.begin();
            for (auto j = m->gbuckets.begin(); j != m->gbuckets.end(); ++j)
                if (j->second.last_use < lru->second.last_use) lru = j;
            cudaGraphExecDestroy(lru->second.exec);
            m->gbuckets.erase(lru);
        }
        jd_batch db{};
        db.n_rows = s.Bb;
        db.n_tokens = s.Tb;
        db.n_markers = s.Mb;
        db.max_row_len = Lb;
        db.tokens = m->d_tokens;
        db.cu_seqlens = m->d_cu;
        db.mask_pos = m->d_mask;
        db.opt_off = m->d_opt;
        db.row_type = m->d_type;
        jd_outputs o{m->i_logits, m->i_probs, m->i_choice, m->i_score, m->i_noul, m->i_maxp};
        jd_model::Bucket bk;
        TRY(capture_forward(m, &db, &o, nullptr, st, &bk.exec));
        bk.launches = m->launches;
        it = m->gbuckets.emplace(key, bk).first;
    } else {
        ++m->g_replays;
    }
    it->second.last_use = ++m->gclock;
    CK(cudaGraphLaunch(it->second.exec, st));
    m->launches = it->second.launches;
    return JD_OK;
}

// Resolves the no-allocation path's static array on `dev` (defined with it below).
jd_status noalloc_prepare(int dev);

}  // namespace

// ================================================================== C ABI

extern "C" jd_status jd_model_create(const jd_model_config *cfg, const char *weights_path, int device,
                                     jd_model **out) {
    clear_error();
    if (!out || !cfg || !weights_path) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    if (cfg->max_tokens < 1 || cfg->max_rows < 1 || cfg->max_markers < 1)
        return fail(JD_ERR_INVALID_ARG, "capacities must be positive");
    if (cfg->precision != JD_PREC_BF16 && cfg->precision != JD_PREC_FP32 && cfg->precision != JD_PREC_FP8)
        return fail(JD_ERR_INVALID_ARG, "unknown precision %d", cfg->precision);
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return fail(JD_ERR_CUDA, "no CUDA device");
    if (device < 0 || device >= ndev) return fail(JD_ERR_INVALID_ARG, "device %d out of range", device);
    CK(cudaSetDevice(device));
    cudaDeviceProp prop;
    CK(cudaGetDeviceProperties(&prop, device));
    if (prop.major != 10) return fail(JD_ERR_CUDA, "this library is built for sm_100a; device is sm_%d%d", prop.major, prop.minor);

    jd_model *m = new jd_model();
    m->cfg = *cfg;
    m->device = device;
    m->fp32 = cfg->precision == JD_PREC_FP32;
    m->fp8 = cfg->precision == JD_PREC_FP8;
    m->T_cap = (cfg->max_tokens + 127) / 128 * 128;
    m->B_cap = cfg->max_rows;
    m->M_cap = (cfg->max_markers + 127) / 128 * 128;
    jd_status s = JD_OK;
    {
        cudaError_t e = init_kernel_attributes();
        if (e != cudaSuccess) s = fail(JD_ERR_CUDA, "kernel attributes: %s", cudaGetErrorString(e));
    }
    if (s == JD_OK) s = load_weights(m, weights_path);
    if (s == JD_OK) s = alloc_workspace(m);
    // BF16 models can serve jd_forward_noalloc: load the module that holds its static array
    // now, at start-up, so that no later call of that entry point allocates.
    if (s == JD_OK && cfg->precision == JD_PREC_BF16) s = noalloc_prepare(device);
    if (s == JD_OK) {
        cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) s = fail(JD_ERR_CUDA, "setup: %s", cudaGetErrorString(e));
    }
    if (s != JD_OK) {
        jd_model_destroy(m);
        return s;
    }
    *out = m;
    return JD_OK;
}

// A second handle on the weights of `base` (their device memory stays owned by base) with a
// workspace, staging buffers and graph cache of its own ("Julia-1 MLX", "Performance": single
// requests served from several threads, each on its own stream).
extern "C" jd_status jd_model_create_shared(const jd_model *base, const jd_model_config *cfg, jd_model **out) {
    clear_error();
    if (!out || !cfg || !base) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    *out = nullptr;
    if (cfg->max_tokens < 1 || cfg->max_rows < 1 || cfg->max_markers < 1)
        return fail(JD_ERR_INVALID_ARG, "capacities must be positive");
    if (cfg->precision != base->cfg.precision) return fail(JD_ERR_INVALID_ARG, "precision differs from the base model's");
    CK(cudaSetDevice(base->device));
    jd_model *m = new jd_model();
    m->cfg = *cfg;
    m->device = base->device;
    m->fp32 = base->fp32;
    m->fp8 = base->fp8;
    m->T_cap = (cfg->max_tokens + 127) / 128 * 128;
    m->B_cap = cfg->max_rows;
    m->M_cap = (cfg->max_markers + 127) / 128 * 128;
    share_weights(*m, base);
    jd_status s = alloc_workspace(m);
    if (s == JD_OK) {
        cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) s = fail(JD_ERR_CUDA, "setup: %s", cudaGetErrorString(e));
    }
    if (s != JD_OK) {
        jd_model_destroy(m);
        return s;
    }
    *out = m;
    return JD_OK;
}

extern "C" void jd_model_destroy(jd_model *m) {
    if (!m) return;
    cudaSetDevice(m->device);
    if (m->gexec) cudaGraphExecDestroy(m->gexec);
    for (auto &h : m->hs)
        if (h.done) cudaEventDestroy(h.done);
    for (auto &kv : m->gbuckets) cudaGraphExecDestroy(kv.second.exec);
    for (cudaEvent_t e : m->ev) cudaEventDestroy(e);
    for (void *p : m->allocs) cudaFree(p);
    if (m->route_buf) cudaFree(m->route_buf);
    for (void *p : m->hallocs) cudaFreeHost(p);
    delete m;
}

extern "C" size_t jd_model_device_bytes(const jd_model *m) { return m ? m->bytes : 0; }

extern "C" jd_status jd_set_graph_mode(jd_model *m, int enable) {
    clear_error();
    if (!m) return fail(JD_ERR_INVALID_ARG, "model is NULL");
    m->graph_mode = enable != 0;
    return JD_OK;
}

extern "C" jd_status jd_graph_stats(const jd_model *m, int64_t *captures, int64_t *replays, int32_t *buckets) {
    clear_error();
    if (!m) return fail(JD_ERR_INVALID_ARG, "model is NULL");
    if (captures) *captures = m->g_captures;
    if (replays) *replays = m->g_replays;
    if (buckets) *buckets = (int32_t)m->gbuckets.size();
    return JD_OK;
}

extern "C" jd_status jd_decide(jd_model *m, const jd_batch *b, const jd_outputs *out, const jd_taps *taps,
                               void *stream) {
    clear_error();
    if (!m || !out) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    TRY(check_batch(m, b));
    if (!out->logits || !out->probs || !out->choice || !out->score || !out->noul || !out->max_p)
        return fail(JD_ERR_INVALID_ARG, "an output pointer is NULL");
    CK(cudaSetDevice(m->device));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    m->last_stream = st;
    if (m->prof) {
        TRY(enqueue_forward(m, b, out, taps, st));
        return collect_profile(m, st);
    }
    if (!m->graph_mode) return enqueue_forward(m, b, out, taps, st);

    PadShape ps;
    int Lb = 0;
    if (!taps && graph_bucket(m, b, &ps, &Lb)) {
        // the padded batch into the model's staging, the bucket's graph, the real rows out
        LK(launch_pad_batch(ps, b->tokens, b->cu_seqlens, b->mask_pos, b->opt_off, b->row_type, m->d_tokens,
                            m->d_cu, m->d_mask, m->d_opt, m->d_type, st));
        TRY(bucket_replay(m, ps, Lb, st));
        LK(launch_unpad_outputs(b->n_markers, b->n_rows, m->i_logits, m->i_probs, m->i_choice, m->i_score,
                                m->i_noul, m->i_maxp, out->logits, out->probs, out->choice, out->score, out->noul,
                                out->max_p, st));
        m->launches += 2;
        return JD_OK;
    }

    std::vector<uintptr_t> key = {(uintptr_t)b->n_tokens,  (uintptr_t)b->n_rows,     (uintptr_t)b->n_markers,
                                  (uintptr_t)b->tokens,    (uintptr_t)b->cu_seqlens, (uintptr_t)b->mask_pos,
                                  (uintptr_t)b->opt_off,   (uintptr_t)b->row_type,   (uintptr_t)out->logits,
                                  (uintptr_t)out->probs,   (uintptr_t)out->choice,   (uintptr_t)out->score,
                                  (uintptr_t)out->noul,    (uintptr_t)out->max_p,
                                  (uintptr_t)b->max_row_len,
                                  (uintptr_t)(taps ? taps->encoder_out : nullptr),
                                  (uintptr_t)(taps ? taps->marker_state : nullptr)};
    if (!m->gexec || key != m->gkey) {
        if (m->gexec) {
            cudaGraphExecDestroy(m->gexec);
            m->gexec = nullptr;
        }
        TRY(capture_forward(m, b, out, taps, st, &m->gexec));
        m->gexec_launches = m->launches;
        m->gkey = key;
    } else {
        ++m->g_replays;
    }
    CK(cudaGraphLaunch(m->gexec, st));
    m->launches = m->gexec_launches;
    return JD_OK;
}

extern "C" jd_status jd_forward(jd_model *m, const jd_batch *b, float *logits, void *stream) {
    clear_error();
    if (!m || !logits) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    TRY(check_batch(m, b));
    jd_outputs o{logits, m->i_probs, m->i_choice, m->i_score, m->i_noul, m->i_maxp};
    return jd_decide(m, b, &o, nullptr, stream);
}

namespace {

// Queue one host batch on `st` through the pinned slot h: copies in, forward pass (a bucket's
// graph in graph mode), outputs and the status word copied back, h.done recorded.
jd_status host_enqueue(jd_model *m, const jd_batch *hb, jd_model::HostSlot &h, cudaStream_t st) {
    const int T = hb->n_tokens, B = hb->n_rows, M = hb->n_markers;
    // graph mode: the batch padded to its bucket on the host, so that its graph reads it from the
    // staging arrays and writes the internal outputs directly
    PadShape ps = pad_shape(T, B, M);
    int Lb = 0;
    const bool bucket = m->graph_mode && !m->prof && graph_bucket(m, hb, &ps, &Lb);
    if (!bucket) ps = PadShape{T, B, M, T, B, M};
    memcpy(h.h_tokens, hb->tokens, sizeof(int) * T);
    memcpy(h.h_cu, hb->cu_seqlens, sizeof(int) * (B + 1));
    memcpy(h.h_mask, hb->mask_pos, sizeof(int) * M);
    memcpy(h.h_opt, hb->opt_off, sizeof(int) * (B + 1));
    memcpy(h.h_type, hb->row_type, sizeof(int) * B);
    for (int i = T; i < ps.Tb; ++i) h.h_tokens[i] = pad_token_at(ps, hb->tokens, i);
    for (int i = B + 1; i <= ps.Bb; ++i) {
        h.h_cu[i] = pad_cu_at(ps, hb->cu_seqlens, i);
        h.h_opt[i] = pad_opt_at(ps, hb->opt_off, i);
    }
    for (int i = M; i < ps.Mb; ++i) h.h_mask[i] = pad_mask_at(ps, hb->mask_pos, i);
    for (int i = B; i < ps.Bb; ++i) h.h_type[i] = pad_type_at(ps, hb->row_type, i);
    CK(cudaMemcpyAsync(m->d_tokens, h.h_tokens, sizeof(int) * ps.Tb, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(m->d_cu, h.h_cu, sizeof(int) * (ps.Bb + 1), cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(m->d_mask, h.h_mask, sizeof(int) * ps.Mb, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(m->d_opt, h.h_opt, sizeof(int) * (ps.Bb + 1), cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(m->d_type, h.h_type, sizeof(int) * ps.Bb, cudaMemcpyHostToDevice, st));
    if (bucket) {
        m->last_stream = st;
        TRY(bucket_replay(m, ps, Lb, st));
    } else {
        jd_batch db = *hb;
        db.tokens = m->d_tokens;
        db.cu_seqlens = m->d_cu;
        db.mask_pos = m->d_mask;
        db.opt_off = m->d_opt;
        db.row_type = m->d_type;
        db.head_len = nullptr;
        db.trunc = nullptr;
        jd_outputs o{m->i_logits, m->i_probs, m->i_choice, m->i_score, m->i_noul, m->i_maxp};
        TRY(jd_decide(m, &db, &o, nullptr, st));
    }
    CK(cudaMemcpyAsync(h.h_logits, m->i_logits, sizeof(float) * M, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(h.h_probs, m->i_probs, sizeof(float) * M, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(h.h_choice, m->i_choice, sizeof(int) * B, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(h.h_score, m->i_score, sizeof(float) * B, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(h.h_noul, m->i_noul, sizeof(float) * B, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(h.h_maxp, m->i_maxp, sizeof(float) * B, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(h.h_status, m->status, sizeof(unsigned), cudaMemcpyDeviceToHost, st));
    CK(cudaEventRecord(h.done, st));
    h.B = B;
    h.M = M;
    return JD_OK;
}

// Wait for slot h's call and copy its outputs out (its own copy of the status word decides).
jd_status host_finish(jd_model::HostSlot &h, jd_host_outputs *ho) {
    CK(cudaEventSynchronize(h.done));
    const int B = h.B, M = h.M;
    if (*h.h_status)
        return fail(JD_ERR_DEVICE_STATUS, "device status 0x%x (1: wait timeout, 2: token id range, 4: index)",
                    *h.h_status);
    if (ho->logits) memcpy(ho->logits, h.h_logits, sizeof(float) * M);
    if (ho->probs) memcpy(ho->probs, h.h_probs, sizeof(float) * M);
    if (ho->choice) memcpy(ho->choice, h.h_choice, sizeof(int) * B);
    if (ho->score) memcpy(ho->score, h.h_score, sizeof(float) * B);
    if (ho->noul) memcpy(ho->noul, h.h_noul, sizeof(float) * B);
    if (ho->max_p) memcpy(ho->max_p, h.h_maxp, sizeof(float) * B);
    ho->n_rows = B;
    ho->n_markers = M;
    return JD_OK;
}

}  // namespace

extern "C" jd_status jd_decide_packed_host(jd_model *m, const jd_batch *hb, jd_host_outputs *ho, void *stream) {
    clear_error();
    if (!m || !hb || !ho) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    TRY(check_batch(m, hb));
    if (m->submitted != m->collected)
        return fail(JD_ERR_INVALID_ARG, "collect the submitted calls (jd_decide_host_collect) first");
    CK(cudaSetDevice(m->device));
    TRY(host_enqueue(m, hb, m->hs[0], static_cast<cudaStream_t>(stream)));
    return host_finish(m->hs[0], ho);
}

extern "C" jd_status jd_decide_host_submit(jd_model *m, const jd_row *rows, int32_t n_rows, const jd_encode_opts *opts,
                                           void *stream, int64_t *ticket) {
    clear_error();
    if (!m || !ticket) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (m->submitted - m->collected >= 2)
        return fail(JD_ERR_INVALID_ARG, "two calls in flight: collect one (jd_decide_host_collect) first");
    CK(cudaSetDevice(m->device));
    jd_model::HostSlot &h = m->hs[m->submitted % 2];
    if (!h.h_tokens) TRY(alloc_host_slot(m, h));
    jd_batch *hb = nullptr;
    int32_t bad = -1;
    jd_status s = jd_serialize(rows, n_rows, opts, &hb, &bad);
    if (s != JD_OK) return s;
    s = check_batch(m, hb);
    if (s == JD_OK) s = host_enqueue(m, hb, h, static_cast<cudaStream_t>(stream));
    jd_batch_free(hb);
    if (s != JD_OK) return s;
    *ticket = m->submitted++;
    return JD_OK;
}

extern "C" jd_status jd_decide_host_collect(jd_model *m, int64_t ticket, jd_host_outputs *ho) {
    clear_error();
    if (!m || !ho) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (ticket != m->collected || m->collected >= m->submitted)
        return fail(JD_ERR_INVALID_ARG, "ticket %lld is not the oldest call in flight", (long long)ticket);
    CK(cudaSetDevice(m->device));
    jd_status s = host_finish(m->hs[ticket % 2], ho);
    ++m->collected;  // a failed call is collected too: its slot is free again
    return s;
}

extern "C" jd_status jd_decide_host(jd_model *m, const jd_row *rows, int32_t n_rows, const jd_encode_opts *opts,
                                    jd_host_outputs *ho, void *stream) {
    jd_batch *hb = nullptr;
    int32_t bad = -1;
    jd_status s = jd_serialize(rows, n_rows, opts, &hb, &bad);
    if (s != JD_OK) return s;
    s = jd_decide_packed_host(m, hb, ho, stream);
    jd_batch_free(hb);
    return s;
}

// ================================================================== router rounds on the device
//
// The same tournament as jd_route_host with the candidates, the rows of every round and the
// survivor rule on the device: the requests are uploaded once; per round the host reads back
// four counters (rows, tokens, markers, longest row) to size the forward pass's launches, and
// nothing else crosses until the final outputs.

namespace {

struct RouteLayout {
    size_t off[16] = {};
    size_t bytes = 0;
    size_t add(size_t n) {
        const size_t o = bytes;
        bytes += (n + 63) / 64 * 64;  // 64-byte aligned pieces
        return o;
    }
};

}  // namespace

extern "C" jd_status jd_route_device(jd_model *m, const jd_route_request *reqs, int32_t n_requests,
                                     const jd_encode_opts *opts, jd_route_outputs *out, void *stream) {
    clear_error();
    if (!m || !opts || !out || (n_requests > 0 && !reqs) || n_requests < 0)
        return fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (n_requests > 0 && !out->winner) return fail(JD_ERR_INVALID_ARG, "out->winner is NULL");
    if (out->rows_per_round && out->max_rounds < 0) return fail(JD_ERR_INVALID_ARG, "max_rounds < 0");
    if (opts->max_length < 1 || opts->max_length > MAX_POS || opts->head_budget < 1 || opts->vocab < 1)
        return fail(JD_ERR_INVALID_ARG, "max_length must be in [1, 8192] and head_budget >= 1");
    auto in_vocab = [&](const int32_t *p, int n) {
        for (int i = 0; i < n; ++i)
            if (p[i] < 0 || p[i] >= opts->vocab) return false;
        return true;
    };
    const int32_t special[3] = {opts->bos, opts->eos, opts->mask};
    if (!in_vocab(special, 3)) return fail(JD_ERR_TOKEN_RANGE, "bos/eos/mask id outside [0, %d)", opts->vocab);
    out->n_rounds = 0;
    if (n_requests == 0) return JD_OK;

    // the request pool: req[6] per request, lab[2] per label, then every id
    std::vector<int32_t> req((size_t)n_requests * 6), lab, ids;
    for (int r = 0; r < n_requests; ++r) {
        const jd_route_request &q = reqs[r];
        if (q.n_labels < 1 || q.n_labels > 4096 || !q.labels || !q.n_label_ids)
            return fail(JD_ERR_INVALID_ARG, "request %d: 1..4096 labels required", r);
        if (q.n_question < 0 || q.n_state < 0 || (q.n_question && !q.question) || (q.n_state && !q.state))
            return fail(JD_ERR_INVALID_ARG, "request %d has a null array or a negative length", r);
        if (!in_vocab(q.question, q.n_question) || !in_vocab(q.state, q.n_state))
            return fail(JD_ERR_TOKEN_RANGE, "request %d: token id outside [0, %d)", r, opts->vocab);
        int32_t *rq = req.data() + (size_t)r * 6;
        rq[0] = (int32_t)ids.size();
        rq[1] = q.n_question;
        ids.insert(ids.end(), q.question, q.question + q.n_question);
        rq[2] = (int32_t)ids.size();
        rq[3] = q.n_state;
        ids.insert(ids.end(), q.state, q.state + q.n_state);
        rq[4] = (int32_t)(lab.size() / 2);
        rq[5] = q.n_labels;
        for (int i = 0; i < q.n_labels; ++i) {
            const int n = q.n_label_ids[i];
            if (n < 0 || (n && !q.labels[i])) return fail(JD_ERR_INVALID_ARG, "request %d label %d is invalid", r, i);
            if (!in_vocab(q.labels[i], n))
                return fail(JD_ERR_TOKEN_RANGE, "request %d label %d: token id outside [0, %d)", r, i, opts->vocab);
            lab.push_back((int32_t)ids.size());
            lab.push_back(n);
            ids.insert(ids.end(), q.labels[i], q.labels[i] + n);
        }
        if (ids.size() > 0x7fffffffu) return fail(JD_ERR_INVALID_ARG, "requests too large");
    }
    const size_t n_req = (size_t)n_requests, n_lab = lab.size() / 2;
    const int bound = (int)std::max(n_lab / 2, n_req) + 1;  // rows of any round: two candidates or more each

    RouteLayout ly;
    const size_t o_pool = ly.add((req.size() + lab.size() + ids.size()) * 4);
    const size_t o_cand0 = ly.add(n_lab * 4), o_cand1 = ly.add(n_lab * 4);
    const size_t o_nc0 = ly.add(n_req * 4), o_nc1 = ly.add(n_req * 4);
    const size_t o_rowoff = ly.add((n_req + 1) * 4), o_desc = ly.add((size_t)bound * 12);
    const size_t o_plan = ly.add((size_t)bound * sizeof(RoutePlan));
    const size_t o_cu = ly.add(((size_t)bound + 1) * 4), o_opt = ly.add(((size_t)bound + 1) * 4);
    const size_t o_cnt = ly.add(RC_COUNT * 4);
    const size_t o_win = ly.add(n_req * 4), o_winp = ly.add(n_req * 4);
    const size_t o_finc = ly.add(n_req * 20 * 4), o_finp = ly.add(n_req * 20 * 4);
    CK(cudaSetDevice(m->device));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    m->last_stream = st;
    if (ly.bytes > m->route_bytes) {
        CK(cudaStreamSynchronize(st));
        if (m->route_buf) cudaFree(m->route_buf);
        m->route_buf = nullptr;
        m->route_bytes = 0;
        void *p = nullptr;
        cudaError_t e = cudaMalloc(&p, ly.bytes);
        if (e != cudaSuccess) return fail(JD_ERR_CUDA, "router workspace (%zu bytes): %s", ly.bytes, cudaGetErrorString(e));
        m->route_buf = p;
        m->route_bytes = ly.bytes;
    }
    uint8_t *base = static_cast<uint8_t *>(m->route_buf);
    auto I = [&](size_t o) { return reinterpret_cast<int *>(base + o); };
    std::vector<int32_t> pool;
    pool.reserve(req.size() + lab.size() + ids.size());
    pool.insert(pool.end(), req.begin(), req.end());
    pool.insert(pool.end(), lab.begin(), lab.end());
    pool.insert(pool.end(), ids.begin(), ids.end());
    CK(cudaMemcpyAsync(base + o_pool, pool.data(), pool.size() * 4, cudaMemcpyHostToDevice, st));

    RouteArgs a;
    a.n_req = n_requests;
    a.req = I(o_pool);
    a.lab = a.req + req.size();
    a.ids = a.lab + lab.size();
    a.strict = opts->strict != 0;
    a.head_budget = opts->head_budget;
    a.max_length = opts->max_length;
    a.bos = opts->bos;
    a.eos = opts->eos;
    a.mask = opts->mask;
    int *cand[2] = {I(o_cand0), I(o_cand1)}, *nc[2] = {I(o_nc0), I(o_nc1)};
    int *cnt = I(o_cnt), *cu = I(o_cu), *opt = I(o_opt), *row_off = I(o_rowoff), *desc = I(o_desc);
    RoutePlan *plan = reinterpret_cast<RoutePlan *>(base + o_plan);
    LK(launch_route_init(a, cand[0], nc[0], st));

    int cur = 0, round = 0;
    bool final_round = false;
    for (;;) {
        LK(cudaMemsetAsync(cnt, 0, RC_COUNT * 4, st));
        LK(launch_route_plan_round(a, cand[cur], nc[cur], final_round ? 1 : 0, bound, row_off, desc, plan, cu, opt,
                                   cnt, st));
        CK(cudaMemcpyAsync(m->h_route, cnt, RC_COUNT * 4, cudaMemcpyDeviceToHost, st));
        CK(cudaMemcpyAsync(m->h_route + RC_COUNT, m->status, 4, cudaMemcpyDeviceToHost, st));
        CK(cudaStreamSynchronize(st));
        const int B = m->h_route[RC_ROWS], T = m->h_route[RC_TOKENS], M = m->h_route[RC_MARKERS];
        const int L = m->h_route[RC_LONGEST], err = m->h_route[RC_ERR];
        if (m->h_route[RC_COUNT])
            return fail(JD_ERR_DEVICE_STATUS, "device status 0x%x (1: wait timeout, 2: token id range, 4: index)",
                        (unsigned)m->h_route[RC_COUNT]);
        if (err & RE_OPTION_48) return fail(JD_ERR_OVERFLOW, "round %d: an option is longer than 48 tokens", round + 1);
        if (err & RE_HEAD_BUDGET)
            return fail(JD_ERR_OVERFLOW, "round %d: question plus options over the head budget %d", round + 1,
                        opts->head_budget);
        if (err & RE_MAX_LENGTH) return fail(JD_ERR_OVERFLOW, "round %d: a row is longer than max_length", round + 1);
        if (B == 0 && !final_round) {
            final_round = true;
            continue;
        }
        if (B > 0) {
            if (T > m->cfg.max_tokens || B > m->cfg.max_rows || M > m->cfg.max_markers || L > MAX_POS)
                return fail(JD_ERR_CAPACITY, "round %d (%d tokens, %d rows, %d markers) exceeds the capacity (%d, %d, %d)",
                            round + 1, T, B, M, m->cfg.max_tokens, m->cfg.max_rows, m->cfg.max_markers);
            LK(launch_route_write(a, cand[cur], desc, plan, cu, opt, B, m->d_tokens, m->d_mask, m->d_type, st));
            jd_batch db{};
            db.n_rows = B;
            db.n_tokens = T;
            db.n_markers = M;
            db.max_row_len = L;
            db.tokens = m->d_tokens;
            db.cu_seqlens = cu;
            db.mask_pos = m->d_mask;
            db.opt_off = opt;
            db.row_type = m->d_type;
            jd_outputs o{m->i_logits, m->i_probs, m->i_choice, m->i_score, m->i_noul, m->i_maxp};
            TRY(enqueue_forward(m, &db, &o, nullptr, st));
            if (out->rows_per_round && round < out->max_rounds) out->rows_per_round[round] = B;
            ++round;
        }
        if (final_round) break;
        LK(launch_route_survive(a, cand[cur], nc[cur], cand[cur ^ 1], nc[cur ^ 1], row_off, opt, m->i_probs, st));
        cur ^= 1;
    }
    LK(launch_route_final(a, cand[cur], nc[cur], row_off, opt, m->i_probs, I(o_win),
                          reinterpret_cast<float *>(base + o_winp), I(o_finc), reinterpret_cast<float *>(base + o_finp),
                          st));
    std::vector<int32_t> win(n_req), finc(n_req * 20);
    std::vector<float> winp(n_req), finp(n_req * 20);
    CK(cudaMemcpyAsync(win.data(), base + o_win, n_req * 4, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(winp.data(), base + o_winp, n_req * 4, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(finc.data(), base + o_finc, n_req * 80, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(finp.data(), base + o_finp, n_req * 80, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(m->h_route + RC_COUNT, m->status, 4, cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    if (m->h_route[RC_COUNT])
        return fail(JD_ERR_DEVICE_STATUS, "device status 0x%x (1: wait timeout, 2: token id range, 4: index)",
                    (unsigned)m->h_route[RC_COUNT]);
    std::copy(win.begin(), win.end(), out->winner);
    if (out->winner_p) std::copy(winp.begin(), winp.end(), out->winner_p);
    if (out->final_candidates) std::copy(finc.begin(), finc.end(), out->final_candidates);
    if (out->final_probs) std::copy(finp.begin(), finp.end(), out->final_probs);
    out->n_rounds = round;
    return JD_OK;
}

extern "C" jd_status jd_check_status(jd_model *m) {
    clear_error();
    if (!m) return fail(JD_ERR_INVALID_ARG, "model is NULL");
    CK(cudaSetDevice(m->device));
    CK(cudaStreamSynchronize(m->last_stream));
    unsigned stv = 0;
    CK(cudaMemcpy(&stv, m->status, sizeof(unsigned), cudaMemcpyDeviceToHost));
    if (stv) return fail(JD_ERR_DEVICE_STATUS, "device status 0x%x (1: wait timeout, 2: token id range, 4: index)", stv);
    return JD_OK;
}

extern "C" int32_t jd_last_launch_count(const jd_model *m) { return m ? m->launches : 0; }

extern "C" jd_status jd_set_profiling(jd_model *m, int enable) {
    clear_error();
    if (!m) return fail(JD_ERR_INVALID_ARG, "model is NULL");
    CK(cudaSetDevice(m->device));
    if (enable && m->ev.empty()) {
        m->ev.resize(192);
        m->ev_name.resize(192);
        for (auto &e : m->ev) CK(cudaEventCreate(&e));
    }
    m->prof = enable != 0;
    m->prof_acc.clear();
    return JD_OK;
}

extern "C" jd_status jd_profile_report(jd_model *m, char *buf, size_t n) {
    clear_error();
    if (!m || !buf || n == 0) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    std::string s;
    char line[160];
    for (auto &kv : m->prof_acc) {
        snprintf(line, sizeof(line), "%s %ld %.6f\n", kv.first.c_str(), kv.second.first, kv.second.second);
        s += line;
    }
    if (s.size() + 1 > n) return fail(JD_ERR_INVALID_ARG, "buffer too small (%zu bytes needed)", s.size() + 1);
    memcpy(buf, s.c_str(), s.size() + 1);
    return JD_OK;
}

// ================================================================== forward without allocation
//
// For callers that cannot allocate device memory once they are running: for
// example a serving loop that must stay inside a fixed memory budget after
// start-up, or a host that hands this library a device but forbids it from
// calling the CUDA allocator.  Such a caller creates its jd_model at start-up
// and then calls jd_forward_noalloc, which keeps every intermediate of the
// forward pass in one file-scope __device__ array instead of the model's
// workspace.  The launch sequence is the one jd_forward uses.

namespace {

constexpr int NA_TOKENS = 1024;   // largest batch (packed tokens) the array holds
constexpr int NA_ROWS = 32;
constexpr int NA_MARKERS = 128;
constexpr int NA_MAX_DEVICES = 64;

constexpr size_t na_up(size_t b) { return (b + 255) / 256 * 256; }
// byte offsets of the workspace inside the array (BF16 activations)
constexpr size_t NA_X = 0;
constexpr size_t NA_XN = NA_X + na_up((size_t)NA_TOKENS * D * 4);
constexpr size_t NA_QKV = NA_XN + na_up((size_t)NA_TOKENS * D * 2);
constexpr size_t NA_O = NA_QKV + na_up((size_t)NA_TOKENS * QKV * 2);
constexpr size_t NA_Y = NA_O + na_up((size_t)NA_TOKENS * D * 2);
constexpr size_t NA_TOKROW = NA_Y + na_up((size_t)NA_TOKENS * HFF * 2);
constexpr size_t NA_POS = NA_TOKROW + na_up((size_t)NA_TOKENS * 4);
constexpr size_t NA_QBOFF = NA_POS + na_up((size_t)NA_TOKENS * 4);
constexpr size_t NA_HM = NA_QBOFF + na_up(qb_ints(NA_ROWS, NA_TOKENS) * 4);
constexpr size_t NA_XM = NA_HM + na_up((size_t)NA_MARKERS * D * 4);
constexpr size_t NA_QM = NA_XM + na_up((size_t)NA_MARKERS * D * 2);
constexpr size_t NA_OM = NA_QM + na_up((size_t)NA_MARKERS * D * 2);
constexpr size_t NA_XNM = NA_OM + na_up((size_t)NA_MARKERS * D * 2);
constexpr size_t NA_YM = NA_XNM + na_up((size_t)NA_MARKERS * D * 2);
constexpr size_t NA_STATUS = NA_YM + na_up((size_t)NA_MARKERS * HFF * 2);
constexpr size_t NA_PROBS = NA_STATUS + 256;
constexpr size_t NA_CHOICE = NA_PROBS + na_up((size_t)NA_MARKERS * 4);
constexpr size_t NA_SCORE = NA_CHOICE + na_up((size_t)NA_ROWS * 4);
constexpr size_t NA_NOUL = NA_SCORE + na_up((size_t)NA_ROWS * 4);
constexpr size_t NA_MAXP = NA_NOUL + na_up((size_t)NA_ROWS * 4);
constexpr size_t NA_BYTES = NA_MAXP + na_up((size_t)NA_ROWS * 4);  // about 9.7 MB

// Held by every GPU that loads the library, until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NA_BYTES];

struct NoAllocSlot {
    bool ready = false;
    uint8_t *base = nullptr;  // device address of g_noalloc_scratch on this device
    CUtensorMap tm_xn{}, tm_o{}, tm_y_enc{}, tm_y_head{}, tm_qkv{}, tm_xm{}, tm_om{}, tm_xnm{}, tm_ym{};
    CUtensorMap tm_o64{}, tm_y_enc64{}, tm_y_head64{};  // residual GEMM A operands: box 32 x 128, 64-byte swizzle
    CUtensorMap to_qkv{}, to_y_enc{}, to_y_head{}, to_qm{}, to_ym{};
    CUtensorMap tm_x32{};  // FP32 residual stream, box 32 x 128
    CUtensorMap tm_qkv128{};
};
NoAllocSlot g_na_slot[NA_MAX_DEVICES];
std::mutex g_na_mutex;
jd_model g_na_view[NA_MAX_DEVICES];  // per-device view: the caller's weights + the array's workspace

// Once per device, with that device current: resolve the array's device
// address (a host-side reference to the symbol is not a device pointer) and
// describe its buffers for TMA.
jd_status noalloc_setup(int dev) {
    NoAllocSlot &s = g_na_slot[dev];
    if (s.ready) return JD_OK;
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return fail(JD_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    s.base = static_cast<uint8_t *>(p);
    TRY(make_map(&s.tm_xn, s.base + NA_XN, D, NA_TOKENS, D, 64, 128));
    TRY(make_map(&s.tm_o, s.base + NA_O, D, NA_TOKENS, D, 64, 128));
    TRY(make_map(&s.tm_y_enc, s.base + NA_Y, FF, NA_TOKENS, FF, 64, 128));
    TRY(make_map(&s.tm_y_head, s.base + NA_Y, HFF, NA_TOKENS, HFF, 64, 128));
    TRY(make_map(&s.tm_o64, s.base + NA_O, D, NA_TOKENS, D, 32, 128, false, true));
    TRY(make_map(&s.tm_y_enc64, s.base + NA_Y, FF, NA_TOKENS, FF, 32, 128, false, true));
    TRY(make_map(&s.tm_y_head64, s.base + NA_Y, HFF, NA_TOKENS, HFF, 32, 128, false, true));
    TRY(make_map(&s.tm_qkv, s.base + NA_QKV, QKV, NA_TOKENS, QKV, 64, 64));
    TRY(make_map(&s.tm_xm, s.base + NA_XM, D, NA_MARKERS, D, 64, 128));
    TRY(make_map(&s.tm_om, s.base + NA_OM, D, NA_MARKERS, D, 64, 128));
    TRY(make_map(&s.tm_xnm, s.base + NA_XNM, D, NA_MARKERS, D, 64, 128));
    TRY(make_map(&s.tm_ym, s.base + NA_YM, HFF, NA_MARKERS, HFF, 64, 128));
    TRY(make_map(&s.to_qkv, s.base + NA_QKV, QKV, NA_TOKENS, QKV, 64, 32));
    TRY(make_map(&s.tm_x32, s.base + NA_X, D, NA_TOKENS, D, 32, 128, true));
    TRY(make_map(&s.tm_qkv128, s.base + NA_QKV, QKV, NA_TOKENS, QKV, 64, 128));
    TRY(make_map(&s.to_y_enc, s.base + NA_Y, FF, NA_TOKENS, FF, 64, 32));
    TRY(make_map(&s.to_y_head, s.base + NA_Y, HFF, NA_TOKENS, HFF, 64, 32));
    TRY(make_map(&s.to_qm, s.base + NA_QM, D, NA_MARKERS, D, 64, 32));
    TRY(make_map(&s.to_ym, s.base + NA_YM, HFF, NA_MARKERS, HFF, 64, 32));
    s.ready = true;
    return JD_OK;
}

// Point the device's view at the caller's weights and at the array's buffers
// (plain field copies; nothing is allocated).
void noalloc_view(jd_model &v, const jd_model *m, const NoAllocSlot &s) {
    v.cfg = m->cfg;
    v.device = m->device;
    v.fp32 = false;
    v.fp8 = false;
    share_weights(v, m);
    uint8_t *b = s.base;
    v.x = reinterpret_cast<float *>(b + NA_X);
    v.xn = b + NA_XN; v.qkv = b + NA_QKV; v.o = b + NA_O; v.y = b + NA_Y;
    v.tok_row = reinterpret_cast<int *>(b + NA_TOKROW);
    v.pos = reinterpret_cast<int *>(b + NA_POS);
    v.qb_off = reinterpret_cast<int *>(b + NA_QBOFF);
    v.hm = reinterpret_cast<float *>(b + NA_HM);
    v.xm = b + NA_XM; v.qm = b + NA_QM; v.om = b + NA_OM; v.xnm = b + NA_XNM; v.ym = b + NA_YM;
    v.status = reinterpret_cast<unsigned *>(b + NA_STATUS);
    v.tm_xn = s.tm_xn; v.tm_o = s.tm_o; v.tm_y_enc = s.tm_y_enc; v.tm_y_head = s.tm_y_head; v.tm_qkv = s.tm_qkv;
    v.tm_o64 = s.tm_o64; v.tm_y_enc64 = s.tm_y_enc64; v.tm_y_head64 = s.tm_y_head64;
    v.tm_xm = s.tm_xm; v.tm_om = s.tm_om; v.tm_xnm = s.tm_xnm; v.tm_ym = s.tm_ym;
    v.to_qkv = s.to_qkv; v.to_y_enc = s.to_y_enc; v.to_y_head = s.to_y_head; v.to_qm = s.to_qm; v.to_ym = s.to_ym;
    v.tm_x32 = s.tm_x32;
    v.tm_qkv128 = s.tm_qkv128;
    v.prof = false;
    v.graph_mode = false;
}

jd_status noalloc_prepare(int dev) {
    if (dev < 0 || dev >= NA_MAX_DEVICES) return JD_OK;  // jd_forward_noalloc refuses such devices
    std::lock_guard<std::mutex> lock(g_na_mutex);
    return noalloc_setup(dev);
}

}  // namespace

extern "C" jd_status jd_forward_noalloc(jd_model *m, const jd_batch *b, float *logits, void *stream) {
    clear_error();
    if (!m || !b || !logits) return fail(JD_ERR_INVALID_ARG, "NULL argument");
    if (m->cfg.precision != JD_PREC_BF16) return fail(JD_ERR_INVALID_ARG, "jd_forward_noalloc serves BF16 models only");
    if (m->device < 0 || m->device >= NA_MAX_DEVICES) return fail(JD_ERR_INVALID_ARG, "device ordinal too large");
    if (b->n_rows < 1 || b->n_tokens < 1 || b->n_markers < 1) return fail(JD_ERR_INVALID_ARG, "empty batch");
    if (b->n_tokens > NA_TOKENS || b->n_rows > NA_ROWS || b->n_markers > NA_MARKERS)
        return fail(JD_ERR_CAPACITY,
                    "jd_forward_noalloc takes at most %d tokens, %d rows and %d markers (got %d, %d, %d)",
                    NA_TOKENS, NA_ROWS, NA_MARKERS, b->n_tokens, b->n_rows, b->n_markers);
    if (!b->tokens || !b->cu_seqlens || !b->mask_pos || !b->opt_off || !b->row_type)
        return fail(JD_ERR_INVALID_ARG, "batch has a NULL array");
    CK(cudaSetDevice(m->device));
    std::lock_guard<std::mutex> lock(g_na_mutex);
    TRY(noalloc_setup(m->device));
    jd_model &v = g_na_view[m->device];
    noalloc_view(v, m, g_na_slot[m->device]);
    uint8_t *base = g_na_slot[m->device].base;
    jd_outputs o{logits, reinterpret_cast<float *>(base + NA_PROBS), reinterpret_cast<int *>(base + NA_CHOICE),
                 reinterpret_cast<float *>(base + NA_SCORE), reinterpret_cast<float *>(base + NA_NOUL),
                 reinterpret_cast<float *>(base + NA_MAXP)};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return enqueue_forward(&v, b, &o, nullptr, st);
}

extern "C" jd_status jd_noalloc_check_status(jd_model *m, void *stream) {
    clear_error();
    if (!m) return fail(JD_ERR_INVALID_ARG, "model is NULL");
    if (m->cfg.precision != JD_PREC_BF16) return fail(JD_ERR_INVALID_ARG, "jd_forward_noalloc serves BF16 models only");
    if (m->device < 0 || m->device >= NA_MAX_DEVICES) return fail(JD_ERR_INVALID_ARG, "device ordinal too large");
    CK(cudaSetDevice(m->device));
    uint8_t *base = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_na_mutex);
        TRY(noalloc_setup(m->device));
        base = g_na_slot[m->device].base;
    }
    CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    unsigned stv = 0;
    CK(cudaMemcpy(&stv, base + NA_STATUS, sizeof(unsigned), cudaMemcpyDeviceToHost));
    if (stv)
        return fail(JD_ERR_DEVICE_STATUS, "jd_forward_noalloc device status 0x%x (1: wait timeout, 2: token id range, 4: index)",
                    stv);
    return JD_OK;
}
