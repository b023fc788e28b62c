// The decision head after the last head layer, in one launch: gather of the
// marker states -> LayerNorm -> scorer -> per-question softmax -> read-outs.
//
// "Julia-1: one score per mask token", "The decision head", step 4: each
// option's logit is LayerNorm -> Linear(384, 384) -> GELU -> Linear(384, 1)
// of the hidden state at its <mask> marker (the single-Linear variant,
// LayerNorm -> Linear(384, 1), is a model option).  "Three modes through one
// head": a softmax across the question's options at temperature 1; choice =
// argmax (lowest index on ties), score = sum_i i p_i, noul = p(true) = p_1 for
// noul rows (NaN otherwise), and the largest probability.  FP32 throughout.
//
// A cluster of eight CTAs takes a run of consecutive rows (the launch picks
// the run length so that about one wave of clusters covers the batch; a batch
// of a few rows gets one row per cluster).  CTA r owns the 48 hidden units
// [48 r, 48 r + 48) and keeps their W1 columns in registers (twelve warps, four
// units each, every lane twelve of the 384 inputs).  The rows' markers stream
// through shared memory eight at a time: the CTA's warps normalize them, each
// warp forms its 4 x 8 dot products (lanes split the 384-long sums; a
// butterfly transpose-reduce leaves each lane one (unit, marker) sum), applies
// bias, GELU and output weight, and sums its four units per marker; the
// twelve warps' sums are added in warp order and sent to CTA 0 through
// distributed shared memory.  CTA 0 adds the eight partial logits of each
// marker in rank order, writes the logits and runs the read-outs, one warp per
// row.  Every sum has a fixed order, so the results do not depend on
// scheduling.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace jd {

namespace {
constexpr int HD_CLUSTER = 8;                  // CTAs per cluster
constexpr int HD_UNITS = D / HD_CLUSTER;       // hidden units per CTA (48)
constexpr int HD_WARPS = HD_UNITS / 4;         // one quad of units per warp (12)
constexpr int HD_THREADS = HD_WARPS * 32;
constexpr int HD_MAX_ROWS = 64;                // rows per cluster at most
constexpr int HD_MAXM = HD_MAX_ROWS * 20;      // markers per cluster (2..20 options per row)
constexpr int HD_TARGET_CLUSTERS = 18;         // about one wave of eight-CTA clusters on 148 SMs
// shared memory: one chunk of normalized states [8][D], warp sums [HD_WARPS][8],
// partial logits [HD_CLUSTER][HD_MAXM], logits [HD_MAXM]
constexpr int HD_OFF_W = 8 * D * 4;
constexpr int HD_OFF_P = HD_OFF_W + HD_WARPS * 8 * 4;
constexpr int HD_OFF_Z = HD_OFF_P + HD_CLUSTER * HD_MAXM * 4;
constexpr int HD_SMEM = HD_OFF_Z + HD_MAXM * 4;

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Store v at the shared-memory address of `local` in CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_f32(const void *local, uint32_t rank, float v) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}
}  // namespace

__global__ void __cluster_dims__(HD_CLUSTER, 1, 1) __launch_bounds__(HD_THREADS) k_head(HeadArgs a, int rows_per_cluster) {
    extern __shared__ __align__(16) uint8_t hsm[];
    float *sn = reinterpret_cast<float *>(hsm);             // [8][D] normalized states of the chunk
    float *sw = reinterpret_cast<float *>(hsm + HD_OFF_W);  // [HD_WARPS][8] per-warp sums
    float *sp = reinterpret_cast<float *>(hsm + HD_OFF_P);  // [HD_CLUSTER][HD_MAXM] partial logits
    float *sz = reinterpret_cast<float *>(hsm + HD_OFF_Z);  // [HD_MAXM] logits
    const uint32_t rank = cluster_rank();
    const int grp = blockIdx.x / HD_CLUSTER;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r0 = grp * rows_per_cluster, r1 = min(a.n_rows, r0 + rows_per_cluster);
    if (r0 >= a.n_rows) return;  // the whole cluster
    const int m0 = a.opt_off[r0], nm = a.opt_off[r1] - m0;
    if (nm < 0 || nm > 20 * rows_per_cluster || m0 < 0 || m0 + nm > a.n_markers) {  // not a jd_serialize batch
        if (rank == 0 && tid == 0) atomicOr(a.status, ST_BAD_INDEX);
        return;  // the whole cluster
    }

    const int ul = warp * 4;                   // first of the warp's four units, CTA-local
    const int u0 = (int)rank * HD_UNITS + ul;  // global unit index
    float w[12][4];                            // W1[u0 + u][k] for the lane's inputs k = lane + 32 i
    if (!a.linear) {
#pragma unroll
        for (int i = 0; i < 12; ++i) {
            const float4 t = *reinterpret_cast<const float4 *>(a.w1t + (size_t)(lane + 32 * i) * D + u0);
            w[i][0] = t.x; w[i][1] = t.y; w[i][2] = t.z; w[i][3] = t.w;
        }
    }
    const int ua = u0 + (lane >> 3);
    const float b1 = a.linear ? 0.f : a.b1[ua], w2 = a.linear ? 0.f : a.w2[ua];
    cluster_sync();  // every CTA of the cluster runs before any writes into CTA 0's shared memory

    // the marker states of the next chunk are loaded into registers while the current one computes
    float v[12];
    auto load_chunk = [&](int mc) {
        const int mi = mc + warp;
        if (warp < 8 && mi < nm) {
            const float *src = a.hm + (size_t)(m0 + mi) * D;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const float4 x = *reinterpret_cast<const float4 *>(src + j * 128 + lane * 4);
                v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 12; ++k) v[k] = 0.f;
        }
    };
    load_chunk(0);
    for (int mc = 0; mc < nm; mc += 8) {
        // 1. LayerNorm (gain and bias, FP32, two-pass moments) of markers mc .. mc + 7 (zero past nm)
        if (warp < 8) {
            const int mi = mc + warp;
            if (mi < nm) {
                if (a.tap && rank == 0) {
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        *reinterpret_cast<float4 *>(a.tap + (size_t)(m0 + mi) * D + j * 128 + lane * 4) =
                            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
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
                    const float4 g = *reinterpret_cast<const float4 *>(a.ln_g + c);
                    const float4 b = *reinterpret_cast<const float4 *>(a.ln_b + c);
                    v[4 * j] = v[4 * j] * rstd * g.x + b.x;
                    v[4 * j + 1] = v[4 * j + 1] * rstd * g.y + b.y;
                    v[4 * j + 2] = v[4 * j + 2] * rstd * g.z + b.z;
                    v[4 * j + 3] = v[4 * j + 3] * rstd * g.w + b.w;
                }
            }
#pragma unroll
            for (int j = 0; j < 3; ++j)
                *reinterpret_cast<float4 *>(sn + warp * D + j * 128 + lane * 4) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
        __syncthreads();
        if (mc + 8 < nm) load_chunk(mc + 8);
        if (!a.linear) {
            // 2. z[b][u] = b1[u] + sum_k n[b][k] W1[u][k] for the warp's units; contribution W2[u] GELU(z)
            float acc[32];  // index 8 u + b: unit u0 + u, marker mc + b; partial over the lane's inputs
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = 0.f;
#pragma unroll
            for (int i = 0; i < 12; ++i) {
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const float x = sn[b * D + lane + 32 * i];
#pragma unroll
                    for (int u = 0; u < 4; ++u) acc[8 * u + b] = fmaf(x, w[i][u], acc[8 * u + b]);
                }
            }
            // butterfly transpose-reduce: after the step of offset o, value i of lane L stands for
            // index i + o * bit(L, o); at the end lane L holds the full sum of index L
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const bool up = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < o; ++i) {
                    const float send = up ? acc[i] : acc[i + o];
                    const float keep = up ? acc[i + o] : acc[i];
                    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            // lane L: unit u0 + (L >> 3), marker mc + (L & 7); sum the warp's four units per marker
            float c = w2 * gelu_erf(acc[0] + b1);
            c += __shfl_xor_sync(0xffffffffu, c, 8);
            c += __shfl_xor_sync(0xffffffffu, c, 16);
            if (lane < 8) sw[warp * 8 + lane] = c;
        }
        __syncthreads();
        // 3. the CTA's partial logit of each marker of the chunk (warps in order), to CTA 0
        if (tid < 8 && mc + tid < nm) {
            float s = 0.f;
            if (!a.linear) {
                for (int k = 0; k < HD_WARPS; ++k) s += sw[k * 8 + tid];
            } else if (rank == 0) {  // LayerNorm -> Linear(384, 1)
                for (int k = 0; k < D; ++k) s = fmaf(sn[tid * D + k], a.w2[k], s);
            }
            st_cluster_f32(&sp[rank * HD_MAXM + mc + tid], 0, s);
        }
        __syncthreads();  // sn and sw are rewritten by the next chunk
    }
    cluster_sync();
    if (rank != 0) return;

    // 4. logits (partials in rank order), then per-row softmax and read-outs
    for (int mi = tid; mi < nm; mi += HD_THREADS) {
        float z = a.b2[0];
        for (int r = 0; r < HD_CLUSTER; ++r) z += sp[r * HD_MAXM + mi];
        sz[mi] = z;
        a.logits[m0 + mi] = z;
    }
    __syncthreads();
    for (int r = r0 + warp; r < r1; r += HD_WARPS) {
        const int b = a.opt_off[r] - m0, k = a.opt_off[r + 1] - a.opt_off[r];
        float mx = -INFINITY;
        int arg = 0x7fffffff;
        for (int i = lane; i < k; i += 32) {
            const float v = sz[b + i];
            if (v > mx) { mx = v; arg = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, mx, o);
            const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
            if (om > mx || (om == mx && oa < arg)) { mx = om; arg = oa; }
        }
        float s = 0.f;
        for (int i = lane; i < k; i += 32) s += expf(sz[b + i] - mx);
        s = warp_sum(s);
        const float inv = 1.0f / s;
        float scv = 0.f, p1 = 0.f;
        for (int i = lane; i < k; i += 32) {
            const float p = expf(sz[b + i] - mx) * inv;
            a.probs[m0 + b + i] = p;
            scv += (float)i * p;
            if (i == 1) p1 = p;
        }
        scv = warp_sum(scv);
        p1 = warp_sum(p1);
        if (lane == 0) {
            a.choice[r] = arg;
            a.score[r] = scv;
            a.noul[r] = a.row_type[r] == 2 ? p1 : __int_as_float(0x7fc00000);
            a.max_p[r] = inv;  // exp(max - max) / sum
        }
    }
}

cudaError_t head_init_attributes() {
    return cudaFuncSetAttribute(k_head, cudaFuncAttributeMaxDynamicSharedMemorySize, HD_SMEM);
}

cudaError_t launch_head(const HeadArgs &a, cudaStream_t st) {
    if (a.n_rows <= 0 || a.n_markers <= 0) return cudaSuccess;
    const int rpc = std::min(HD_MAX_ROWS, std::max(1, (a.n_rows + HD_TARGET_CLUSTERS - 1) / HD_TARGET_CLUSTERS));
    const int clusters = (a.n_rows + rpc - 1) / rpc;
    k_head<<<clusters * HD_CLUSTER, HD_THREADS, HD_SMEM, st>>>(a, rpc);
    return cudaGetLastError();
}

}  // namespace jd
