// router_topk.cu -- router GEMM, fp32 scores, top-k selection and gates.
//
// "Mixture-of-Experts" (Vector Institute post), router section: one score per
// expert h = x W_r, softmax over experts, top-k, gates from the full softmax
// (Eq. moe-output) or renormalised over the selected experts.  "Fine-tuning
// and serving MoE models", How an MoE layer actually works: the router softmax
// runs in fp32.  "Fine-Tuning Mixture of Experts (MoE) Models: Router
// Optimization Techniques", How It Works 2: a per-expert bias steers the
// selection only; gates come from the unbiased scores.
//
// This FFMA version serves fp32 layers; bf16 layers use router_sm100.cu.
// One CTA handles 32 tokens and all E (<= 256) experts.  The logits of a token
// live in the registers of one warp (expert e on lane e % 32), so the softmax,
// the k rounds of warp arg-max and the gates never leave registers.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kTok = 32;          // tokens per CTA
constexpr int kThreads = 256;     // 8 warps, 4 tokens each
constexpr int kKc = 32;           // d_model chunk staged in shared memory

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Order-preserving map of a finite fp32 key to an unsigned integer.
__device__ __forceinline__ unsigned ordered_key(float f) {
    const unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename TX>
__device__ __forceinline__ void load_x_vec(const TX *src, float *dst);

template <>
__device__ __forceinline__ void load_x_vec<float>(const float *src, float *dst) {
    float4 v = *reinterpret_cast<const float4 *>(src);
    dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
}

// Compare-exchange for the lane-local sort: order by key descending, then
// expert id ascending (the tie rule of the selection).
__device__ __forceinline__ void cex(unsigned &ka, int &ia, float &ga, unsigned &kb, int &ib, float &gb) {
    const bool sw = ka < kb || (ka == kb && ia > ib);
    const unsigned tk = sw ? kb : ka; kb = sw ? ka : kb; ka = tk;
    const int ti = sw ? ib : ia; ib = sw ? ia : ib; ia = ti;
    const float tg = sw ? gb : ga; gb = sw ? ga : gb; ga = tg;
}

// Sorting networks for 2, 4 and 8 candidates per lane (Batcher's odd-even
// merge sort for 8).
template <int EPT>
__device__ __forceinline__ void lane_sort(unsigned (&k)[EPT], int (&id)[EPT], float (&g)[EPT]) {
#define CEX(i, j) cex(k[i], id[i], g[i], k[j], id[j], g[j])
    if constexpr (EPT == 2) {
        CEX(0, 1);
    } else if constexpr (EPT == 4) {
        CEX(0, 1); CEX(2, 3); CEX(0, 2); CEX(1, 3); CEX(1, 2);
    } else if constexpr (EPT == 8) {
        CEX(0, 1); CEX(2, 3); CEX(4, 5); CEX(6, 7);
        CEX(0, 2); CEX(1, 3); CEX(4, 6); CEX(5, 7);
        CEX(1, 2); CEX(5, 6);
        CEX(0, 4); CEX(1, 5); CEX(2, 6); CEX(3, 7);
        CEX(2, 4); CEX(3, 5);
        CEX(1, 2); CEX(3, 4); CEX(5, 6);
    }
#undef CEX
}

// Scores, top-k and gates of token t, whose logits h[j] (expert lane + 32 j,
// logit offset included) sit in the registers of one warp; sb[j] is the
// selection bias of the same expert (0 without one).  The token's
// normalised scores are added into psum_acc.
//
// Selection: each lane sorts its EPT candidates by (key desc, id asc); then
// k rounds, each taking the largest head key over the warp (redux.sync on an
// order-preserving integer image of the fp32 key) and, among the lanes that
// hold it, the lowest expert id.  The winner lane pops its head.  Lane r
// keeps the winner of round r, so slot r of idx and gate is written by lane r.
template <int EPT>
__device__ __forceinline__ void select_token(const RouterArgs &a, const float (&h)[EPT], const float (&sb)[EPT],
                                             int t, float (&psum_acc)[EPT]) {
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k;
    const bool softmax = a.score == MOE_SCORE_SOFTMAX;
    float gs[EPT], kf[EPT];                  // gate source; selection key
    if (softmax) {
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < EPT; ++j) if (lane + 32 * j < E) m = fmaxf(m, h[j]);
        m = warp_max(m);
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < EPT; ++j) { gs[j] = (lane + 32 * j < E) ? expf(h[j] - m) : 0.f; z += gs[j]; }
        const float inv = 1.f / warp_sum(z);
#pragma unroll
        for (int j = 0; j < EPT; ++j) { gs[j] *= inv; psum_acc[j] += gs[j]; kf[j] = h[j] + sb[j]; }
    } else {
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            gs[j] = (lane + 32 * j < E) ? 1.f / (1.f + expf(-h[j])) : 0.f;
            z += gs[j];
        }
        const float inv = 1.f / warp_sum(z);
#pragma unroll
        for (int j = 0; j < EPT; ++j) { psum_acc[j] += gs[j] * inv; kf[j] = gs[j] + sb[j]; }
    }
    unsigned key[EPT];
    int id[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        id[j] = lane + 32 * j;
        // absent experts rank below every real key; a NaN key ranks just above them
        key[j] = id[j] < E ? (kf[j] == kf[j] ? ordered_key(kf[j]) : 1u) : 0u;
    }
    lane_sort<EPT>(key, id, gs);
    unsigned my_id = 0;
    float my_g = 0.f;
    for (int r = 0; r < k; ++r) {
        const unsigned kmax = __reduce_max_sync(0xffffffffu, key[0]);
        const unsigned be = __reduce_min_sync(0xffffffffu, key[0] == kmax ? (unsigned)id[0] : 0xffffffffu);
        const int wl = (int)(be & 31u);
        const float gw = __shfl_sync(0xffffffffu, gs[0], wl);
        if (lane == r) { my_id = be; my_g = gw; }
        if (lane == wl) {
#pragma unroll
            for (int j = 0; j + 1 < EPT; ++j) { key[j] = key[j + 1]; id[j] = id[j + 1]; gs[j] = gs[j + 1]; }
            key[EPT - 1] = 0u;
            id[EPT - 1] = 0x7fffffff;
        }
    }
    const float selsum = warp_sum(lane < k ? my_g : 0.f);
    if (lane < k) {
        a.idx[(size_t)t * k + lane] = (int)my_id;
        a.gate[(size_t)t * k + lane] = (softmax && !a.renorm) ? my_g : my_g / selsum;
    }
}

// The 32 tokens starting at t0 (warp w holds tokens t0 + 4w .. t0 + 4w + 3;
// acc[i][j] is the logit of token 4w + i for expert lane + 32 j).
// add_bias: add logit_bias to acc first (the tensor-core path has);
// write_logits: store the logits to logits_out.
template <int EPT>
__device__ __forceinline__ void select_tokens(const RouterArgs &a, float (&acc)[4][EPT], int t0, bool add_bias,
                                              bool write_logits, const float (&sb)[EPT], float (&psum_acc)[EPT]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E;
    float lb[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) lb[j] = (add_bias && a.logit_bias && lane + 32 * j < E) ? a.logit_bias[lane + 32 * j] : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + warp * 4 + i;
        if (t >= a.T) break;                         // uniform across the warp
        float h[EPT];
#pragma unroll
        for (int j = 0; j < EPT; ++j) h[j] = acc[i][j] + lb[j];
        if (write_logits) {
#pragma unroll
            for (int j = 0; j < EPT; ++j)
                if (lane + 32 * j < E) a.logits_out[(size_t)t * E + lane + 32 * j] = h[j];
        }
        select_token<EPT>(a, h, sb, t, psum_acc);
    }
}

template <int EPT>
__device__ __forceinline__ void load_sel_bias(const RouterArgs &a, float (&sb)[EPT]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < EPT; ++j) sb[j] = (a.sel_bias && lane + 32 * j < a.E) ? a.sel_bias[lane + 32 * j] : 0.f;
}

// The CTA's row of the per-block score sums: warp partials added in warp order.
template <int EPT>
__device__ __forceinline__ void write_psum(const RouterArgs &a, float (*part)[EPT * 32], const float (&psum_acc)[EPT]) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int j = 0; j < EPT; ++j) part[warp][lane + 32 * j] = psum_acc[j];
    __syncthreads();
    for (int e = tid; e < a.E; e += kThreads) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) s += part[w][e];
        a.psum[(size_t)blockIdx.x * a.E + e] = s;
    }
}

template <typename TX, int EPT>
__global__ void __launch_bounds__(kThreads) router_topk_kernel(RouterArgs a) {
    pdl_wait_then_release();
    constexpr int VEC = 16 / sizeof(TX);              // x elements per 16-byte load
    constexpr int EW = EPT * 32;                      // expert slots per warp row
    __shared__ float xs[kTok][kKc + 1];
    __shared__ float wsm[kKc][EW];
    __shared__ float part[kThreads / 32][EW];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * kTok;
    const int d = a.d, E = a.E;

    float acc[4][EPT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EPT; ++j) acc[i][j] = 0.f;

    const TX *x = static_cast<const TX *>(a.x);
    for (int k0 = 0; k0 < d; k0 += kKc) {
        // x chunk [32 tokens][32]: 16-byte vector loads (d % 8 == 0)
        for (int v = tid; v < kTok * (kKc / VEC); v += kThreads) {
            const int tt = v / (kKc / VEC), kv = (v % (kKc / VEC)) * VEC;
            float vals[VEC];
            const int t = t0 + tt;
            if (t < a.T && k0 + kv < d) {
                load_x_vec<TX>(x + (size_t)t * d + k0 + kv, vals);
            } else {
#pragma unroll
                for (int i = 0; i < VEC; ++i) vals[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < VEC; ++i) xs[tt][kv + i] = vals[i];
        }
        // W_r chunk [32][E] (row-major [d, E], coalesced along E)
        for (int v = tid; v < kKc * EW; v += kThreads) {
            const int kk = v / EW, e = v % EW;
            wsm[kk][e] = (k0 + kk < d && e < E) ? a.Wr[(size_t)(k0 + kk) * E + e] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kKc; ++kk) {
            float xv[4], wv[EPT];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[warp * 4 + i][kk];
#pragma unroll
            for (int j = 0; j < EPT; ++j) wv[j] = wsm[kk][lane + 32 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < EPT; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }

    float psum_acc[EPT], sb[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) psum_acc[j] = 0.f;
    load_sel_bias<EPT>(a, sb);
    select_tokens<EPT>(a, acc, t0, /*add_bias=*/true, a.logits_out != nullptr, sb, psum_acc);
    write_psum<EPT>(a, part, psum_acc);
}

// Selection for bf16 layers: `parts` holds `splits` partial logits [T, E]
// (offset already added to split 0) from the tensor-core router, added in
// split order; then the same per-warp selection as the fp32 path.  One CTA
// takes 32 tokens (many small CTAs keep the SMs evenly loaded), so the score
// sums have T/32 rows, as for fp32 layers.
constexpr int kSelTok = 32;

template <int EPT>
__global__ void __launch_bounds__(kThreads) router_select_kernel(RouterArgs a, const float *__restrict__ parts,
                                                                 int splits) {
    pdl_wait_then_release();
    __shared__ float part[kThreads / 32][EPT * 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float psum_acc[EPT], sb[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) psum_acc[j] = 0.f;
    load_sel_bias<EPT>(a, sb);
    const size_t plane = (size_t)a.T * a.E;
    for (int grp = 0; grp < kSelTok / kTok; ++grp) {
        const int t0 = blockIdx.x * kSelTok + grp * kTok;
        if (t0 >= a.T) break;
        float acc[4][EPT];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = t0 + warp * 4 + i;
#pragma unroll
            for (int j = 0; j < EPT; ++j) {
                const int e = lane + 32 * j;
                acc[i][j] = (t < a.T && e < a.E) ? parts[(size_t)t * a.E + e] : 0.f;
            }
        }
        for (int sp = 1; sp < splits; ++sp) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = t0 + warp * 4 + i;
#pragma unroll
                for (int j = 0; j < EPT; ++j) {
                    const int e = lane + 32 * j;
                    if (t < a.T && e < a.E) acc[i][j] += parts[sp * plane + (size_t)t * a.E + e];
                }
            }
        }
        select_tokens<EPT>(a, acc, t0, /*add_bias=*/false, splits > 1 && a.logits_out != nullptr, sb, psum_acc);
    }
    write_psum<EPT>(a, part, psum_acc);
}

template <typename TX>
cudaError_t launch_router_t(const RouterArgs &a, cudaStream_t st) {
    const dim3 blocks((a.T + kTok - 1) / kTok), threads(kThreads);
    if (a.E <= 32) return launch_kernel(router_topk_kernel<TX, 1>, blocks, threads, 0, st, a.pdl, a);
    if (a.E <= 64) return launch_kernel(router_topk_kernel<TX, 2>, blocks, threads, 0, st, a.pdl, a);
    if (a.E <= 128) return launch_kernel(router_topk_kernel<TX, 4>, blocks, threads, 0, st, a.pdl, a);
    return launch_kernel(router_topk_kernel<TX, 8>, blocks, threads, 0, st, a.pdl, a);
}

}  // namespace

int router_blocks(int T, bool bf16) { return bf16 ? (T + kSelTok - 1) / kSelTok : (T + kTok - 1) / kTok; }
static_assert(kSelTok % kTok == 0, "selection blocks hold whole 32-token groups");

// bf16 layers: logits on the tensor cores (router_sm100.cu), then the
// warp-per-token selection; fp32 layers: this FFMA kernel end to end, which
// keeps every product in fp32.
cudaError_t launch_router(const RouterArgs &a, bool bf16, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    if (!bf16) return launch_router_t<float>(a, st);
    // one split writes the logits straight to logits_out when asked for them;
    // several write partials to the workspace and the selection adds them
    const int splits = router_logit_splits(a.T, a.d, a.num_sms);
    float *parts = (splits == 1 && a.logits_out) ? a.logits_out : a.logits_ws;
    cudaError_t e = launch_router_logits_tc(a, parts, splits, st);
    if (e != cudaSuccess) return e;
    const dim3 blocks((a.T + kSelTok - 1) / kSelTok), threads(kThreads);
    const float *cparts = parts;
    if (a.E <= 32) return launch_kernel(router_select_kernel<1>, blocks, threads, 0, st, true, a, cparts, splits);
    if (a.E <= 64) return launch_kernel(router_select_kernel<2>, blocks, threads, 0, st, true, a, cparts, splits);
    if (a.E <= 128) return launch_kernel(router_select_kernel<4>, blocks, threads, 0, st, true, a, cparts, splits);
    return launch_kernel(router_select_kernel<8>, blocks, threads, 0, st, true, a, cparts, splits);
}

}  // namespace moe
