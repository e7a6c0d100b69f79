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

// Scores, top-k and gates for the 32 tokens starting at t0 (warp w holds
// tokens t0 + 4w .. t0 + 4w + 3; acc[i][j] is the logit of token 4w + i for
// expert lane + 32 j), adding each token's normalised scores into psum_acc.
// add_bias: add logit_bias to acc first (the tensor-core path has added it).
template <int EPT>
__device__ __forceinline__ void select_tokens(const RouterArgs &a, float (&acc)[4][EPT], int t0, bool add_bias,
                                              float (&psum_acc)[EPT]) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, k = a.k;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + warp * 4 + i;
        if (t >= a.T) break;                         // uniform across the warp
        float h[EPT], sc[EPT], key[EPT];
        bool valid[EPT];
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const int e = lane + 32 * j;
            valid[j] = e < E;
            h[j] = acc[i][j] + ((add_bias && a.logit_bias && valid[j]) ? a.logit_bias[e] : 0.f);
        }
        float norm;
        if (a.score == MOE_SCORE_SOFTMAX) {
            float m = -INFINITY;
#pragma unroll
            for (int j = 0; j < EPT; ++j) if (valid[j]) m = fmaxf(m, h[j]);
            m = warp_max(m);
            float z = 0.f;
#pragma unroll
            for (int j = 0; j < EPT; ++j) { sc[j] = valid[j] ? expf(h[j] - m) : 0.f; z += sc[j]; }
            norm = warp_sum(z);
#pragma unroll
            for (int j = 0; j < EPT; ++j) { sc[j] = sc[j] / norm; key[j] = h[j]; }
            norm = 1.f;                              // sc already normalised
        } else {
            float z = 0.f;
#pragma unroll
            for (int j = 0; j < EPT; ++j) { sc[j] = valid[j] ? 1.f / (1.f + expf(-h[j])) : 0.f; z += sc[j]; }
            norm = warp_sum(z);
#pragma unroll
            for (int j = 0; j < EPT; ++j) key[j] = sc[j];
        }
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            if (a.sel_bias && valid[j]) key[j] += a.sel_bias[lane + 32 * j];
            psum_acc[j] += (a.score == MOE_SCORE_SOFTMAX) ? sc[j] : sc[j] / norm;
        }
        if (a.logits_out && add_bias) {
#pragma unroll
            for (int j = 0; j < EPT; ++j)
                if (valid[j]) a.logits_out[(size_t)t * E + lane + 32 * j] = h[j];
        }
        // k rounds of warp arg-max on (key desc, expert id asc): each lane
        // offers its best untaken expert; redux.sync picks the largest key
        // (as an order-preserving integer), then the lowest expert id among
        // the lanes holding it.  The owner lane records the slot.
        unsigned taken = 0;
        int slot[EPT];
#pragma unroll
        for (int j = 0; j < EPT; ++j) slot[j] = -1;
        for (int r = 0; r < k; ++r) {
            float bk = 0.f;
            int bj = -1;
#pragma unroll
            for (int j = 0; j < EPT; ++j)
                if (valid[j] && !(taken & (1u << j)) && (bj < 0 || key[j] > bk)) { bk = key[j]; bj = j; }
            const unsigned offer = (bj >= 0 && bk == bk) ? ordered_key(bk) : 0u;
            const unsigned kmax = __reduce_max_sync(0xffffffffu, offer);
            const unsigned cand = (bj >= 0 && offer == kmax) ? (unsigned)(lane + 32 * bj) : 0xffffffffu;
            const unsigned be = __reduce_min_sync(0xffffffffu, cand);
            if (be < (unsigned)E && (int)(be & 31u) == lane) {
                taken |= 1u << (be >> 5);
#pragma unroll
                for (int j = 0; j < EPT; ++j)
                    if ((unsigned)j == (be >> 5)) slot[j] = r;
            }
        }
        float mine = 0.f;
#pragma unroll
        for (int j = 0; j < EPT; ++j) if (slot[j] >= 0) mine += sc[j];
        const float selsum = warp_sum(mine);
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            if (slot[j] >= 0) {
                const float g = (a.score == MOE_SCORE_SOFTMAX && !a.renorm) ? sc[j] : sc[j] / selsum;
                a.idx[(size_t)t * k + slot[j]] = lane + 32 * j;
                a.gate[(size_t)t * k + slot[j]] = g;
            }
        }
    }
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

    float psum_acc[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) psum_acc[j] = 0.f;
    select_tokens<EPT>(a, acc, t0, /*add_bias=*/true, psum_acc);
    write_psum<EPT>(a, part, psum_acc);
}

// Selection for bf16 layers: logits [T, E] (offset already added) from the
// tensor-core router, same per-warp selection as the fp32 path; one CTA takes
// 64 tokens (two groups of 32), so the score sums have T/64 rows.
constexpr int kSelTok = 64;

template <int EPT>
__global__ void __launch_bounds__(kThreads) router_select_kernel(RouterArgs a, const float *__restrict__ logits) {
    __shared__ float part[kThreads / 32][EPT * 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float psum_acc[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) psum_acc[j] = 0.f;
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
                acc[i][j] = (t < a.T && e < a.E) ? logits[(size_t)t * a.E + e] : 0.f;
            }
        }
        select_tokens<EPT>(a, acc, t0, /*add_bias=*/false, psum_acc);
    }
    write_psum<EPT>(a, part, psum_acc);
}

template <typename TX>
cudaError_t launch_router_t(const RouterArgs &a, cudaStream_t st) {
    const int blocks = (a.T + kTok - 1) / kTok;
    if (a.E <= 32) router_topk_kernel<TX, 1><<<blocks, kThreads, 0, st>>>(a);
    else if (a.E <= 64) router_topk_kernel<TX, 2><<<blocks, kThreads, 0, st>>>(a);
    else if (a.E <= 128) router_topk_kernel<TX, 4><<<blocks, kThreads, 0, st>>>(a);
    else router_topk_kernel<TX, 8><<<blocks, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

int router_blocks(int T, bool bf16) { return bf16 ? (T + kSelTok - 1) / kSelTok : (T + kTok - 1) / kTok; }

// bf16 layers: logits on the tensor cores (router_sm100.cu), then the
// warp-per-token selection; fp32 layers: this FFMA kernel end to end, which
// keeps every product in fp32.
cudaError_t launch_router(const RouterArgs &a, bool bf16, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    if (!bf16) return launch_router_t<float>(a, st);
    float *logits = a.logits_out ? a.logits_out : a.logits_ws;
    cudaError_t e = launch_router_logits_tc(a, logits, st);
    if (e != cudaSuccess) return e;
    const int blocks = (a.T + kSelTok - 1) / kSelTok;
    if (a.E <= 32) router_select_kernel<1><<<blocks, kThreads, 0, st>>>(a, logits);
    else if (a.E <= 64) router_select_kernel<2><<<blocks, kThreads, 0, st>>>(a, logits);
    else if (a.E <= 128) router_select_kernel<4><<<blocks, kThreads, 0, st>>>(a, logits);
    else router_select_kernel<8><<<blocks, kThreads, 0, st>>>(a, logits);
    return cudaGetLastError();
}

}  // namespace moe
