// combine_balance.cu -- weighted combine back to token order, and the
// balance-loss statistics.
//
// Combine: y_t = sum over the selected experts of gate * E_i(x_t) ("Mixture-
// of-Experts" post, Eq. moe-output; "Fine-tuning and serving MoE models", the
// index-add of the gated expert outputs).  The gates are already applied by
// the grouped GEMM epilogue, so this is a gather-sum of k rows per token (plus
// the shared expert's row), in slot order with fp32 accumulation: the result
// does not depend on scheduling.  A dropped assignment (row -1) adds nothing.
//
// Balance: f_e = counts_e / (T k), P_e = mean over tokens of the normalised
// score, L = E sum f_e P_e (Vector Institute post, Eq. balance; Router
// Optimization page, How It Works 1), in the reduction order of balance.cuh.
// The forward pass computes them in the dispatch scan instead; this kernel
// serves the standalone entry point.
#include "balance.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

template <typename TY>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void add(const uint4 &v, float *acc) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
        }
    }
    __device__ __forceinline__ static uint4 pack(const float *acc) {
        uint4 v;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        return v;
    }
};
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void add(const uint4 &v, float *acc) {
        acc[0] += __uint_as_float(v.x); acc[1] += __uint_as_float(v.y);
        acc[2] += __uint_as_float(v.z); acc[3] += __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float *acc) {
        return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]),
                          __float_as_uint(acc[2]), __float_as_uint(acc[3]));
    }
};

constexpr int kCombThreads = 256;

// One warp per token (grid-stride); lanes stride over 16-byte column vectors.
// The row is taken in blocks of 256 vectors (4 KiB of bf16): for each block,
// each slot's part arrives in one burst of eight 16-byte loads per lane and
// joins the fp32 sums in slot order (then the shared expert's row), so the
// sum order -- and the result -- is that of a plain per-element loop.
template <typename TY>
__global__ void __launch_bounds__(kCombThreads) combine_kernel(CombineArgs a) {
    pdl_wait_then_release();
    using V = Vec16<TY>;
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (kCombThreads / 32);
    const int nvec = a.d / V::N;
    const uint4 *yp = static_cast<const uint4 *>(a.y_perm);
    uint4 *y = static_cast<uint4 *>(a.y);
    for (int t = blockIdx.x * (kCombThreads / 32) + (threadIdx.x >> 5); t < a.T; t += nwarps) {
        int my_row = -1;
        if (lane < a.k) {
            my_row = a.row_of[(size_t)t * a.k + lane];
            if (my_row >= a.rows_routed) {
                record_error(a.status, MOE_ERR_DEVICE_BOUNDS, t);
                my_row = -1;
            }
        }
        const int64_t shared_row = a.rows_routed + t;
        // every lane runs the column loop (the row indices come by shuffle
        // from lanes 0..k-1); lanes past the row's last vector only idle
        for (int vb = 0; vb < nvec; vb += 256) {
            float acc[8][V::N];
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int i = 0; i < V::N; ++i) acc[j][i] = 0.f;
            for (int s = 0; s <= a.k; ++s) {
                int64_t r;
                if (s < a.k) r = __shfl_sync(0xffffffffu, my_row, s);
                else r = a.has_shared ? shared_row : -1;
                if (r < 0) continue;                                    // the same on every lane
                uint4 q[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int v = vb + 32 * j + lane;
                    if (v < nvec) q[j] = __ldg(yp + (size_t)r * nvec + v);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (vb + 32 * j + lane < nvec) V::add(q[j], acc[j]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int v = vb + 32 * j + lane;
                if (v < nvec) y[(size_t)t * nvec + v] = V::pack(acc[j]);
            }
        }
    }
}

// 32 warps; for each block of 32 experts, the P sums in the balance.cuh order
// (psum_block32: warp w ends with expert e0 + w), then the loss terms meet in
// loss_tree.  Everything in double; the result does not depend on scheduling
// and equals the forward pass's (dispatch scan and permute).
__global__ void __launch_bounds__(1024) balance_kernel(BalanceArgs a) {
    pdl_wait_then_release();
    __shared__ double red[256];
    __shared__ double cls[32][33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < 256) red[threadIdx.x] = 0.0;
    for (int e0 = 0; e0 < a.E; e0 += 32) {
        const double sum = psum_block32(a.psum, a.nblk, a.E, e0, cls);
        const int e = e0 + warp;
        if (e < a.E && lane == 0) {
            const double P = sum / (double)a.T;
            const double f = (double)a.counts[e] / ((double)a.T * (double)a.k);
            a.f[e] = (float)f;
            a.P[e] = (float)P;
            red[e] = f * P;
        }
    }
    const double s = loss_tree(red);
    if (threadIdx.x == 0) *a.loss = (double)a.E * s;
}

// Auxiliary-loss-free bias update ("Fine-Tuning Mixture of Experts (MoE)
// Models: Router Optimization Techniques", How It Works 2, and its router
// module): b_e <- b_e - gamma * sign(count_e - T k / E), in double.
__global__ void bias_update_kernel(const int32_t *counts, float *bias, double gamma, int T, int k, int E) {
    pdl_wait_then_release();
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const double err = (double)counts[e] - (double)T * (double)k / (double)E;
    const double sgn = err > 0.0 ? 1.0 : (err < 0.0 ? -1.0 : 0.0);
    bias[e] = (float)((double)bias[e] - gamma * sgn);
}

// Routing health: entropy -sum P log P of the mean routing distribution
// (Router Optimization page, Best Practices 6), max/min count ratio and the
// largest load share ("Fine-tuning and serving MoE models", Utilization is a
// first-class metric).  One CTA; fixed-order tree sums in double.
__global__ void __launch_bounds__(256) routing_health_kernel(const int32_t *counts, const float *P, double *out,
                                                             int T, int k, int E) {
    pdl_wait_then_release();
    __shared__ double hs[256];
    __shared__ int mx[256], mn[256];
    const int e = threadIdx.x;
    double h = 0.0;
    int cmax = -1, cmin = 0x7fffffff;
    if (e < E) {
        const double p = (double)P[e];
        if (p > 0.0) h = -p * log(p);
        cmax = cmin = counts[e];
    }
    hs[e] = h; mx[e] = cmax; mn[e] = cmin;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (e < o) {
            hs[e] += hs[e + o];
            mx[e] = max(mx[e], mx[e + o]);
            mn[e] = min(mn[e], mn[e + o]);
        }
        __syncthreads();
    }
    if (e == 0) {
        out[0] = hs[0];
        out[1] = mn[0] > 0 ? (double)mx[0] / (double)mn[0] : (double)INFINITY;
        out[2] = (double)mx[0] / ((double)T * (double)k);
    }
}

}  // namespace

cudaError_t launch_bias_update(const int32_t *counts, float *bias, double gamma, int T, int k, int E,
                               cudaStream_t st) {
    bias_update_kernel<<<(E + 255) / 256, 256, 0, st>>>(counts, bias, gamma, T, k, E);
    return cudaGetLastError();
}

cudaError_t launch_routing_health(const int32_t *counts, const float *P, double *out, int T, int k, int E,
                                  cudaStream_t st) {
    routing_health_kernel<<<1, 256, 0, st>>>(counts, P, out, T, k, E);
    return cudaGetLastError();
}

cudaError_t launch_combine(const CombineArgs &a, bool bf16, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    const int warps_per_block = kCombThreads / 32;
    int blocks = (a.T + warps_per_block - 1) / warps_per_block;
    const int cap = a.num_sms * 8;
    if (blocks > cap) blocks = cap;
    if (bf16) return launch_kernel(combine_kernel<__nv_bfloat16>, dim3(blocks), dim3(kCombThreads), 0, st, a.pdl, a);
    return launch_kernel(combine_kernel<float>, dim3(blocks), dim3(kCombThreads), 0, st, a.pdl, a);
}

cudaError_t launch_balance(const BalanceArgs &a, cudaStream_t st) {
    balance_kernel<<<1, 1024, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
