// ffn_f32.cu -- grouped expert FFN for fp32 layers (FFMA on the SIMT pipes).
//
// Expert definitions: GELU expert Linear-GELU-Linear with biases ("Fine-tuning
// and serving MoE models", How an MoE layer actually works; nn.GELU is the
// exact-erf form); SwiGLU expert W_down(SiLU(W_gate x) * (W_up x)) ("Fine-
// Tuning Mixture of Experts (MoE) Models: Router Optimization Techniques",
// What Is It?).  The gate of each row scales the second GEMM's output, so the
// combine is a plain sum (Vector Institute post, Eq. moe-output).
//
// fp32 keeps the whole layer at fp32 accuracy (a tf32 tensor-core product
// would not).  Two launches (GEMM1 with the activation fused, GEMM2 with bias
// and gate fused), one CTA per 64x64 output tile; the tile's expert is found
// from the device-side offsets, so no host synchronisation is needed.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int BM = 64, BN = 64, BK = 16, kThreads = 256;
constexpr int kMaxGroups = 257;

enum { MODE_GELU = 0, MODE_SWIGLU = 1, MODE_DOWN = 2 };

struct GroupTable {
    int mt_start[kMaxGroups + 1];
};

__device__ __forceinline__ float gelu_erf(float v) { return 0.5f * v * (1.f + erff(v * 0.70710678118654752f)); }
__device__ __forceinline__ float silu(float v) { return v / (1.f + expf(-v)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads) simt_grouped_gemm(FfnArgs a) {
    pdl_wait_then_release();
    __shared__ GroupTable tab;
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    __shared__ float Bs2[MODE == MODE_SWIGLU ? BK : 1][BN + 4];

    const int tid = threadIdx.x;
    const int G = a.n_groups + (a.S > 0 ? 1 : 0);
    if (tid == 0) {
        int acc = 0;
        for (int g = 0; g < G; ++g) {
            tab.mt_start[g] = acc;
            const int rows = g < a.n_groups ? a.offsets[g + 1] - a.offsets[g] : a.T;
            acc += (rows + BM - 1) / BM;
        }
        tab.mt_start[G] = acc;
    }
    __syncthreads();
    const int mt = blockIdx.x;
    if (mt >= tab.mt_start[G]) return;
    int g = 0;
    while (tab.mt_start[g + 1] <= mt) ++g;
    const bool shared = g >= a.n_groups;
    const int rows = shared ? a.T : a.offsets[g + 1] - a.offsets[g];
    const int e = shared ? 0 : (a.n_groups == a.E ? g : g % a.E);     // weight expert of the group
    const int m0 = (mt - tab.mt_start[g]) * BM;
    const int64_t out_row0 = shared ? a.shared_base : (int64_t)a.offsets[g];

    const float *A;
    int64_t lda;
    int K, N;
    const float *W, *W2nd = nullptr, *bias = nullptr;
    if (MODE != MODE_DOWN) {
        K = a.d;
        N = shared ? a.S : a.F;
        A = shared ? static_cast<const float *>(a.x) : static_cast<const float *>(a.x_perm) + out_row0 * a.d;
        lda = a.d;
        W = shared ? static_cast<const float *>(a.Wsg) : static_cast<const float *>(a.W1) + (size_t)e * a.F * a.d;
        if (MODE == MODE_SWIGLU)
            W2nd = shared ? static_cast<const float *>(a.Wsu) : static_cast<const float *>(a.Wu) + (size_t)e * a.F * a.d;
        if (MODE == MODE_GELU && !shared && a.b1) bias = a.b1 + (size_t)e * a.F;
    } else {
        K = shared ? a.S : a.F;
        N = a.d;
        A = static_cast<const float *>(a.H) + out_row0 * a.hF;
        lda = a.hF;
        W = shared ? static_cast<const float *>(a.Wsd) : static_cast<const float *>(a.W2) + (size_t)e * a.d * a.F;
        if (!shared && a.b2) bias = a.b2 + (size_t)e * a.d;
    }
    const int n0 = blockIdx.y * BN;
    if (n0 >= N) return;

    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4], acc2[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { acc[i][j] = 0.f; acc2[i][j] = 0.f; }

    const int lr = tid / 4, lk = (tid % 4) * 4;       // loader: row / col-quad
    for (int k0 = 0; k0 < K; k0 += BK) {
        {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m0 + lr < rows && k0 + lk < K) v = *reinterpret_cast<const float4 *>(A + (m0 + lr) * lda + k0 + lk);
            As[lk + 0][lr] = v.x; As[lk + 1][lr] = v.y; As[lk + 2][lr] = v.z; As[lk + 3][lr] = v.w;
            float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n0 + lr < N && k0 + lk < K) w = *reinterpret_cast<const float4 *>(W + (size_t)(n0 + lr) * K + k0 + lk);
            Bs[lk + 0][lr] = w.x; Bs[lk + 1][lr] = w.y; Bs[lk + 2][lr] = w.z; Bs[lk + 3][lr] = w.w;
            if (MODE == MODE_SWIGLU) {
                float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
                if (n0 + lr < N && k0 + lk < K) u = *reinterpret_cast<const float4 *>(W2nd + (size_t)(n0 + lr) * K + k0 + lk);
                Bs2[lk + 0][lr] = u.x; Bs2[lk + 1][lr] = u.y; Bs2[lk + 2][lr] = u.z; Bs2[lk + 3][lr] = u.w;
            }
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float av[4], bv[4], uv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
            if (MODE == MODE_SWIGLU) {
#pragma unroll
                for (int j = 0; j < 4; ++j) uv[j] = Bs2[kk][tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
                    if (MODE == MODE_SWIGLU) acc2[i][j] = fmaf(av[i], uv[j], acc2[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m0 + ty * 4 + i;
        if (r >= rows) continue;
        const int64_t orow = out_row0 + r;
        float gscale = 1.f;
        if (MODE == MODE_DOWN && !shared) gscale = a.row_gate[orow];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= N) continue;
            float v = acc[i][j];
            if (bias) v += bias[n];
            if (MODE == MODE_GELU) {
                static_cast<float *>(a.H)[orow * a.hF + n] = gelu_erf(v);
            } else if (MODE == MODE_SWIGLU) {
                static_cast<float *>(a.H)[orow * a.hF + n] = silu(v) * acc2[i][j];
            } else {
                static_cast<float *>(a.y_perm)[orow * a.d + n] = gscale * v;
            }
        }
    }
}

}  // namespace

cudaError_t launch_ffn_f32(const FfnArgs &a, cudaStream_t st) {
    if (a.routed_rows == 0 && (a.S == 0 || a.T == 0)) return cudaSuccess;
    const int64_t routed = a.routed_rows;
    int64_t mtiles = (routed + BM - 1) / BM + a.n_groups;
    if (a.S > 0) mtiles += (a.T + BM - 1) / BM + 1;
    const int n1 = (a.F > a.S ? a.F : a.S);
    dim3 g1((unsigned)mtiles, (unsigned)((n1 + BN - 1) / BN));
    cudaError_t e = a.act == MOE_ACT_SWIGLU
                        ? launch_kernel(simt_grouped_gemm<MODE_SWIGLU>, g1, dim3(kThreads), 0, st, a.pdl, a)
                        : launch_kernel(simt_grouped_gemm<MODE_GELU>, g1, dim3(kThreads), 0, st, a.pdl, a);
    if (e != cudaSuccess) return e;
    dim3 g2((unsigned)mtiles, (unsigned)((a.d + BN - 1) / BN));
    return launch_kernel(simt_grouped_gemm<MODE_DOWN>, g2, dim3(kThreads), 0, st, true, a);
}

}  // namespace moe
