// quant_fp8.cu -- per-row e4m3 quantization of bf16 activations.
//
// FP8 experts are the serving page's advice to quantize experts ("Fine-tuning
// and serving MoE models", Serving: throughput does not scale the way you
// expect, consequences for capacity planning).  The activations that feed an
// e4m3 expert GEMM (x, and each expert's hidden activation H) get one scale
// per row:
//   amax  = max_j |v_j|
//   inv   = 448 / amax            (0 for a zero row)
//   code  = e4m3(v_j * inv)       round to nearest even, saturating at 448
//   scale = amax / 448
// all in fp32 with correctly rounded division and product, so the codes are
// a function of the bf16 inputs alone.
//
// One warp per row: 16-byte loads of eight bf16 values, a warp max, then a
// second pass (the row is in L1/L2 by then) that converts pairs with the
// hardware's satfinite e4m3x2 conversion and stores eight codes per lane.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ void unpack8(const uint4 &u, float *f) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 p = __bfloat1622float2(h[i]);
        f[2 * i] = p.x;
        f[2 * i + 1] = p.y;
    }
}

__global__ void __launch_bounds__(kQuantThreads) quant_rows_kernel(QuantArgs a) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    int64_t nrows = a.rows;
    if (a.rows_limit) {
        const int64_t lim = *a.rows_limit;
        nrows = lim < 0 ? 0 : (lim < nrows ? lim : nrows);
    }
    const int64_t wid = ((int64_t)blockIdx.x * kQuantThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kQuantThreads) >> 5;
    const int nvec = a.cols >> 3;
    for (int64_t r = wid; r < nrows; r += nw) {
        const int64_t row = a.row0 + r;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.in + row * a.ld_in);
        float amax = 0.f;
        for (int v = lane; v < nvec; v += 32) {
            float f[8];
            unpack8(src[v], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
        uint2 *dst = reinterpret_cast<uint2 *>(a.out + row * a.ld_out);
        for (int v = lane; v < nvec; v += 32) {
            float f[8];
            unpack8(src[v], f);
            uint32_t w[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(f[4 * h], inv), __fmul_rn(f[4 * h + 1], inv)), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(f[4 * h + 2], inv), __fmul_rn(f[4 * h + 3], inv)), __NV_SATFINITE, __NV_E4M3);
                w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            dst[v] = make_uint2(w[0], w[1]);
        }
        if (lane == 0) a.scale[row] = __fdiv_rn(amax, 448.f);
    }
}

}  // namespace

cudaError_t launch_quant_rows(const QuantArgs &a, cudaStream_t st) {
    if (a.rows <= 0 || a.cols <= 0) return cudaSuccess;
    const int sms = a.num_sms > 0 ? a.num_sms : 148;
    const int64_t want = (a.rows + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
    const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    return launch_kernel(quant_rows_kernel, dim3(grid), dim3(kQuantThreads), 0, st, a.pdl, a);
}

}  // namespace moe
