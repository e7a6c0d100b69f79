// balance.cuh -- the one reduction order of the balance statistics, shared by
// the standalone balance kernel and the dispatch scan that computes them in
// the forward pass, so both give the same bits.
//
// f_e = counts_e / (T k), P_e = mean over tokens of the normalised score,
// L = E sum_e f_e P_e (Vector Institute post, Eq. balance; Router Optimization
// page, How It Works 1).  The router leaves per-block partial sums of the
// normalised scores in psum [nblk, E].
#pragma once

#include "common.cuh"

namespace moe {

// Column e of psum summed in double by one warp: lane l adds rows l, l + 32,
// l + 64, ... in order, then the 32 lane sums meet in a butterfly (addition
// is commutative, so every lane ends with the same value).
__device__ __forceinline__ double psum_column(const float *psum, int nblk, int E, int e) {
    const int lane = threadIdx.x & 31;
    double s = 0.0;
    for (int b0 = 0; b0 < nblk; b0 += 32 * 16) {   // sixteen independent loads in flight
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int b = b0 + lane + 32 * j;
            v[j] = b < nblk ? psum[(size_t)b * E + e] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (b0 + lane + 32 * j < nblk) s += (double)v[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// The loss from the per-expert terms f_e P_e in red[0..255] (zero past E):
// a fixed halving tree over 256 entries, run by the first 256 threads of the
// block; every thread of the block must call it.
__device__ __forceinline__ double loss_tree(double *red) {
    for (int o = 128; o > 0; o >>= 1) {
        __syncthreads();
        if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    }
    __syncthreads();
    return red[0];
}

// The same tree run by one warp over contrib[0..E) (zero past E): lane l
// holds entries l + 32 j; the halving steps 128, 64, 32 are register adds in
// the same operand order, 16 .. 1 are shuffles.  Every lane returns lane 0's
// value, which equals loss_tree's bit for bit.
__device__ __forceinline__ double loss_tree_warp(const double *contrib, int E) {
    const int lane = threadIdx.x & 31;
    double v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = lane + 32 * j < E ? contrib[lane + 32 * j] : 0.0;
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] += v[j + 4];
#pragma unroll
    for (int j = 0; j < 2; ++j) v[j] += v[j + 2];
    v[0] += v[1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[0] += __shfl_down_sync(0xffffffffu, v[0], o);
    return __shfl_sync(0xffffffffu, v[0], 0);
}

}  // namespace moe
