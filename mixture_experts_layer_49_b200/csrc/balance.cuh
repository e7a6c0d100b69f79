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

// P sums of the 32 experts e0 .. e0+31 in double, by a block of 32 warps.
// The order, for expert e: residue class w of rows (w, w + 32, w + 64, ...)
// summed in ascending row order, then the 32 class sums meet in a butterfly
// over w (addition is commutative, so every lane of the butterfly ends with
// the same value).  Warp w reads rows of class w, its lane l takes expert
// e0 + l, so every load is one 128-byte row segment; the class sums cross
// over through shared memory and warp w then returns expert e0 + w's sum.
// Every thread of the block must call it; red is a [32][33] shared array.
__device__ __forceinline__ double psum_block32(const float *psum, int nblk, int E, int e0, double (*red)[33]) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int e = e0 + lane;
    double s = 0.0;
    for (int b0 = w; b0 < nblk; b0 += 32 * 16) {     // sixteen independent loads in flight
        float v[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int b = b0 + 32 * j;
            v[j] = (b < nblk && e < E) ? psum[(size_t)b * E + e] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (b0 + 32 * j < nblk) s += (double)v[j];
    }
    red[w][lane] = s;
    __syncthreads();
    double t = red[lane][w];                         // lane = residue class, warp w = expert e0 + w
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    __syncthreads();                                 // red may be reused
    return t;
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
