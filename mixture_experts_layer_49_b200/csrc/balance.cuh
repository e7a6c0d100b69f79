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
    int b = lane;
    for (; b + 96 < nblk; b += 128) {           // four independent loads in flight
        const float v0 = psum[(size_t)b * E + e];
        const float v1 = psum[(size_t)(b + 32) * E + e];
        const float v2 = psum[(size_t)(b + 64) * E + e];
        const float v3 = psum[(size_t)(b + 96) * E + e];
        s += (double)v0; s += (double)v1; s += (double)v2; s += (double)v3;
    }
    for (; b < nblk; b += 32) s += (double)psum[(size_t)b * E + e];
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

}  // namespace moe
