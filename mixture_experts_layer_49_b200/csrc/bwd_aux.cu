// bwd_aux.cu -- the memory-bound and per-token steps of the layer's backward
// pass (the contractions run in bwd_sm100.cu).
//
// For the loss ell = sum_t <dy_t, y_t> + alpha * L_aux (the task gradient dy
// of the layer output plus the weighted balance loss, "Fine-Tuning Mixture of
// Experts (MoE) Models: Router Optimization Techniques", How It Works 1):
//   scale_rows       dZ[r] = gate[r] * dy[token(r)]: the gradient of the
//                    gated expert output of every packed row (bf16)
//   router_bwd       per token: the gate gradients dg_s = <dy_t, E_e(x_t)>
//                    (from the partial dot products the down-projection
//                    dgrad leaves, divided by the gate), through the gate
//                    normalisation (full softmax, softmax over the selected
//                    logits, or normalised sigmoid) to the logits, plus the
//                    balance-loss term through P: dh [T, E] (fp32 and bf16)
//   column_sums      per group and column, the sum over the group's rows (in
//                    row order): bias gradients, and d(logit offset)
//   dx_combine       dx_t = the packed rows' input gradients in slot order
//                    + the shared expert's + the router's, one rounding
//   to_bf16          W_r as bf16 (the router's input-gradient GEMM operand)
// Expert selection and capacity are piecewise constant and carry no gradient.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

// dZ[r, :] = gate[r] * dy[row_token[r], :] for r < offsets[E] (rows past the
// device count are left alone).  One warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256) scale_rows_kernel(BwdAuxArgs a) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    const int64_t nrows = a.offsets[a.E];
    const int nvec = a.d / 8;
    const int64_t nwarps = (int64_t)gridDim.x * 8;
    for (int64_t r = blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows; r += nwarps) {
        const int t = a.row_token[r];
        const float g = a.row_gate[r];
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.dy) + (int64_t)t * a.d);
        uint4 *dst = reinterpret_cast<uint4 *>(a.dZ + r * a.d);
        for (int v = lane; v < nvec; v += 32) {
            uint4 in = __ldg(src + v), out;
            const __nv_bfloat162 *hi = reinterpret_cast<const __nv_bfloat162 *>(&in);
            __nv_bfloat162 *ho = reinterpret_cast<__nv_bfloat162 *>(&out);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(hi[i]);
                ho[i] = __floats2bfloat162_rn(g * f.x, g * f.y);
            }
            dst[v] = out;
        }
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The score of expert e, held by lane e % 32 in register e / 32, to every lane.
template <int EPL>
__device__ __forceinline__ float score_of(const float (&sc)[EPL], int e) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const float t = __shfl_sync(0xffffffffu, sc[i], e & 31);
        if (i == (e >> 5)) v = t;
    }
    return v;
}

// One warp per token; expert e lives in lane e % 32, register e / 32.
template <int EPL>
__global__ void __launch_bounds__(256) router_bwd_kernel(BwdAuxArgs a) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= a.T) return;
    const int E = a.E, k = a.k;
    float h[EPL], sc[EPL], dh[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        h[i] = e < E ? a.logits[(int64_t)t * E + e] : -INFINITY;
        dh[i] = 0.f;
    }
    // scores: softmax p, or sigmoid s
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) mx = fmaxf(mx, h[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float norm = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        if (a.score == MOE_SCORE_SOFTMAX) sc[i] = e < E ? __expf(h[i] - mx) : 0.f;
        else sc[i] = e < E ? 1.f / (1.f + __expf(-h[i])) : 0.f;
        norm += sc[i];
    }
    norm = warp_sum(norm);
    if (a.score == MOE_SCORE_SOFTMAX) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) sc[i] /= norm;
    }
    // gate gradients of the slots (lane s holds slot s)
    float dgs = 0.f, gs = 0.f;
    int es = -1;
    for (int s = 0; s < k; ++s) {
        const int row = a.row_of[(int64_t)t * k + s];
        const int e = a.idx[(int64_t)t * k + s];
        const float g = a.gate[(int64_t)t * k + s];
        float dg = 0.f;
        if (row >= 0) {
            float acc = 0.f;
            for (int j = lane; j < a.part_ld; j += 32) acc += a.part[(int64_t)row * a.part_ld + j];
            acc = warp_sum(acc);
            dg = g != 0.f ? acc / g : 0.f;
            if (a.b2) {            // GELU experts: the output bias adds <dy_t, b2_e>
                float bb = 0.f;
                const __nv_bfloat16 *dyt = static_cast<const __nv_bfloat16 *>(a.dy) + (int64_t)t * a.d;
                for (int j = lane; j < a.d; j += 32) bb += __bfloat162float(dyt[j]) * a.b2[(int64_t)e * a.d + j];
                dg += warp_sum(bb);
            }
        }
        if (lane == s) { dgs = dg; gs = g; es = e; }
    }
    // through the gate normalisation
    const bool in_slot = lane < k;
    if (a.score == MOE_SCORE_SOFTMAX && a.renorm == 0) {
        // g_s = p_{e_s}: dh = p (dp - <dp, p>), dp_e = sum of dg over slots choosing e
        float dot = 0.f;
        for (int s = 0; s < k; ++s) {
            const int e = __shfl_sync(0xffffffffu, es, s);
            const float dg = __shfl_sync(0xffffffffu, dgs, s);
            const float pv = score_of(sc, e);
            dot += pv * dg;
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i * 32 + lane == e) dh[i] += pv * dg;
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) dh[i] -= sc[i] * dot;
    } else if (a.score == MOE_SCORE_SOFTMAX) {
        // renormalised over the selection: dh_sel = g (dg - <dg, g>)
        const float dot = warp_sum(in_slot ? gs * dgs : 0.f);
        for (int s = 0; s < k; ++s) {
            const int e = __shfl_sync(0xffffffffu, es, s);
            const float v = __shfl_sync(0xffffffffu, gs * (dgs - dot), s);
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i * 32 + lane == e) dh[i] += v;
        }
    } else {
        // sigmoid: g_s = s_{e_s} / S_sel: ds_sel = (dg - <dg, g>) / S_sel, dh = ds s (1 - s)
        const float dot = warp_sum(in_slot ? gs * dgs : 0.f);
        float ssel = 0.f;
        for (int s = 0; s < k; ++s) ssel += score_of(sc, __shfl_sync(0xffffffffu, es, s));
        for (int s = 0; s < k; ++s) {
            const int e = __shfl_sync(0xffffffffu, es, s);
            const float v = __shfl_sync(0xffffffffu, (dgs - dot) / ssel, s);
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i * 32 + lane == e) dh[i] += v * sc[i] * (1.f - sc[i]);
        }
    }
    // balance loss through P: c_e = alpha E f_e / T, pnorm = p (softmax) or s / S_all
    if (a.alpha != 0.f) {
        const float inv_T = 1.f / (float)a.T;
        float cv[EPL], cq = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = i * 32 + lane;
            const float f = e < E ? (float)a.counts[e] / ((float)a.T * (float)k) : 0.f;
            cv[i] = a.alpha * (float)E * f * inv_T;
            const float q = a.score == MOE_SCORE_SOFTMAX ? sc[i] : sc[i] / norm;
            cq += cv[i] * q;
        }
        cq = warp_sum(cq);
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (a.score == MOE_SCORE_SOFTMAX) dh[i] += sc[i] * (cv[i] - cq);
            else dh[i] += (cv[i] - cq) / norm * sc[i] * (1.f - sc[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        if (e < E) {
            a.dh[(int64_t)t * E + e] = dh[i];
            a.dh_bf16[(int64_t)t * a.dh_ld + e] = __float2bfloat16_rn(dh[i]);
        }
    }
}

// out[g][c] = sum over rows r of group g (ascending) of in[r][c] (bf16 rows,
// row stride ld) -- or of fp32 rows when in_f32.  One thread per (group,
// column); consecutive threads take consecutive columns.
__global__ void __launch_bounds__(256) column_sums_kernel(ColSumArgs a) {
    pdl_wait_then_release();
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= (int64_t)a.G * a.cols) return;
    const int g = (int)(i / a.cols), c = (int)(i % a.cols);
    const int r0 = a.offsets ? a.offsets[g] : 0;
    const int r1 = a.offsets ? a.offsets[g + 1] : a.rows;
    float acc = 0.f;
    if (a.in_f32) {
        const float *in = static_cast<const float *>(a.in);
        for (int r = r0; r < r1; ++r) acc += in[(int64_t)r * a.ld + c];
    } else {
        const __nv_bfloat16 *in = static_cast<const __nv_bfloat16 *>(a.in);
        for (int r = r0; r < r1; ++r) acc += __bfloat162float(in[(int64_t)r * a.ld + c]);
    }
    a.out[(int64_t)g * a.cols + c] = acc;
}

// Column sums of an fp32 [rows][cols] array in two deterministic passes:
// pass 1, block (rb, cb) sums rows rb*256 .. rb*256+255 of its 256 columns
// (thread per column, rows in order) into part[rb][c]; pass 2 sums the parts
// of each column in block order.
__global__ void __launch_bounds__(256) col_partials_kernel(const float *in, int64_t rows, int cols, int64_t ld,
                                                           float *part) {
    pdl_wait_then_release();
    const int c = blockIdx.y * 256 + threadIdx.x;
    if (c >= cols) return;
    const int64_t r0 = (int64_t)blockIdx.x * 256;
    const int64_t r1 = r0 + 256 < rows ? r0 + 256 : rows;
    float acc = 0.f;
    for (int64_t r = r0; r < r1; ++r) acc += in[r * ld + c];
    part[(int64_t)blockIdx.x * cols + c] = acc;
}

__global__ void __launch_bounds__(256) col_finish_kernel(const float *part, int nparts, int cols, float *out) {
    pdl_wait_then_release();
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c >= cols) return;
    float acc = 0.f;
    for (int b = 0; b < nparts; ++b) acc += part[(int64_t)b * cols + c];
    out[c] = acc;
}

// dx[t] = sum_s dX_rows[row_of[t, s]] (slot order) + dX_shared[t] + dX_router[t]
__global__ void __launch_bounds__(256) dx_combine_kernel(BwdAuxArgs a) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * 8;
    const int nvec = a.d / 4;
    for (int t = blockIdx.x * 8 + (threadIdx.x >> 5); t < a.T; t += nwarps) {
        int my_row = -1;
        if (lane < a.k) my_row = a.row_of[(int64_t)t * a.k + lane];
        for (int v0 = 0; v0 < nvec; v0 += 32) {
            const int v = v0 + lane;
            const bool in_row = v < nvec;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int s = 0; s < a.k; ++s) {
                const int r = __shfl_sync(0xffffffffu, my_row, s);
                if (in_row && r >= 0) {       // four bf16 values of the packed row
                    const uint2 x = __ldg(reinterpret_cast<const uint2 *>(a.dX_rows + (int64_t)r * a.d) + v);
                    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.x));
                    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x.y));
                    acc.x += lo.x; acc.y += lo.y; acc.z += hi.x; acc.w += hi.y;
                }
            }
            if (!in_row) continue;
            if (a.dX_shared) {
                const float4 x = __ldg(reinterpret_cast<const float4 *>(a.dX_shared + (int64_t)t * a.d) + v);
                acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
            }
            const float4 x = __ldg(reinterpret_cast<const float4 *>(a.dX_router + (int64_t)t * a.d) + v);
            acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
            __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(static_cast<__nv_bfloat16 *>(a.dx) + (int64_t)t * a.d) + 2 * v;
            o[0] = __floats2bfloat162_rn(acc.x, acc.y);
            o[1] = __floats2bfloat162_rn(acc.z, acc.w);
        }
    }
}

// out[r][c] = bf16(in[r][c]) for a fp32 [rows][cols] array, out row stride ldo
__global__ void __launch_bounds__(256) to_bf16_kernel(const float *in, __nv_bfloat16 *out, int64_t rows, int cols,
                                                      int64_t ldo) {
    pdl_wait_then_release();
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (i >= rows * cols) return;
    const int64_t r = i / cols;
    const int c = (int)(i % cols);
    out[r * ldo + c] = __float2bfloat16_rn(in[i]);
}

__global__ void set_pair_kernel(int32_t *p, int32_t a, int32_t b) {
    pdl_wait_then_release();
    if (threadIdx.x == 0) { p[0] = a; p[1] = b; }
}

int blocks_for(int64_t n, int per, int cap) {
    int64_t b = (n + per - 1) / per;
    if (b < 1) b = 1;
    return (int)(b > cap ? cap : b);
}

}  // namespace

cudaError_t launch_scale_rows(const BwdAuxArgs &a, int max_rows, cudaStream_t st) {
    return launch_kernel(scale_rows_kernel, dim3(blocks_for(max_rows, 8, a.num_sms * 8)), dim3(256), 0, st, true, a);
}

cudaError_t launch_router_bwd(const BwdAuxArgs &a, cudaStream_t st) {
    const dim3 grid((unsigned)((a.T + 7) / 8));
    if (a.E <= 32) return launch_kernel(router_bwd_kernel<1>, grid, dim3(256), 0, st, true, a);
    if (a.E <= 64) return launch_kernel(router_bwd_kernel<2>, grid, dim3(256), 0, st, true, a);
    if (a.E <= 128) return launch_kernel(router_bwd_kernel<4>, grid, dim3(256), 0, st, true, a);
    return launch_kernel(router_bwd_kernel<8>, grid, dim3(256), 0, st, true, a);
}

cudaError_t launch_column_sums(const ColSumArgs &a, cudaStream_t st) {
    const int64_t n = (int64_t)a.G * a.cols;
    if (n == 0) return cudaSuccess;
    return launch_kernel(column_sums_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true, a);
}

cudaError_t launch_dx_combine(const BwdAuxArgs &a, cudaStream_t st) {
    return launch_kernel(dx_combine_kernel, dim3(blocks_for(a.T, 8, a.num_sms * 8)), dim3(256), 0, st, true, a);
}

cudaError_t launch_set_pair(int32_t *p, int32_t a, int32_t b, cudaStream_t st) {
    return launch_kernel(set_pair_kernel, dim3(1), dim3(32), 0, st, true, p, a, b);
}

cudaError_t launch_col_sums_2pass(const float *in, int64_t rows, int cols, int64_t ld, float *part, float *out,
                                  cudaStream_t st) {
    if (rows == 0 || cols == 0) return cudaSuccess;
    const int nparts = (int)((rows + 255) / 256);
    cudaError_t e = launch_kernel(col_partials_kernel, dim3((unsigned)nparts, (unsigned)((cols + 255) / 256)), dim3(256),
                                  0, st, true, in, rows, cols, ld, part);
    if (e != cudaSuccess) return e;
    return launch_kernel(col_finish_kernel, dim3((unsigned)((cols + 255) / 256)), dim3(256), 0, st, true, part, nparts,
                         cols, out);
}

cudaError_t launch_to_bf16(const float *in, __nv_bfloat16 *out, int64_t rows, int cols, int64_t ldo, cudaStream_t st) {
    const int64_t n = rows * cols;
    if (n == 0) return cudaSuccess;
    return launch_kernel(to_bf16_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true, in, out, rows, cols,
                         ldo);
}

}  // namespace moe
