// dispatch.cu -- per-expert counting, capacity, prefix sum and the stable
// permutation of tokens into expert-contiguous order.
//
// Counts are the bincount of the chosen expert ids ("Fine-Tuning Mixture of
// Experts (MoE) Models: Router Optimization Techniques", router module, step
// 5).  An expert keeps at most `capacity` assignments and drops the rest
// ("Mixture-of-Experts" post, expert-capacity paragraph); which ones are kept
// is not fixed by the pages: this library keeps the earliest tokens.  The
// rows are packed into one contiguous workspace per expert so the experts run
// as one grouped GEMM (Router Optimization page, What Most Articles Miss 2).
//
// Three kernels, all deterministic:
//   chunk_hist   one CTA per chunk of 64 tokens: shared-memory counts per expert
//   chunk_scan   one warp per expert: exclusive scan over chunks; counts and
//                kept = min(counts, capacity)
//   permute      one CTA per chunk: offsets = exclusive scan of kept (CTA 0
//                publishes them); the rank of (t, s) among the chunk's
//                assignments to the same expert comes from __match_any_sync
//                over flattened (t, s) order, so rows are stable by token id;
//                then, unless x_perm is null, each token's row of x is read
//                once and written to each of its kept rows (16-byte vectors).
#include "balance.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kChunk = 64;        // tokens per chunk
constexpr int kThreads = 256;
constexpr int kPermThreads = 512;            // permute: 16 warps share the row copies
constexpr int kWarps = kPermThreads / 32;

__global__ void __launch_bounds__(kThreads) chunk_hist_kernel(DispatchArgs a, int nchunks) {
    pdl_wait_then_release();
    __shared__ int cnt[256];
    const int c = blockIdx.x;
    for (int e = threadIdx.x; e < a.E; e += kThreads) cnt[e] = 0;
    __syncthreads();
    const int t0 = c * kChunk;
    const int ntok = min(kChunk, a.T - t0);
    const int npairs = ntok * a.k;
    const int32_t *idx = a.idx + (size_t)t0 * a.k;
    for (int p = threadIdx.x; p < npairs; p += kThreads) {
        const int e = idx[p];
        if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
        else record_error(a.status, MOE_ERR_DEVICE_BOUNDS, t0 * a.k + p);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += kThreads) a.chunk_cnt[(size_t)e * nchunks + c] = cnt[e];
}

// One warp per expert: exclusive scan of the expert's per-chunk counts (each
// lane first sums 8 consecutive chunks, then a warp scan of the lane totals),
// the expert's total count and its kept count.  Experts are independent, so
// the grid covers them 32 per CTA.  With balance outputs, the same warp
// computes f_e, P_e and the loss term f_e P_e (balance.cuh order, the score
// sums read as whole rows of the CTA's 32 experts); the permute kernel adds
// the terms.
__global__ void __launch_bounds__(1024) chunk_scan_kernel(DispatchArgs a, int nchunks) {
    pdl_wait_then_release();
    __shared__ double red[32][33];
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * 32 + (threadIdx.x >> 5);
    double psum_e = 0.0;
    const bool bal = a.loss != nullptr;                    // uniform over the grid
    if (bal) psum_e = psum_block32(a.psum, a.nblk, a.E, blockIdx.x * 32, red);
    if (e >= a.E) return;
    const int32_t *src = a.chunk_cnt + (size_t)e * nchunks;
    int32_t *dst = a.chunk_base + (size_t)e * nchunks;
    int running = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 256) {
        int v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c0 + lane * 8 + i;
            v[i] = c < nchunks ? src[c] : 0;
        }
        int tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) tot += v[i];
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        int run = running + incl - tot;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = c0 + lane * 8 + i;
            if (c < nchunks) dst[c] = run;
            run += v[i];
        }
        running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        a.counts[e] = running;
        a.kept[e] = (a.capacity >= 0 && running > a.capacity) ? a.capacity : running;
        if (bal) {
            const double P = psum_e / (double)a.T;
            const double f = (double)running / ((double)a.T * (double)a.k);
            a.f[e] = (float)f;
            a.P[e] = (float)P;
            a.contrib[e] = f * P;
        }
    }
}

template <typename TX>
__global__ void __launch_bounds__(kPermThreads) permute_kernel(DispatchArgs a, int nchunks) {
    pdl_wait_then_release();
    __shared__ int base[256];
    __shared__ int offs[256];
    __shared__ int wcnt[kWarps][256];
    __shared__ int2 list[kChunk * 32];           // (row, token) of each pair, k <= 32
    const int c = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E, k = a.k;
    for (int e = tid; e < E; e += kPermThreads) {
        base[e] = a.chunk_base[(size_t)e * nchunks + c];
        offs[e] = a.kept[e];
#pragma unroll
        for (int w = 0; w < kWarps; ++w) wcnt[w][e] = 0;
    }
    __syncthreads();
    if (warp == 0) {       // expert offsets: exclusive scan of kept (every CTA; CTA 0 publishes)
        int running = 0, dropped = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < E ? offs[e] : 0;
            const int dv = (c == 0 && e < E) ? a.counts[e] - v : 0;
            int incl = v, dincl = dv;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                const int dn = __shfl_up_sync(0xffffffffu, dincl, o);
                if (lane >= o) { incl += n; dincl += dn; }
            }
            if (e < E) {
                offs[e] = running + incl - v;
                if (c == 0) a.offsets[e] = running + incl - v;
            }
            running += __shfl_sync(0xffffffffu, incl, 31);
            dropped += __shfl_sync(0xffffffffu, dincl, 31);
        }
        if (c == 0 && lane == 0) {
            a.offsets[E] = running;
            if (a.n_dropped) *a.n_dropped = dropped;
        }
    } else if (warp == 1 && c == 0 && a.loss) {       // the balance loss from the scan's terms
        const double sum = loss_tree_warp(a.contrib, E);
        if (lane == 0) *a.loss = (double)E * sum;
    }
    __syncthreads();
    const int t0 = c * kChunk;
    const int npairs = min(kChunk, a.T - t0) * k;
    const int p_lo = warp * npairs / kWarps, p_hi = (warp + 1) * npairs / kWarps;
    const int32_t *idx = a.idx + (size_t)t0 * k;
    const unsigned lt_mask = (1u << lane) - 1u;

    // pass 1: per-warp counts over the warp's contiguous range of pairs
    for (int p0 = p_lo; p0 < p_hi; p0 += 32) {
        const int p = p0 + lane;
        const unsigned active = __ballot_sync(0xffffffffu, p < p_hi);
        if (p < p_hi) {
            int e = idx[p];
            if (e < 0 || e >= E) e = -1;
            const unsigned peers = __match_any_sync(active, e);
            if (e >= 0 && lane == __ffs(peers) - 1) wcnt[warp][e] += __popc(peers);
        }
        __syncwarp();
    }
    __syncthreads();
    // exclusive scan over warps, per expert
    for (int e = tid; e < E; e += kPermThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) { const int v = wcnt[w][e]; wcnt[w][e] = run; run += v; }
    }
    __syncthreads();
    // pass 2: final ranks, rows, drops
    for (int p0 = p_lo; p0 < p_hi; p0 += 32) {
        const int p = p0 + lane;
        const unsigned active = __ballot_sync(0xffffffffu, p < p_hi);
        int e = -1, rank = 0;
        unsigned peers = 0;
        if (p < p_hi) {
            e = idx[p];
            if (e < 0 || e >= E) e = -1;
            peers = __match_any_sync(active, e);
            if (e >= 0) rank = base[e] + wcnt[warp][e] + __popc(peers & lt_mask);
        }
        __syncwarp();
        if (p < p_hi && e >= 0 && lane == __ffs(peers) - 1) wcnt[warp][e] += __popc(peers);
        if (p < p_hi) {
            const int t = t0 + p / k;
            int row = -1;
            if (e >= 0 && (a.capacity < 0 || rank < a.capacity)) {
                row = offs[e] + rank;
                a.row_token[row] = t;
                a.row_gate[row] = a.gate[(size_t)t0 * k + p];
                if (a.row_scale) a.row_scale[row] = a.x_scale[t];
            }
            a.row_of[(size_t)t0 * k + p] = row;
            list[p] = make_int2(row, t);
        }
        __syncwarp();
    }
    if (a.x_perm == nullptr) return;             // row tables only
    __syncthreads();
    // copy x rows into x_perm: one warp per token, its row read once (eight
    // 16-byte loads in flight per lane) and written to each of its kept rows
    const int nvec = a.d * (int)sizeof(TX) / 16;
    const int ntok = min(kChunk, a.T - t0);
    const uint4 *xs = static_cast<const uint4 *>(a.x);
    uint4 *xd = static_cast<uint4 *>(a.x_perm);
    for (int tl = warp; tl < ntok; tl += kWarps) {
        const int my_row = lane < k ? list[tl * k + lane].x : -1;
        if (__ballot_sync(0xffffffffu, my_row >= 0) == 0u) continue;      // every slot dropped
        const uint4 *__restrict__ src = xs + (size_t)(t0 + tl) * nvec;
        // the loop bounds are the same for every lane (the slot rows come by
        // shuffle); lanes past the row's last vector load and store nothing
        for (int v0 = 0; v0 < nvec; v0 += 256) {
            uint4 r[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int v = v0 + 32 * i + lane;
                if (v < nvec) r[i] = __ldg(src + v);
            }
            for (int s = 0; s < k; ++s) {
                const int row = __shfl_sync(0xffffffffu, my_row, s);
                if (row < 0) continue;                                      // same row on every lane
                uint4 *__restrict__ dst = xd + (size_t)row * nvec;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int v = v0 + 32 * i + lane;
                    if (v < nvec) dst[v] = r[i];
                }
            }
        }
    }
}

__global__ void empty_offsets_kernel(DispatchArgs a) {
    pdl_wait_then_release();
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) a.offsets[e] = 0;
    if (threadIdx.x == 0 && a.n_dropped) *a.n_dropped = 0;
    if (a.loss && threadIdx.x < 32) {
        const double sum = loss_tree_warp(a.contrib, a.E);
        if (threadIdx.x == 0) *a.loss = (double)a.E * sum;
    }
}

}  // namespace

int dispatch_chunks(int T) { return (T + kChunk - 1) / kChunk; }

cudaError_t launch_dispatch(const DispatchArgs &a, int x_bytes, cudaStream_t st) {
    const int nchunks = dispatch_chunks(a.T);
    cudaError_t e = cudaSuccess;
    if (nchunks > 0) e = launch_kernel(chunk_hist_kernel, dim3(nchunks), dim3(kThreads), 0, st, a.pdl, a, nchunks);
    if (e != cudaSuccess) return e;
    e = launch_kernel(chunk_scan_kernel, dim3((a.E + 31) / 32), dim3(1024), 0, st, nchunks > 0 || a.pdl, a, nchunks);
    if (e != cudaSuccess) return e;
    if (nchunks == 0)             // no tokens: every count is zero, offsets all zero
        return launch_kernel(empty_offsets_kernel, dim3(1), dim3(256), 0, st, true, a);
    if (x_bytes == 1) return launch_kernel(permute_kernel<uint8_t>, dim3(nchunks), dim3(kPermThreads), 0, st, true, a, nchunks);
    if (x_bytes == 2) return launch_kernel(permute_kernel<__nv_bfloat16>, dim3(nchunks), dim3(kPermThreads), 0, st, true, a, nchunks);
    return launch_kernel(permute_kernel<float>, dim3(nchunks), dim3(kPermThreads), 0, st, true, a, nchunks);
}

}  // namespace moe
