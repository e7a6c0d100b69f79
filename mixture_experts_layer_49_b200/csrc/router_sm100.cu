// router_sm100.cu -- router GEMM, fp32 scores, top-k selection, gates and the
// per-block score sums for bf16 layers, on the tcgen05 tensor cores.
//
// "Mixture-of-Experts" (Vector Institute post), router section: one score per
// expert h = x W_r, softmax over the experts, the k best, gates from the full
// softmax (Eq. moe-output) or renormalised over the selected experts.
// "Fine-tuning and serving MoE models", How an MoE layer actually works, and
// the "Mixture of Experts" tutorial, Selective precision: the router runs in
// fp32 even when the layer is bf16.  "Fine-Tuning Mixture of Experts (MoE)
// Models: Router Optimization Techniques", How It Works 2: a per-expert bias
// steers the selection only.
//
// fp32 accuracy on bf16 tensor cores: x is bf16 already; W_r (fp32) is split
// exactly into three bf16 terms, W = hi + mid + lo (8 + 8 + 8 significand
// bits), so x W = x hi + x mid + x lo with every product exact.  The tensor
// core's fp32 accumulator rounds each K=16 step toward zero, a bias that grows
// with the number of steps, so K is split over up to 8 separate TMEM
// accumulators whose partial sums the epilogue adds in fp32 (round to
// nearest) before anything else reads the logits.
//
// One CTA pair (tcgen05.mma.cta_group::2) per 256 tokens and K range:
//   MMA M = 256 (128 tokens per CTA), N = E rounded up to 16 (each CTA loads
//   half of the rows of the three W_r terms), K = d_model or a slice of it.
//   When the tokens alone give fewer pairs than the GPU holds, K is split
//   over up to four pairs per token block; each writes its partial logits and
//   the selection kernel adds them in split order.
//   warp 0      TMA producer (both CTAs): x tile 128 x 64 and the CTA's half
//               of the three W_r terms per stage (128-byte swizzle)
//   warp 1      TMEM allocator (both CTAs) + single-thread MMA issuer (rank 0)
//   warps 2..5  epilogue, one thread per token: add the K-split accumulators
//               (and the logit offset in split 0), stage the row in shared
//               memory, then each warp stores its 32 rows as one contiguous
//               block with 16-byte vector stores
// Scores, top-k, gates and the per-block score sums then run in the
// warp-per-token selection kernel of router_topk.cu (a per-thread top-k over
// E values was instruction-bound here).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int RM = 128;                       // tokens per CTA
constexpr int RBK = 64;                       // K per stage
constexpr int kThreads = 192;
constexpr uint32_t A_BYTES = RM * RBK * 2;    // 16 KiB
constexpr int kSmemCap = 227 * 1024;
constexpr int kMaxStages = 8;
constexpr int kMaxSplits = 4;

struct TcRouterParams {
    const float *logit_bias;
    float *out;                // [splits][T][E] fp32 (one split: the logits)
    int32_t *status;
    int T, d, E;
    int n_pad;                 // MMA N
    int nparts;                // K-split inside the CTA: separate accumulators
    int pstride;               // TMEM columns between accumulators (>= n_pad, multiple of 32)
    int stages;
    int splits;                // K-split across CTA pairs
    int kb_per_split;
    int ld;                    // staging row stride in floats
    uint32_t b_bytes;          // one W_r term, this CTA's half: n_pad/2 x 64 bf16
    uint32_t idesc;
    uint32_t tmem_cols;
    uint64_t timeout_ns;
};

struct RouterTail {
    uint64_t full[kMaxStages];     // rank 0's collect both CTAs' bytes
    uint64_t empty[kMaxStages];
    uint64_t accf;
    uint32_t tmem_base;
    int abort_flag;
};

// W_r [d, E] fp32 -> three bf16 matrices [3][E][d] (K-major), w = hi + mid + lo.
__global__ void __launch_bounds__(256) split_router_weights(const float *__restrict__ Wr, int d, int E,
                                                            __nv_bfloat16 *__restrict__ out) {
    pdl_wait_then_release();
    __shared__ float tile[32][33];
    const int j0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) {
        const int j = j0 + r, e = e0 + tx;
        tile[r][tx] = (j < d && e < E) ? Wr[(size_t)j * E + e] : 0.f;
    }
    __syncthreads();
    const size_t plane = (size_t)E * d;
    for (int r = ty; r < 32; r += 8) {
        const int e = e0 + r, j = j0 + tx;
        if (e < E && j < d) {
            const float w = tile[tx][r];
            const __nv_bfloat16 hi = __float2bfloat16_rn(w);
            const float r1 = w - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(mid);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
            const size_t o = (size_t)e * d + j;
            out[o] = hi;
            out[plane + o] = mid;
            out[2 * plane + o] = lo;
        }
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const TcRouterParams p) {
    pdl_wait_then_release();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    const uint32_t stage_bytes = A_BYTES + 3u * p.b_bytes;
    RouterTail &s = *reinterpret_cast<RouterTail *>(smem + p.stages * stage_bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int cl = (int)cluster_id_x();
    const int split = cl % p.splits;
    const int t0 = (cl / p.splits) * (2 * RM) + (int)rank * RM;
    const int nk = (p.d + RBK - 1) / RBK;
    const int kb0 = split * p.kb_per_split;
    const int kb1 = min(nk, kb0 + p.kb_per_split);
    // K steps kb0 .. kb1-1 in np contiguous parts (one accumulator each).
    // Pairs start at different parts (rotation by cluster index), so pairs
    // running together read different W_r tiles instead of all hitting the
    // same L2 lines; each part is still summed in ascending K order, so the
    // result does not depend on the rotation.
    const int nkl = kb1 - kb0;
    const int np = min(p.nparts, nkl);
    const int rot = cl % np;
    auto part_begin = [&](int part) { return (part * nkl + np - 1) / np; };

    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < p.stages; ++i) { mbar_init(smem_u32(&s.full[i]), 1); mbar_init(smem_u32(&s.empty[i]), 1); }
        mbar_init(smem_u32(&s.accf), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(&s.tmem_base), p.tmem_cols);
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int pp = 0; pp < np && ok; ++pp) {
                const int part = (pp + rot) % np;
                for (int i = part_begin(part); i < part_begin(part + 1); ++i) {
                    const int kb = kb0 + i;
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) {
                        record_error(p.status, MOE_ERR_TIMEOUT, 11);
                        s.abort_flag = 1;
                        ok = false;
                        break;
                    }
                    const uint32_t fb = mapa_shared(smem_u32(&s.full[stage]), 0);
                    const uint32_t st = base + stage * stage_bytes;
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&s.full[stage]), 2 * stage_bytes);
                    tma_load_2d_pair(st, &tmX, fb, kb * RBK, t0);
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        tma_load_3d_pair(st + A_BYTES + j * p.b_bytes, &tmW, fb, kb * RBK, (int)rank * (p.n_pad / 2), j);
                    if (++stage == p.stages) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int pp = 0; pp < np && ok; ++pp) {
                const int part = (pp + rot) % np;
                const uint32_t dtm = tmem + (uint32_t)(part * p.pstride);
                for (int i = part_begin(part); i < part_begin(part + 1); ++i) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns)) {
                        record_error(p.status, MOE_ERR_TIMEOUT, 12);
                        s.abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = base + stage * stage_bytes;
                    const uint32_t fresh = i == part_begin(part);   // the part's first K step starts its sum
#pragma unroll
                    for (int j = 0; j < 3; ++j)
#pragma unroll
                        for (int k = 0; k < RBK / 16; ++k)
                            mma_bf16_pair(dtm, sdesc(st + k * 32), sdesc(st + A_BYTES + j * p.b_bytes + k * 32),
                                          p.idesc, (fresh && j == 0 && k == 0) ? 0u : 1u);
                    mma_commit_pair(smem_u32(&s.empty[stage]), (uint16_t)0x3);
                    if (++stage == p.stages) { stage = 0; phase ^= 1u; }
                }
            }
            if (ok) mma_commit_pair(smem_u32(&s.accf), (uint16_t)0x3);
        }
    } else {
        const int q = warp & 3;
        const int row0 = t0 + q * 32;                     // the warp's first token
        int ok = 1;
        if (lane == 0) ok = mbar_wait(smem_u32(&s.accf), 0, p.timeout_ns) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
            if (lane == 0) { record_error(p.status, MOE_ERR_TIMEOUT, 13); s.abort_flag = 1; }
        } else {
            __syncwarp();
            tc_fence_after();
            // every MMA has completed, so the stage buffers are free: the warp
            // stages its 32 rows there (row stride ld floats)
            const int E = p.E, ld = p.ld;
            float *stg = reinterpret_cast<float *>(smem) + (size_t)q * 32 * ld;
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16);
            // 16-byte vectors need E % 4 == 0 and a 16-byte aligned output
            const bool vec = (E & 3) == 0 && (reinterpret_cast<uintptr_t>(p.out) & 15u) == 0;
            const bool add_bias = split == 0 && p.logit_bias != nullptr;
            for (int c = 0; c < (E + 31) / 32; ++c) {
                float v[32];
                __syncwarp();
                tmem_ld32(taddr + c * 32, v);
                for (int r = 1; r < np; ++r) {             // fixed order: parts 0, 1, 2, ...
                    float w[32];
                    tmem_ld32(taddr + r * p.pstride + c * 32, w);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] += w[j];
                }
                if (add_bias) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c * 32 + j < E) v[j] += __ldg(p.logit_bias + c * 32 + j);
                }
                float *dst = stg + (size_t)lane * ld + c * 32;
                if (vec) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        if (c * 32 + j < E) *reinterpret_cast<float4 *>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c * 32 + j < E) dst[j] = v[j];
                }
            }
            __syncwarp();
            // the warp's rows are contiguous in the output: copy them as one block
            const int nrows = max(0, min(32, p.T - row0));
            float *out = p.out + ((size_t)split * p.T + row0) * E;
            const int n = nrows * E;
            if (vec) {
                for (int f = lane * 4; f < n; f += 128) {
                    const int r = f / E, col = f - r * E;
                    *reinterpret_cast<float4 *>(out + f) = *reinterpret_cast<const float4 *>(stg + (size_t)r * ld + col);
                }
            } else {
                for (int f = lane; f < n; f += 32) {
                    const int r = f / E, col = f - r * E;
                    out[f] = stg[(size_t)r * ld + col];
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();                                  // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem, p.tmem_cols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode(CUtensorMap *m, int rank, const void *base, const cuuint64_t *dims, const cuuint64_t *strides,
            const cuuint32_t *box) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pairs of 256 tokens; the K-split count multiplies them up to the number of
// pairs the GPU holds at once, at most kMaxSplits and at most one split per
// two 64-deep K steps.
int pair_blocks(int T) { return (T + 2 * RM - 1) / (2 * RM); }

}  // namespace

int router_logit_splits_max(int T) {
    const int pairs = pair_blocks(T);
    if (pairs <= 0) return 1;
    const int s = 128 / pairs;
    return s < 1 ? 1 : (s > kMaxSplits ? kMaxSplits : s);
}

int router_logit_splits(int T, int d, int num_sms) {
    const int pairs = pair_blocks(T);
    if (pairs <= 0) return 1;
    int s = (num_sms / 2) / pairs;
    const int nk = (d + RBK - 1) / RBK;
    if (s > nk / 2) s = nk / 2;
    const int cap = router_logit_splits_max(T);
    if (s > cap) s = cap;
    return s < 1 ? 1 : s;
}

size_t router_split_bytes(int d, int E) { return (size_t)3 * E * d * 2; }

// Logits h = x W_r (+ logit offset) into `out`: [splits][T][E] partial sums.
cudaError_t launch_router_split(const RouterArgs &a, cudaStream_t st) {
    dim3 sg((a.d + 31) / 32, (a.E + 31) / 32);
    return launch_kernel(split_router_weights, sg, dim3(256), 0, st, a.pdl, a.Wr, a.d, a.E,
                         static_cast<__nv_bfloat16 *>(a.wsplit));
}

cudaError_t launch_router_logits_tc(const RouterArgs &a, float *out, int splits, cudaStream_t st) {
    void *wsplit = a.wsplit;
    if (a.T == 0) return cudaSuccess;
    cudaError_t e = cudaSuccess;
    if (!a.split_ready && (e = launch_router_split(a, st)) != cudaSuccess) return e;

    TcRouterParams p{};
    p.logit_bias = a.logit_bias; p.out = out; p.status = a.status;
    p.T = a.T; p.d = a.d; p.E = a.E;
    p.n_pad = (a.E + 15) / 16 * 16;
    p.b_bytes = (uint32_t)(p.n_pad / 2) * RBK * 2;
    p.idesc = make_idesc_bf16(2 * RM, (uint32_t)p.n_pad);
    p.pstride = (p.n_pad + 31) / 32 * 32;
    const int nk = (a.d + RBK - 1) / RBK;
    p.splits = splits;
    p.kb_per_split = (nk + splits - 1) / splits;
    const int nkl = p.kb_per_split;
    int nparts = 512 / p.pstride;
    if (nparts > 8) nparts = 8;
    if (nparts > nkl) nparts = nkl;
    p.nparts = nparts;
    uint32_t cols = 32;
    while ((int)cols < p.nparts * p.pstride) cols <<= 1;
    p.tmem_cols = cols;
    p.timeout_ns = 2000000000ull;
    p.ld = (a.E & 3) == 0 ? a.E + 4 : a.E + 1;
    const size_t stage_bytes = A_BYTES + 3 * (size_t)p.b_bytes;
    const size_t fixed = 1024 + sizeof(RouterTail);
    int stages = (int)((kSmemCap - fixed) / stage_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return cudaErrorInvalidValue;
    // the epilogue stages 128 rows of ld floats in the stage buffers
    const size_t staging = (size_t)RM * p.ld * 4;
    if (staging > (size_t)stages * stage_bytes) return cudaErrorInvalidValue;
    p.stages = stages;
    const size_t smem = fixed + stages * stage_bytes;
    // every split must own at least one K step
    if ((size_t)(splits - 1) * p.kb_per_split >= (size_t)nk) return cudaErrorInvalidValue;

    CUtensorMap mx, mw;
    const cuuint64_t xd[2] = {(cuuint64_t)a.d, (cuuint64_t)a.T};
    const cuuint64_t xs[1] = {(cuuint64_t)a.d * 2};
    const cuuint32_t xb[2] = {RBK, RM};
    if (!encode(&mx, 2, a.x, xd, xs, xb)) return cudaErrorInvalidValue;
    const cuuint64_t wd[3] = {(cuuint64_t)a.d, (cuuint64_t)a.E, 3};
    const cuuint64_t wst[2] = {(cuuint64_t)a.d * 2, (cuuint64_t)a.E * a.d * 2};
    const cuuint32_t wb[3] = {RBK, (cuuint32_t)(p.n_pad / 2), 1};
    if (!encode(&mw, 3, wsplit, wd, wst, wb)) return cudaErrorInvalidValue;

    static bool attr = false;
    if (!attr) {
        e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemCap);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    const int grid = 2 * pair_blocks(a.T) * splits;
    return launch_kernel(router_tc_kernel, dim3(grid), dim3(kThreads), smem, st, a.split_ready ? a.pdl : true, mx, mw,
                         p);
}

}  // namespace moe
