// bwd_sm100.cu -- the grouped GEMMs of the layer's backward pass on the
// 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// The backward pass of the MoE layer (chain rule on the forward definitions:
// expert FFNs from "Fine-tuning and serving MoE models", How an MoE layer
// actually works, and "Fine-Tuning Mixture of Experts (MoE) Models: Router
// Optimization Techniques", What Is It?; the router and its auxiliary loss
// from How It Works 1) consists of contractions whose operands sit in memory
// in both orientations:
//   recompute    G | U = X W_g^T | X W_u^T           A rows, B = weights (K-major both)
//   dgrad, down  dH    = dZ W_d                      B = W_d [d, F] read along its rows:
//                                                    MN-major B
//   dgrad, up    dX    = dG W_g + dU W_u             MN-major B, K split over W_g / W_u
//   wgrad        dW_d  = dZ^T H,  dW_g = dG^T X, ... both operands MN-major, the
//                                                    contraction runs over each
//                                                    expert's rows
// tcgen05.mma reads either orientation from shared memory (the instruction
// descriptor's transpose bits, and the matrix descriptor's leading / stride
// byte offsets), so no operand is ever transposed in memory.
//
// One persistent kernel (one CTA per SM, 352 threads) serves every form:
//   warp 0      TMA producer: A 128 x 64, B 256 x 64 per stage (4 stages of
//               48 KiB).  K-major operands come as one box per operand (64
//               elements of K per 128-byte swizzled row); MN-major operands as
//               64-element-wide boxes of 64 K rows (128-byte rows of MN, 8-row
//               swizzle atoms), 2 for A and 4 for B
//   warp 1      single-thread tcgen05.mma issuer (M = 128, N = 256, K = 16),
//               two 256-column fp32 TMEM accumulators
//   warps 2-9   epilogue: TMEM -> registers, then the form's store
//   warp 10     (groups that split K) zeroes the rows of the last K block
//               that lie past the group's rows, in both operands, before the
//               MMA reads them (the rows beyond belong to another expert)
// Groups: the rows of group g are offsets[g] .. offsets[g+1] (device array).
// Either the groups split M (the rows of A and of the output, K fixed) or
// they split K (each group's rows are the contraction, M and N fixed, one
// output matrix per group).  Every mbarrier wait is bounded; a wait that runs
// out records MOE_ERR_TIMEOUT and the CTA unwinds.  No TMA multicast.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int kThreads = 352;
constexpr uint32_t A_BYTES = BM * BK * 2;          // 16 KiB
constexpr uint32_t B_BYTES = BN * BK * 2;          // 32 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t CHUNK_BYTES = 64 * 128;         // one 64 x 64 MN-major box
constexpr uint32_t TMEM_COLS = 512;
constexpr int kMaxGroups = 257;

// Shared-memory descriptor of an MN-major operand with 128-byte swizzle: the
// MN extent comes in 64-element (128-byte) chunks CHUNK_BYTES apart (leading
// byte offset), K in 8-row swizzle atoms 1024 bytes apart (stride byte offset).
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(CHUNK_BYTES >> 4) << 16;      // LBO: next 64-element MN chunk
    d |= (uint64_t)(1024 >> 4) << 32;             // SBO: next 8 K rows
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;                       // SWIZZLE_128B
    return d;
}

struct SmemB {
    uint64_t full[STAGES];
    uint64_t ready[STAGES];      // groups that split K: the last block's rows masked
    uint64_t empty[STAGES];
    uint64_t accf[2];
    uint64_t acce[2];
    uint64_t drain;              // the MMA thread's last commit: every MMA done before TMEM is freed
    uint32_t tmem_base;
    int abort_flag;
    int tile_start[kMaxGroups + 1];
    int mtiles[kMaxGroups];
    int order[kMaxGroups];       // group of each position in the tile order
};
constexpr size_t kSmemBytes = 1024 + STAGES * STAGE_BYTES + sizeof(SmemB);
static_assert(kSmemBytes <= 227 * 1024, "backward GEMM shared memory");

__device__ __forceinline__ bool aborted(const SmemB &s) {
    return *reinterpret_cast<const volatile int *>(&s.abort_flag) != 0;
}
__device__ __forceinline__ void fail(SmemB &s, const BwdGemmParams &p, int where) {
    record_error(p.status, MOE_ERR_TIMEOUT, where);
    *reinterpret_cast<volatile int *>(&s.abort_flag) = 1;
}

// tile_start and mtiles are indexed by position in the tile order; order[]
// maps a position to its group.
__device__ __forceinline__ void decode(const SmemB &s, int G, int tile, int &g, int &mt, int &nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int local = tile - s.tile_start[lo];
    mt = local % s.mtiles[lo];
    nt = local / s.mtiles[lo];
    g = s.order[lo];
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmB2, const BwdGemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    SmemB &s = *reinterpret_cast<SmemB *>(smem + STAGES * STAGE_BYTES);
    const uint32_t smA = base;
    const uint32_t smB = base + STAGES * A_BYTES;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = p.G;
    constexpr uint32_t kIdesc = make_idesc_bf16(BM, BN) | (A_MN ? (1u << 15) : 0u) | (B_MN ? (1u << 16) : 0u);

    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.ready[i]), 1);
            mbar_init(smem_u32(&s.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&s.accf[i]), 1); mbar_init(smem_u32(&s.acce[i]), 8); }
        mbar_init(smem_u32(&s.drain), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&s.tmem_base), TMEM_COLS);
    pdl_wait_then_release();
    if (tid == 0) s.tile_start[0] = 0;
    // tile order: groups that split K go largest first (every tile of a group
    // costs its K, so the longest tiles start first); groups that split M
    // keep their order.  Position of group g: the number of groups ahead of it.
    for (int g = tid; g < G; g += kThreads) {
        int pos = g;
        if (p.kgroup) {
            const int rg = p.offsets[g + 1] - p.offsets[g];
            pos = 0;
            for (int h = 0; h < G; ++h) {
                const int rh = p.offsets[h + 1] - p.offsets[h];
                pos += (rh > rg || (rh == rg && h < g)) ? 1 : 0;
            }
        }
        s.order[pos] = g;
    }
    __syncthreads();
    // tile table, by position: groups split M (m-tiles over the group's rows) or K (m-tiles over M)
    for (int i = tid; i < G; i += kThreads) {
        const int g = s.order[i];
        const int rows = p.offsets[g + 1] - p.offsets[g];
        const int mt = p.kgroup ? (p.M + BM - 1) / BM : (rows + BM - 1) / BM;
        s.mtiles[i] = mt > 0 ? mt : 1;
        s.tile_start[i + 1] = mt * ((p.N + BN - 1) / BN);
    }
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            int v = g < G ? s.tile_start[g + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += n;
            }
            if (g < G) s.tile_start[g + 1] = carry + v;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int total = s.tile_start[G];
    const uint32_t tmem_base = s.tmem_base;

    if (warp == 0) {
        // ================= TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int last_phase[STAGES];                       // phase of each stage's last load, -1: none
#pragma unroll
            for (int i = 0; i < STAGES; ++i) last_phase[i] = -1;
            for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
                int g, mt, nt;
                decode(s, G, tile, g, mt, nt);
                const int r0 = p.offsets[g];
                const int K = p.kgroup ? p.offsets[g + 1] - r0 : p.K;
                const int nk = (K + BK - 1) / BK;
                const int e = p.b_per_group ? g : 0;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) { fail(s, p, 31); break; }
                    const uint32_t fb = smem_u32(&s.full[stage]);
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const uint32_t a_dst = smA + stage * A_BYTES, b_dst = smB + stage * B_BYTES;
                    // ---- A: rows (K-major) or a K block of the group's rows (MN-major)
                    if (A_MN) {
                        const int krow = (p.kgroup ? r0 : 0) + kb * BK;
                        tma_load_2d(a_dst, &tmA, fb, mt * BM, krow);
                        tma_load_2d(a_dst + CHUNK_BYTES, &tmA, fb, mt * BM + 64, krow);
                    } else {
                        tma_load_2d(a_dst, &tmA, fb, kb * BK, r0 + mt * BM);
                    }
                    // ---- B
                    if (B_MN) {
                        int krow = kb * BK;
                        const CUtensorMap *mb = &tmB;
                        if (p.kgroup) {
                            krow += r0;
                        } else if (p.k_split > 0 && krow >= p.k_split) {
                            mb = &tmB2;
                            krow -= p.k_split;
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (p.kgroup) tma_load_2d(b_dst + c * CHUNK_BYTES, mb, fb, nt * BN + c * 64, krow);
                            else tma_load_3d(b_dst + c * CHUNK_BYTES, mb, fb, nt * BN + c * 64, krow, e);
                        }
                    } else {
                        tma_load_3d(b_dst, &tmB, fb, kb * BK, nt * BN, e);
                    }
#pragma unroll
                    for (int i = 0; i < STAGES; ++i)
                        if (i == stage) last_phase[i] = (int)phase;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // no load may still be writing this CTA's shared memory when it exits
#pragma unroll
            for (int i = 0; i < STAGES; ++i)
                if (last_phase[i] >= 0 && !mbar_wait(smem_u32(&s.full[i]), (uint32_t)last_phase[i], p.timeout_ns))
                    fail(s, p, 36);
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
                int g, mt, nt;
                decode(s, G, tile, g, mt, nt);
                const int K = p.kgroup ? p.offsets[g + 1] - p.offsets[g] : p.K;
                const int nk = (K + BK - 1) / BK;
                if (!mbar_wait(smem_u32(&s.acce[ab]), aphase ^ 1u, p.timeout_ns)) { fail(s, p, 32); break; }
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(ab * BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    const uint32_t bar = p.kgroup ? smem_u32(&s.ready[stage]) : smem_u32(&s.full[stage]);
                    if (!mbar_wait(bar, phase, p.timeout_ns)) { fail(s, p, 33); ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smA + stage * A_BYTES, b0 = smB + stage * B_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t da = A_MN ? sdesc_mn(a0 + k * 2048) : sdesc(a0 + k * 32);
                        const uint64_t db = B_MN ? sdesc_mn(b0 + k * 2048) : sdesc(b0 + k * 32);
                        mma_bf16(dtm, da, db, kIdesc, (kb | k) ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&s.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(smem_u32(&s.accf[ab]));
                if (++ab == 2) { ab = 0; aphase ^= 1u; }
            }
            // every MMA issued here has completed before the TMEM is freed
            mma_commit(smem_u32(&s.drain));
            if (!mbar_wait(smem_u32(&s.drain), 0, p.timeout_ns)) fail(s, p, 37);
        }
    } else if (warp == 10) {
        // ================= K-tail masking (groups that split K)
        if (p.kgroup) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
                int g, mt, nt;
                decode(s, G, tile, g, mt, nt);
                const int K = p.offsets[g + 1] - p.offsets[g];
                const int nk = (K + BK - 1) / BK;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    int okw = 1;
                    if (lane == 0) okw = mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns) ? 1 : 0;
                    okw = __shfl_sync(0xffffffffu, okw, 0);
                    if (!okw) { if (lane == 0) fail(s, p, 34); ok = false; break; }
                    const int valid = K - kb * BK;
                    if (valid < BK) {
                        // rows valid..63 of every 64-row chunk: 2 chunks of A, 4 of B
                        const uint32_t a0 = smA + stage * A_BYTES, b0 = smB + stage * B_BYTES;
                        const int nrow = BK - valid;
                        for (int i = lane; i < 6 * nrow * 8; i += 32) {
                            const int chunk = i / (nrow * 8), rem = i % (nrow * 8);
                            const int row = valid + rem / 8, piece = rem % 8;
                            const uint32_t addr = (chunk < 2 ? a0 + chunk * CHUNK_BYTES : b0 + (chunk - 2) * CHUNK_BYTES) +
                                                  row * 128 + piece * 16;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&s.ready[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else {
        // ================= epilogue: warps 2..9, lane quadrant warp % 4, half of the columns
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        int ab = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
            int g, mt, nt;
            decode(s, G, tile, g, mt, nt);
            const int r0 = p.offsets[g];
            const int rows = p.offsets[g + 1] - r0;
            const int K = p.kgroup ? rows : p.K;
            const int m = mt * BM + q * 32 + lane;                   // row of this thread in the output
            const bool valid = p.kgroup ? (m < p.M) : (m < rows);
            const int64_t orow = p.kgroup ? (int64_t)m : (int64_t)r0 + m;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(smem_u32(&s.accf[ab]), aphase, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) fail(s, p, 35); break; }
            __syncwarp();
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)(ab * BN) + ((uint32_t)(q * 32) << 16);
            float dgp = 0.f;                                         // DGRAD2: this row's partial <H, dH>
            for (int cc = 0; cc < 4; ++cc) {
                const int c0 = half * 128 + cc * 32;                 // column within the tile
                const int col0 = nt * BN + c0;
                float v[32];
                if (K > 0) {
                    tmem_ld32(taddr + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                }
                if (!valid || col0 >= p.N) continue;
                const int ncol = min(32, p.N - col0);
                if (p.mode == BW_STORE_F32) {
                    float *o = static_cast<float *>(p.out) + (p.kgroup ? (int64_t)g * p.out_group_stride : 0) +
                               orow * p.ldo + col0;
                    if (ncol == 32) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<float4 *>(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    } else {
                        for (int i = 0; i < ncol; ++i) o[i] = v[i];
                    }
                } else if (p.mode == BW_STORE_BF16) {
                    const float *bias = p.bias ? p.bias + (int64_t)g * p.bias_group_stride : nullptr;
                    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + orow * p.ldo + col0;
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        if (i < ncol) {
                            const float b0 = bias ? bias[col0 + i] : 0.f;
                            const float b1 = (bias && i + 1 < ncol) ? bias[col0 + i + 1] : 0.f;
                            if (i + 1 < ncol)
                                *reinterpret_cast<__nv_bfloat162 *>(o + i) = __floats2bfloat162_rn(v[i] + b0, v[i + 1] + b1);
                            else
                                o[i] = __float2bfloat16_rn(v[i] + b0);
                        }
                    }
                } else {   // BW_DGRAD2: v = dH (gate applied) for hidden columns col0..col0+31
                    const __nv_bfloat16 *hr = p.H + orow * p.ldh + col0;
                    const __nv_bfloat16 *gr = p.GU + orow * p.ldgu + col0;
                    __nv_bfloat16 *dr = p.dGU + orow * p.ldgu + col0;
                    const bool swiglu = p.act == MOE_ACT_SWIGLU;
                    if (ncol == 32) {            // whole chunk: 16-byte loads and stores
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint4 h4 = *reinterpret_cast<const uint4 *>(hr + u * 8);
                            const uint4 g4 = *reinterpret_cast<const uint4 *>(gr + u * 8);
                            const uint4 u4 = swiglu ? *reinterpret_cast<const uint4 *>(gr + p.F + u * 8)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&h4);
                            const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&g4);
                            const __nv_bfloat162 *uu2 = reinterpret_cast<const __nv_bfloat162 *>(&u4);
                            uint4 dg4, du4;
                            __nv_bfloat162 *dg2 = reinterpret_cast<__nv_bfloat162 *>(&dg4);
                            __nv_bfloat162 *du2 = reinterpret_cast<__nv_bfloat162 *>(&du4);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float2 hf = __bfloat1622float2(h2[j]);
                                const float2 gf = __bfloat1622float2(g2[j]);
                                const float va = v[u * 8 + 2 * j], vb = v[u * 8 + 2 * j + 1];
                                dgp += hf.x * va + hf.y * vb;
                                if (swiglu) {
                                    const float2 uf = __bfloat1622float2(uu2[j]);
                                    const float sa = 1.f / (1.f + __expf(-gf.x)), sb = 1.f / (1.f + __expf(-gf.y));
                                    dg2[j] = __floats2bfloat162_rn(va * uf.x * sa * (1.f + gf.x * (1.f - sa)),
                                                                   vb * uf.y * sb * (1.f + gf.y * (1.f - sb)));
                                    du2[j] = __floats2bfloat162_rn(va * gf.x * sa, vb * gf.y * sb);
                                } else {
                                    const float pa = 0.5f * (1.f + erff(gf.x * 0.70710678118654752f)) +
                                                     gf.x * 0.39894228040143268f * __expf(-0.5f * gf.x * gf.x);
                                    const float pb = 0.5f * (1.f + erff(gf.y * 0.70710678118654752f)) +
                                                     gf.y * 0.39894228040143268f * __expf(-0.5f * gf.y * gf.y);
                                    dg2[j] = __floats2bfloat162_rn(va * pa, vb * pb);
                                }
                            }
                            *reinterpret_cast<uint4 *>(dr + u * 8) = dg4;
                            if (swiglu) *reinterpret_cast<uint4 *>(dr + p.F + u * 8) = du4;
                        }
                    } else {
                        for (int i = 0; i < ncol; ++i) {
                            const float hv = __bfloat162float(hr[i]), gv = __bfloat162float(gr[i]);
                            dgp += hv * v[i];
                            if (swiglu) {
                                const float uv = __bfloat162float(gr[p.F + i]);
                                const float sg = 1.f / (1.f + __expf(-gv));
                                dr[i] = __float2bfloat16_rn(v[i] * uv * sg * (1.f + gv * (1.f - sg)));
                                dr[p.F + i] = __float2bfloat16_rn(v[i] * gv * sg);
                            } else {
                                const float gp = 0.5f * (1.f + erff(gv * 0.70710678118654752f)) +
                                                 gv * 0.39894228040143268f * __expf(-0.5f * gv * gv);
                                dr[i] = __float2bfloat16_rn(v[i] * gp);
                            }
                        }
                    }
                }
            }
            if (p.mode == BW_DGRAD2 && valid) p.part[orow * p.part_ld + nt * 2 + half] = dgp;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&s.acce[ab]));
            if (++ab == 2) { ab = 0; aphase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <bool A_MN, bool B_MN>
cudaError_t launch_variant(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &B2,
                           const BwdGemmParams &p, int grid, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc_bwd_gemm<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_kernel(tc_bwd_gemm<A_MN, B_MN>, dim3(grid), dim3(kThreads), kSmemBytes, st, true, A, B, B2, p);
}

}  // namespace

cudaError_t launch_bwd_gemm(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &B2, bool a_mn, bool b_mn,
                            const BwdGemmParams &p, int num_sms, cudaStream_t st) {
    if (p.G < 1 || p.G > kMaxGroups - 1) return cudaErrorInvalidValue;
    const int grid = num_sms > 0 ? num_sms : 148;
    if (!a_mn && !b_mn) return launch_variant<false, false>(A, B, B2, p, grid, st);
    if (!a_mn && b_mn) return launch_variant<false, true>(A, B, B2, p, grid, st);
    if (a_mn && b_mn) return launch_variant<true, true>(A, B, B2, p, grid, st);
    return cudaErrorInvalidValue;
}

}  // namespace moe
