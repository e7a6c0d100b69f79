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
// One persistent kernel serves every form, on CTA pairs (clusters of two CTAs
// sharing one tcgen05.mma.cta_group::2 of M = 256, N = 256: each CTA holds
// 128 rows of A and half of B's columns, and gets its 128 rows of the
// accumulator in its own TMEM), 352 threads per CTA:
//   warp 0      TMA producer (both CTAs): this CTA's A 128 x 64 and B 128 x 64
//               per stage, six stages of 32 KiB, completion on this CTA's own
//               barriers.  K-major operands come as one box per operand (64
//               elements of K per 128-byte swizzled row); MN-major operands as
//               two 64-element-wide boxes of 64 K rows (128-byte rows of MN,
//               8-row swizzle atoms)
//   warp 10     (both CTAs) once a stage has landed: for groups that split K,
//               zeroes the rows of a group's last K block that lie past the
//               group's rows, in both operands (the rows beyond belong to
//               another expert); then reports the stage ready to the first
//               CTA of the pair
//   warp 1      (first CTA) single-thread MMA issuer once both CTAs' stage is
//               ready, two 256-column fp32 TMEM accumulators; its commits
//               free the stage and hand the accumulator to both CTAs
//   warps 2-9   epilogue (both CTAs): TMEM -> registers, then the form's store
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

constexpr int BM = 128, PM = 256, BN = 256, BNH = 128, BK = 64, STAGES = 6;   // PM: rows per pair, BNH: B rows per CTA
constexpr int kThreads = 352;
constexpr uint32_t A_BYTES = BM * BK * 2;          // 16 KiB: this CTA's 128 A rows
constexpr uint32_t B_BYTES = BNH * BK * 2;         // 16 KiB: this CTA's half of B
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
    uint64_t ready[STAGES];      // first CTA's: both CTAs' stage landed (and masked)
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
constexpr uint32_t STG_BYTES = 32 * 64;            // per epilogue warp: 32 rows x 64 bytes
constexpr size_t kStgOff = (STAGES * STAGE_BYTES + sizeof(SmemB) + 1023) / 1024 * 1024;
constexpr size_t kSmemBytes = 1024 + kStgOff + 8 * STG_BYTES;
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

// The epilogue holds one accumulator row per thread; global memory wants each
// row's bytes from consecutive lanes.  A warp's 32 rows x 64 bytes pass
// through its staging buffer: each lane writes its row as four 16-byte pieces
// (piece c of row r at slot c ^ ((r / 2) % 4), so neither the writes nor the
// reads below hit a bank twice), then the block is read back by pieces.
__device__ __forceinline__ void stage_row64(uint32_t stg, const uint32_t *w) {
    const int lane = threadIdx.x & 31;
    __syncwarp();                                   // the previous block has been read
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t a = stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(w[4 * c]), "r"(w[4 * c + 1]),
                     "r"(w[4 * c + 2]), "r"(w[4 * c + 3]) : "memory");
    }
    __syncwarp();
}
__device__ __forceinline__ uint4 staged_piece(uint32_t stg, int r, int c) {
    uint4 v;
    const uint32_t a = stg + r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
// Store a staged 32 x 64-byte block: rows 0..nrows-1 to dst + r * ld_bytes,
// eight whole 64-byte row segments per warp instruction.
__device__ __forceinline__ void store_staged(uint32_t stg, char *dst, int64_t ld_bytes, int nrows) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = i * 32 + lane, r = j >> 2, c = j & 3;
        if (r < nrows) *reinterpret_cast<uint4 *>(dst + r * ld_bytes + c * 16) = staged_piece(stg, r, c);
    }
}

__device__ __forceinline__ float silu_grad_parts(float g, float &sg) {
    sg = 1.f / (1.f + __expf(-g));
    return sg * (1.f + g * (1.f - sg));
}
__device__ __forceinline__ float gelu_grad(float g) {
    return 0.5f * (1.f + erff(g * 0.70710678118654752f)) + g * 0.39894228040143268f * __expf(-0.5f * g * g);
}

template <bool A_MN, bool B_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
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
    const uint32_t rank = cluster_ctarank();
    const int pair = (int)cluster_id_x(), npairs = (int)ncluster_x();
    const int G = p.G;
    constexpr uint32_t kIdesc = make_idesc_bf16(PM, BN) | (A_MN ? (1u << 15) : 0u) | (B_MN ? (1u << 16) : 0u);

    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.ready[i]), 2);
            mbar_init(smem_u32(&s.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&s.accf[i]), 1); mbar_init(smem_u32(&s.acce[i]), 16); }
        mbar_init(smem_u32(&s.drain), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(&s.tmem_base), TMEM_COLS);   // warp 1 of both CTAs
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
        const int mt = p.kgroup ? (p.M + PM - 1) / PM : (rows + PM - 1) / PM;
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
    cluster_sync();                                  // barriers of both CTAs initialised
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
            for (int tile = pair; tile < total && !aborted(s); tile += npairs) {
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
                    const int m0 = mt * PM + (int)rank * BM;          // this CTA's first row of the tile
                    if (A_MN) {
                        const int krow = (p.kgroup ? r0 : 0) + kb * BK;
                        tma_load_2d(a_dst, &tmA, fb, m0, krow);
                        tma_load_2d(a_dst + CHUNK_BYTES, &tmA, fb, m0 + 64, krow);
                    } else {
                        tma_load_2d(a_dst, &tmA, fb, kb * BK, r0 + m0);
                    }
                    const int n0 = nt * BN + (int)rank * BNH;         // this CTA's first B row (column of C)
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
                        for (int c = 0; c < 2; ++c) {
                            if (p.kgroup) tma_load_2d(b_dst + c * CHUNK_BYTES, mb, fb, n0 + c * 64, krow);
                            else tma_load_3d(b_dst + c * CHUNK_BYTES, mb, fb, n0 + c * 64, krow, e);
                        }
                    } else {
                        tma_load_3d(b_dst, &tmB, fb, kb * BK, n0, e);
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
        // ================= MMA issuer (first CTA of the pair)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            for (int tile = pair; tile < total && !aborted(s); tile += npairs) {
                int g, mt, nt;
                decode(s, G, tile, g, mt, nt);
                const int K = p.kgroup ? p.offsets[g + 1] - p.offsets[g] : p.K;
                const int nk = (K + BK - 1) / BK;
                if (!mbar_wait(smem_u32(&s.acce[ab]), aphase ^ 1u, p.timeout_ns)) { fail(s, p, 32); break; }
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(ab * BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.ready[stage]), phase, p.timeout_ns)) { fail(s, p, 33); ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smA + stage * A_BYTES, b0 = smB + stage * B_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t da = A_MN ? sdesc_mn(a0 + k * 2048) : sdesc(a0 + k * 32);
                        const uint64_t db = B_MN ? sdesc_mn(b0 + k * 2048) : sdesc(b0 + k * 32);
                        mma_bf16_pair(dtm, da, db, kIdesc, (kb | k) ? 1u : 0u);
                    }
                    mma_commit_pair(smem_u32(&s.empty[stage]), (uint16_t)0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&s.accf[ab]), (uint16_t)0x3);
                if (++ab == 2) { ab = 0; aphase ^= 1u; }
            }
            // every MMA issued here has completed before the TMEM is freed
            mma_commit_pair(smem_u32(&s.drain), (uint16_t)0x1);
            if (!mbar_wait(smem_u32(&s.drain), 0, p.timeout_ns)) fail(s, p, 37);
        }
    } else if (warp == 10) {
        // ================= stage landed (and, for groups that split K, masked): tell the MMA issuer
        {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = pair; tile < total && !aborted(s); tile += npairs) {
                int g, mt, nt;
                decode(s, G, tile, g, mt, nt);
                const int K = p.kgroup ? p.offsets[g + 1] - p.offsets[g] : p.K;
                const int nk = (K + BK - 1) / BK;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    int okw = 1;
                    if (lane == 0) okw = mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns) ? 1 : 0;
                    okw = __shfl_sync(0xffffffffu, okw, 0);
                    if (!okw) { if (lane == 0) fail(s, p, 34); ok = false; break; }
                    const int valid = K - kb * BK;
                    if (p.kgroup && valid < BK) {
                        // rows valid..63 of every 64-row chunk: 2 chunks of A, 2 of B
                        const uint32_t a0 = smA + stage * A_BYTES, b0 = smB + stage * B_BYTES;
                        const int nrow = BK - valid;
                        for (int i = lane; i < 4 * nrow * 8; i += 32) {
                            const int chunk = i / (nrow * 8), rem = i % (nrow * 8);
                            const int row = valid + rem / 8, piece = rem % 8;
                            const uint32_t addr = (chunk < 2 ? a0 + chunk * CHUNK_BYTES : b0 + (chunk - 2) * CHUNK_BYTES) +
                                                  row * 128 + piece * 16;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.ready[stage]), 0));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else {
        // ================= epilogue: warps 2..9, lane quadrant warp % 4, half of the columns
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const uint32_t stg = base + (uint32_t)kStgOff + (uint32_t)(warp - 2) * STG_BYTES;
        // fp32 outputs leave in 16-byte pieces when the rows allow it (dW_r's rows of E values may not)
        const bool vec_f32 = ((reinterpret_cast<uintptr_t>(p.out) | (uintptr_t)(p.ldo * 4) |
                               (uintptr_t)(p.out_group_stride * 4)) & 15u) == 0;
        int ab = 0;
        uint32_t aphase = 0;
        for (int tile = pair; tile < total && !aborted(s); tile += npairs) {
            int g, mt, nt;
            decode(s, G, tile, g, mt, nt);
            const int r0 = p.offsets[g];
            const int rows = p.offsets[g + 1] - r0;
            const int K = p.kgroup ? rows : p.K;
            const int m = mt * PM + (int)rank * BM + q * 32 + lane;  // row of this thread in the output
            const bool valid = p.kgroup ? (m < p.M) : (m < rows);
            const int64_t orow = p.kgroup ? (int64_t)m : (int64_t)r0 + m;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(smem_u32(&s.accf[ab]), aphase, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) fail(s, p, 35); break; }
            __syncwarp();
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)(ab * BN) + ((uint32_t)(q * 32) << 16);
            // valid rows are a prefix of the warp's 32 rows; the warp's first row is orow - lane
            const int nrows = __popc(__ballot_sync(0xffffffffu, valid));
            const int64_t orow0 = orow - lane;
            float dgp[2] = {0.f, 0.f};                               // DGRAD2: rows lane/2 and 16 + lane/2
            for (int cc = 0; cc < 4; ++cc) {
                const int c0 = half * 128 + cc * 32;                 // column within the tile
                const int col0 = nt * BN + c0;
                float v[32];
                __syncwarp();                                        // the TMEM load is warp-collective
                if (K > 0) {
                    tmem_ld32(taddr + c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                }
                if (nrows == 0 || col0 >= p.N) continue;            // uniform over the warp
                const int ncol = min(32, p.N - col0);
                if (p.mode == BW_STORE_F32) {
                    float *o = static_cast<float *>(p.out) + (p.kgroup ? (int64_t)g * p.out_group_stride : 0);
                    if (ncol == 32 && vec_f32) {
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            stage_row64(stg, reinterpret_cast<const uint32_t *>(v + hh * 16));
                            store_staged(stg, reinterpret_cast<char *>(o + orow0 * p.ldo + col0 + hh * 16),
                                         p.ldo * 4, nrows);
                        }
                    } else if (valid) {
                        float *orp = o + orow * p.ldo + col0;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < ncol) orp[i] = v[i];
                    }
                } else if (p.mode == BW_STORE_BF16) {    // N and ldo multiples of 32 and 8 (host-checked)
                    const float *bias = p.bias ? p.bias + (int64_t)g * p.bias_group_stride + col0 : nullptr;
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float b0 = bias ? __ldg(bias + 2 * i) : 0.f, b1 = bias ? __ldg(bias + 2 * i + 1) : 0.f;
                        const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * i] + b0, v[2 * i + 1] + b1);
                        w[i] = *reinterpret_cast<const uint32_t *>(&t);
                    }
                    stage_row64(stg, w);
                    store_staged(stg, reinterpret_cast<char *>(static_cast<__nv_bfloat16 *>(p.out) + orow0 * p.ldo + col0),
                                 p.ldo * 2, nrows);
                } else {   // BW_DGRAD2: v = dH (gate applied) for hidden columns col0..col0+31 (F a multiple of 32)
                    const bool swiglu = p.act == MOE_ACT_SWIGLU;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {                 // 16 columns at a time
                        stage_row64(stg, reinterpret_cast<const uint32_t *>(v + hh * 16));
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int j = i * 32 + lane, r = j >> 1, c = j & 1;   // row r, columns c*8 .. c*8+7
                            if (r >= nrows) continue;
                            const uint4 d0 = staged_piece(stg, r, 2 * c), d1 = staged_piece(stg, r, 2 * c + 1);
                            float dh[8];
                            dh[0] = __uint_as_float(d0.x); dh[1] = __uint_as_float(d0.y);
                            dh[2] = __uint_as_float(d0.z); dh[3] = __uint_as_float(d0.w);
                            dh[4] = __uint_as_float(d1.x); dh[5] = __uint_as_float(d1.y);
                            dh[6] = __uint_as_float(d1.z); dh[7] = __uint_as_float(d1.w);
                            const int64_t row = orow0 + r;
                            const int col = col0 + hh * 16 + c * 8;
                            const uint4 h4 = *reinterpret_cast<const uint4 *>(p.H + row * p.ldh + col);
                            const uint4 g4 = *reinterpret_cast<const uint4 *>(p.GU + row * p.ldgu + col);
                            const uint4 u4 = swiglu ? *reinterpret_cast<const uint4 *>(p.GU + row * p.ldgu + p.F + col)
                                                    : make_uint4(0u, 0u, 0u, 0u);
                            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&h4);
                            const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&g4);
                            const __nv_bfloat162 *uu2 = reinterpret_cast<const __nv_bfloat162 *>(&u4);
                            uint4 dg4, du4;
                            __nv_bfloat162 *dg2 = reinterpret_cast<__nv_bfloat162 *>(&dg4);
                            __nv_bfloat162 *du2 = reinterpret_cast<__nv_bfloat162 *>(&du4);
                            float acc = 0.f;
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const float2 hf = __bfloat1622float2(h2[t]);
                                const float2 gf = __bfloat1622float2(g2[t]);
                                const float va = dh[2 * t], vb = dh[2 * t + 1];
                                acc += hf.x * va + hf.y * vb;
                                if (swiglu) {
                                    const float2 uf = __bfloat1622float2(uu2[t]);
                                    float sa, sb;
                                    const float pa = silu_grad_parts(gf.x, sa), pb = silu_grad_parts(gf.y, sb);
                                    dg2[t] = __floats2bfloat162_rn(va * uf.x * pa, vb * uf.y * pb);
                                    du2[t] = __floats2bfloat162_rn(va * gf.x * sa, vb * gf.y * sb);
                                } else {
                                    dg2[t] = __floats2bfloat162_rn(va * gelu_grad(gf.x), vb * gelu_grad(gf.y));
                                }
                            }
                            dgp[i] += acc;
                            *reinterpret_cast<uint4 *>(p.dGU + row * p.ldgu + col) = dg4;
                            if (swiglu) *reinterpret_cast<uint4 *>(p.dGU + row * p.ldgu + p.F + col) = du4;
                        }
                    }
                }
            }
            if (p.mode == BW_DGRAD2) {
                // lanes 2m and 2m+1 hold halves of rows m and 16 + m; row `lane`'s sum goes to this lane
#pragma unroll
                for (int i = 0; i < 2; ++i) dgp[i] += __shfl_xor_sync(0xffffffffu, dgp[i], 1);
                const float a0 = __shfl_sync(0xffffffffu, dgp[0], (lane & 15) * 2);
                const float a1 = __shfl_sync(0xffffffffu, dgp[1], (lane & 15) * 2);
                if (valid) p.part[orow * p.part_ld + nt * 2 + half] = lane < 16 ? a0 : a1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.acce[ab]), 0));
            if (++ab == 2) { ab = 0; aphase ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();                                  // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <bool A_MN, bool B_MN>
cudaError_t launch_variant(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &B2,
                           const BwdGemmParams &p, int num_sms, cudaStream_t st) {
    static int grid = 0;                           // clusters of two that fit at once, times two
    if (grid == 0) {
        cudaError_t e = cudaFuncSetAttribute(tc_bwd_gemm<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, tc_bwd_gemm<A_MN, B_MN>, &cfg);
        if (e != cudaSuccess || nclusters < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        grid = 2 * nclusters;
    }
    return launch_kernel(tc_bwd_gemm<A_MN, B_MN>, dim3(grid), dim3(kThreads), kSmemBytes, st, true, A, B, B2, p);
}

}  // namespace

cudaError_t launch_bwd_gemm(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &B2, bool a_mn, bool b_mn,
                            const BwdGemmParams &p, int num_sms, cudaStream_t st) {
    if (p.G < 1 || p.G > kMaxGroups - 1) return cudaErrorInvalidValue;
    // bf16 outputs and the fused activation backward move whole 32-column chunks in 16-byte pieces
    if (p.mode == BW_STORE_BF16 && (p.N % 32 != 0 || p.ldo % 8 != 0)) return cudaErrorInvalidValue;
    if (p.mode == BW_DGRAD2 && (p.N % 32 != 0 || p.F % 32 != 0 || p.ldh % 8 != 0 || p.ldgu % 8 != 0))
        return cudaErrorInvalidValue;
    const int nsm = num_sms > 0 ? num_sms : 148;
    if (!a_mn && !b_mn) return launch_variant<false, false>(A, B, B2, p, nsm, st);
    if (!a_mn && b_mn) return launch_variant<false, true>(A, B, B2, p, nsm, st);
    if (a_mn && b_mn) return launch_variant<true, true>(A, B, B2, p, nsm, st);
    return cudaErrorInvalidValue;
}

}  // namespace moe
