// ffn_sm100.cu -- grouped expert FFN for bf16 layers on the 5th-generation
// tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Expert definitions: GELU expert Linear-GELU-Linear with biases ("Fine-tuning
// and serving MoE models", How an MoE layer actually works); SwiGLU expert
// W_down(SiLU(W_gate x) * (W_up x)) ("Fine-Tuning Mixture of Experts (MoE)
// Models: Router Optimization Techniques", What Is It?).  Running all experts
// in one grouped launch instead of one launch per expert is what the pages
// recommend (Router Optimization page, What Most Articles Miss 2; serving
// tutorial, grouped GEMM remark).
//
// Two persistent kernels per GEMM, launched back to back on the stream:
//   tc_grouped_gemm_pair  one cluster of two CTAs per pair of SMs
//               (tcgen05.mma.cta_group::2, M = 256, N = 256): every group's
//               256-row blocks and a last block of more than 128 rows
//   tc_grouped_gemm       one CTA per SM (M = 128, N = 256): a last block of
//               1..128 rows, which mostly streams the weights of small experts
// Roles (both kernels, 320 threads, warp-specialised):
//   warp 0      TMA producer: A (activations) and B (weights) tiles, 64 deep
//               in K, 128-byte swizzle, mbarrier transaction counts
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer, fp32
//               accumulators in TMEM, two 256-column accumulators so the
//               epilogue of tile i overlaps the mainloop of tile i+1
//   warps 2..9  epilogue (two warps per TMEM lane quadrant, each taking half
//               of the columns): four tcgen05.ld of 32 columns under one
//               wait, fused activation (SwiGLU: gate and up halves of one
//               N=256 accumulator; GELU: bias + exact-erf GELU) or fused bias
//               + gate scale; a warp whose 32 rows are all valid stores
//               through a 2 KiB swizzled staging buffer and TMA tensor
//               stores, others store directly
// Tiles: groups are the routed experts (rows offsets[e]..offsets[e+1] of the
// packed activations) plus an optional shared expert over all T tokens.  The
// tile list is built on the device from `offsets` (no host round trip); a
// tile may start mid-way through the packed buffer, rows past the group's end
// are computed but never stored.  Within a group the m index runs fastest so
// CTAs working at the same time share one weight tile through L2.
//
// e4m3 experts (the F8 instantiations): the same kernels with e4m3 A and B
// tiles (128 elements per 128-byte swizzled row, kind::f8f6f4 MMAs of 32
// elements of K); the epilogue multiplies each fp32 accumulator by its row's
// activation scale and its column's weight scale before the activation or
// gate (the scales are loaded before the accumulator wait; a column's scale
// reaches the warp's rows by shuffle in the SwiGLU GEMM, and through a
// per-warp shared-memory slot read as float4 broadcasts in the others, whose
// down projection also folds the row's gate into its row scale).
//
// Training forward (the SAVE instantiations of the first GEMM): the epilogue
// also stores the pre-activations -- G and U before the SwiGLU, W_1 x + b_1
// before the GELU -- in bf16 through the same staging buffer, for the
// backward pass to read instead of recomputing them.
//
// INT4 weight-only experts (tc_w4_gemm_pair, further below): the pair kernel
// with its B operand decoded on the chip by four extra warps per CTA.
//
// Every mbarrier wait is bounded (a global-timer limit); a wait that runs out
// records MOE_ERR_TIMEOUT in the workspace status word and the CTA unwinds,
// freeing its TMEM.  No TMA multicast is used.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int BM = 128;                 // rows per tile (MMA M)
constexpr int BK = 64;                  // K per stage: one 128-byte swizzle atom of bf16
constexpr int BNB = 256;                // B rows per stage (MMA N)
constexpr int STAGES = 4;
constexpr int kThreads = 320;                // 10 warps: producer, MMA, 8 epilogue
constexpr uint32_t A_BYTES = BM * BK * 2;       // 16 KiB
constexpr uint32_t B_BYTES = BNB * BK * 2;      // 32 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;             // 2 accumulators x 256 fp32 columns
constexpr int kMaxGroups = 257;

enum { GM_SWIGLU = 0, GM_GELU = 1, GM_DOWN = 2 };

constexpr uint32_t kIdesc = make_idesc_bf16(BM, BNB);   // M=128, N=256
constexpr uint32_t kIdescF8 = make_idesc_e4m3(BM, BNB);
// K elements per stage: one 128-byte swizzle row of bf16 or of e4m3
template <bool F8> constexpr int bk_elems() { return F8 ? 128 : 64; }

struct GemmParams {
    const int32_t *offsets;   // [E+1]: routed group g holds rows offsets[g] .. offsets[g+1]
    const float *bias;        // [E, N_routed] or null (GELU b1 / b2)
    const float *row_gate;    // [rows] (GM_DOWN) or null
    __nv_bfloat16 *out;       // row stride ldo
    int32_t *status;
    int E, T;                 // E: routed groups (the shared group, if any, is group E)
    int E_w;                  // experts in the weight tensors: routed group g uses expert g % E_w
    int K_routed, K_shared;
    int N_routed, N_shared;
    int has_shared;
    int ldo;
    int64_t shared_a_row;     // first A row of the shared group
    int64_t shared_out_row;   // first output row of the shared group
    // training forward (SAVE instantiations of the first GEMM): the
    // pre-activations as bf16 -- SwiGLU: G in columns 0..N-1 and U in N..2N-1
    // of each row, GELU: W_1 x + b_1 -- routed row r at pre + r * pre_ld,
    // shared row t at pre_s + t * pre_ld_s
    __nv_bfloat16 *pre, *pre_s;
    int64_t pre_ld, pre_ld_s;
    int tail_mode;            // 1-CTA kernel: 0 all rows; 1 only a group's last rows
                              // when rows % 256 is in 1..128 (the rest runs in pair tiles)
    uint64_t timeout_ns;
    // e4m3 operands: the accumulator is scaled by its A row's scale and its
    // output column's scale before the epilogue's arithmetic
    const float *row_scale;         // routed groups: scale of packed A row r
    const float *shared_row_scale;  // shared group: scale of A row shared_a_row + i
    const float *col_scale;         // [E, N_routed] (SwiGLU: the gate projection)
    const float *col_scale2;        // [E, N_routed] SwiGLU up projection
    const float *sh_col_scale;      // [N_shared]
    const float *sh_col_scale2;     // [N_shared]
};

// Weight expert of routed group g (groups are the experts themselves, or, for
// rows gathered from several sources, consecutive runs of all E_w experts).
__device__ __forceinline__ int group_expert(const GemmParams &p, int g) {
    return p.E == p.E_w ? g : g % p.E_w;
}

struct SmemTail {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t accf[2];
    uint64_t acce[2];
    uint32_t tmem_base;
    int abort_flag;
    int tile_start[kMaxGroups + 1];
    int mtiles[kMaxGroups];
    int rows[kMaxGroups];     // rows this launch computes for the group
    int row0[kMaxGroups];     // routed groups: first packed row (offsets[g] + start)
    int start[kMaxGroups];    // first row of the group this launch computes
};

// Epilogue staging: one 2 KiB buffer per epilogue warp (32 rows x 32 bf16),
// 1024-byte aligned after the tail, then a 512-byte column-scale slot per
// epilogue warp (e4m3 tiles).
constexpr uint32_t STG_BYTES = 32 * 32 * 2;
constexpr size_t kStgOff = (STAGES * STAGE_BYTES + sizeof(SmemTail) + 1023) / 1024 * 1024;
constexpr uint32_t SCL_BYTES = 512;        // e4m3: a warp's 128 column scales
constexpr size_t kSmemBytes = 1024 /*align slack*/ + kStgOff + 8 * STG_BYTES + 8 * SCL_BYTES;
static_assert(kSmemBytes <= 227 * 1024, "1-CTA kernel shared memory");

__device__ __forceinline__ float gelu_erf(float v) { return 0.5f * v * (1.f + erff(v * 0.70710678118654752f)); }
// SiLU with the fast reciprocal division: its few-ulp fp32 error sits far
// below the bf16 rounding of H; a large negative v gives exp overflow, a
// quotient of 0 and silu = -0.
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }

__device__ __forceinline__ void store8(__nv_bfloat16 *dst, const float *v) {
    uint4 pk;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&pk);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4 *>(dst) = pk;
}

// Store one 32-column chunk of the warp's 32 rows (h: this lane's row) with a
// TMA tensor store: the chunk goes to the warp's 2 KiB staging buffer in the
// 64-byte swizzled layout (16-byte piece c of row r at piece c ^ ((r / 2) % 4),
// conflict-free), then one store writes the 32 x 32 block in whole 64-byte row
// segments.  The previous store from the buffer must have read it first.
__device__ __forceinline__ void stage_store32(uint32_t stg, const CUtensorMap *tmO, int col0, int row0, const float *h) {
    const int lane = threadIdx.x & 31;
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(h[2 * i], h[2 * i + 1]);
        pk[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
    if (lane == 0) tma_store_wait_read();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t a = stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * c]), "r"(pk[4 * c + 1]),
                     "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3]) : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmO, stg, col0, row0);
        tma_store_commit();
    }
}

// The scale of column col0 + lane (0 past N): one coalesced load per warp
// and 32-column chunk; the epilogue hands each column's scale to every row
// (lane) with a shuffle (SwiGLU) or through the warp's shared-memory slot.
__device__ __forceinline__ float col_scale_lane(const float *cs, int col0, int N) {
    const int c = col0 + (int)(threadIdx.x & 31);
    return c < N ? __ldg(cs + c) : 0.f;
}

// e4m3 tiles: this thread's row scale and the column scales its warp's
// chunks need (SwiGLU: gate scales of chunks half*2, half*2+1, then the up
// scales; otherwise chunks half*4 .. half*4+3), loaded before the accumulator
// wait so their latency overlaps it.
template <int MODE>
__device__ __forceinline__ void preload_scales(const GemmParams &p, bool sh, int g, int nt, int half, int N,
                                               bool valid, int64_t arow, float &rscale, float *csv) {
    rscale = valid ? __ldg((sh ? p.shared_row_scale : p.row_scale) + arow) : 0.f;
    const float *cs = sh ? p.sh_col_scale : p.col_scale + (size_t)group_expert(p, g) * p.N_routed;
    if (MODE == GM_SWIGLU) {
        const float *cs2 = sh ? p.sh_col_scale2 : p.col_scale2 + (size_t)group_expert(p, g) * p.N_routed;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int col0 = nt * 128 + (half * 2 + cc) * 32;
            csv[cc] = col_scale_lane(cs, col0, N);
            csv[2 + cc] = col_scale_lane(cs2, col0, N);
        }
    } else {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) csv[cc] = col_scale_lane(cs, nt * BNB + (half * 4 + cc) * 32, N);
    }
}

// Epilogue of one accumulator row (this thread's TMEM lane) for one tile:
// the warp's half of the columns (SwiGLU: gate chunks half*2, half*2+1 and
// the up chunks 128 columns on; otherwise chunks half*4 .. half*4+3) arrive
// with one TMEM wait, then the fused activation or bias + gate scale.  When
// all 32 rows of the warp are valid, each 32-column chunk leaves through the
// staging buffer and a TMA store (row0: the warp's first output row);
// otherwise each valid row stores its columns below N with 16-byte stores.
template <int MODE, bool F8, bool SAVE = false>
__device__ __forceinline__ void epilogue_row(uint32_t taddr, int half, int nt, bool valid, int N,
                                             __nv_bfloat16 *orow_ptr, const float *bias, float gscale,
                                             const CUtensorMap *tmO, uint32_t stg, int row0, float rscale,
                                             const float *csv, float *scl, const CUtensorMap *tmP = nullptr,
                                             int prow0 = 0, __nv_bfloat16 *prow_ptr = nullptr) {
    float v[128];
    const bool staged = __all_sync(0xffffffffu, valid);
    if (MODE == GM_SWIGLU) {
        const int c0 = half * 2;
        tmem_ld32x4(taddr + c0 * 32, taddr + (c0 + 1) * 32, taddr + 128 + c0 * 32, taddr + 128 + (c0 + 1) * 32, v);
        if (SAVE) {                                   // G and U as computed, before the activation
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int col0 = nt * 128 + (c0 + cc) * 32;
                if (col0 >= N) continue;                  // uniform over the warp
                if (staged) {
                    stage_store32(stg, tmP, col0, prow0, v + cc * 32);
                    stage_store32(stg, tmP, N + col0, prow0, v + 64 + cc * 32);
                } else if (valid) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        store8(prow_ptr + col0 + u * 8, v + cc * 32 + u * 8);
                        store8(prow_ptr + N + col0 + u * 8, v + 64 + cc * 32 + u * 8);
                    }
                }
            }
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int col0 = nt * 128 + (c0 + cc) * 32;
            float *h = v + cc * 32;                  // in place of the gate values
            if (F8) {                                // gate and up column scales
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    h[i] *= rscale * __shfl_sync(0xffffffffu, csv[cc], i);
                    v[64 + cc * 32 + i] *= rscale * __shfl_sync(0xffffffffu, csv[2 + cc], i);
                }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) h[i] = silu(h[i]) * v[64 + cc * 32 + i];
            if (staged) {
                if (col0 < N) stage_store32(stg, tmO, col0, row0, h);
            } else if (valid) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (col0 + u * 8 < N) store8(orow_ptr + col0 + u * 8, h + u * 8);
            }
        }
    } else {
        const int c0 = half * 4;
        tmem_ld32x4(taddr + c0 * 32, taddr + (c0 + 1) * 32, taddr + (c0 + 2) * 32, taddr + (c0 + 3) * 32, v);
        if (F8) {
            const int lane = threadIdx.x & 31;
#pragma unroll
            for (int j = 0; j < 4; ++j) scl[j * 32 + lane] = csv[j];
            __syncwarp();
        }
        // no bias: the down projection's gate joins the row scale
        const float rs = (F8 && MODE == GM_DOWN && bias == nullptr) ? rscale * gscale : rscale;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int col0 = nt * BNB + (c0 + cc) * 32;
            if (col0 >= N) continue;                  // uniform over the warp
            float *h = v + cc * 32;                  // in place
            if (F8) {
                const float4 *c4 = reinterpret_cast<const float4 *>(scl + cc * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 a = c4[i];
                    h[4 * i] *= a.x * rs; h[4 * i + 1] *= a.y * rs;
                    h[4 * i + 2] *= a.z * rs; h[4 * i + 3] *= a.w * rs;
                }
            }
            if (SAVE && MODE == GM_GELU) {                // the pre-activation W_1 x + b_1, then GELU
#pragma unroll
                for (int i = 0; i < 32; ++i) h[i] += (bias && col0 + i < N) ? __ldg(bias + col0 + i) : 0.f;
                if (staged) {
                    stage_store32(stg, tmP, col0, prow0, h);
                } else if (valid) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (col0 + u * 8 < N) store8(prow_ptr + col0 + u * 8, h + u * 8);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) h[i] = gelu_erf(h[i]);
            } else if (!F8 || bias != nullptr) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float z = h[i] + ((bias && col0 + i < N) ? __ldg(bias + col0 + i) : 0.f);
                    h[i] = (MODE == GM_GELU) ? gelu_erf(z) : gscale * z;
                }
            } else if (MODE == GM_GELU) {
#pragma unroll
                for (int i = 0; i < 32; ++i) h[i] = gelu_erf(h[i]);
            }                                         // e4m3 down, no bias: the gate is in rs
            if (staged) {
                stage_store32(stg, tmO, col0, row0, h);
            } else if (valid) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (col0 + u * 8 < N) store8(orow_ptr + col0 + u * 8, h + u * 8);
            }
        }
    }
}

__device__ __forceinline__ void decode(const SmemTail &s, int G, int tile, int &g, int &mt, int &nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int local = tile - s.tile_start[g];
    mt = local % s.mtiles[g];
    nt = local / s.mtiles[g];
}

__device__ __forceinline__ bool aborted(const SmemTail &s) {
    return *reinterpret_cast<const volatile int *>(&s.abort_flag) != 0;
}
__device__ __forceinline__ void fail(SmemTail &s, const GemmParams &p, int where) {
    record_error(p.status, MOE_ERR_TIMEOUT, where);
    *reinterpret_cast<volatile int *>(&s.abort_flag) = 1;
}

template <int MODE, bool F8, bool SAVE = false>
__global__ void __launch_bounds__(kThreads, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                const __grid_constant__ CUtensorMap tmBs, const __grid_constant__ CUtensorMap tmBs2,
                const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmP,
                const __grid_constant__ CUtensorMap tmPs, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    SmemTail &s = *reinterpret_cast<SmemTail *>(smem + STAGES * STAGE_BYTES);
    const uint32_t smA = base;                          // STAGES x 16 KiB
    const uint32_t smB = base + STAGES * A_BYTES;       // STAGES x 32 KiB

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int BNO = (MODE == GM_SWIGLU) ? 128 : 256;   // output columns per tile
    const int G = p.E + (p.has_shared ? 1 : 0);

    // ---- independent of the previous kernel: barriers, TMEM, descriptors
    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) { mbar_init(smem_u32(&s.full[i]), 1); mbar_init(smem_u32(&s.empty[i]), 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&s.accf[i]), 1); mbar_init(smem_u32(&s.acce[i]), 8); }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&s.tmem_base), TMEM_COLS);   // whole warp; address lands in smem
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
    }
    // Last blocks (tail mode) touch only rows the CTA-pair launch before them
    // leaves alone and read only what the kernel before that wrote (complete
    // once the pair launch started, which is when this launch can begin), so
    // they start at once on the SMs the pair launch frees and wait for it
    // only before exiting: whatever waits for this launch then also sees the
    // pair launch's results.
    if (p.tail_mode) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    else pdl_wait_then_release();
    if (tid == 0) s.tile_start[0] = 0;
    // ---- tile table from the device-side offsets
    for (int g = tid; g < G; g += kThreads) {
        const bool sh = g >= p.E;
        int rows = sh ? p.T : p.offsets[g + 1] - p.offsets[g];
        int start = 0;
        if (p.tail_mode) {
            const int rem = rows % (2 * BM);
            start = rows - rem;
            rows = (rem > 0 && rem <= BM) ? rem : 0;
        }
        const int n = sh ? p.N_shared : p.N_routed;
        const int mt = (rows + BM - 1) / BM;
        s.rows[g] = rows;
        s.start[g] = start;
        s.row0[g] = sh ? 0 : p.offsets[g] + start;
        s.mtiles[g] = mt > 0 ? mt : 1;
        s.tile_start[g + 1] = mt * ((n + BNO - 1) / BNO);
    }
    __syncthreads();
    if (warp == 0) {            // inclusive scan of the per-group tile counts
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
            for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
                int g, mt, nt;
                decode(s, G, tile, g, mt, nt);
                const bool sh = g >= p.E;
                const int K = sh ? p.K_shared : p.K_routed;
                const int nk = (K + bk_elems<F8>() - 1) / bk_elems<F8>();
                const int a_row = sh ? (int)p.shared_a_row + s.start[g] + mt * BM : s.row0[g] + mt * BM;
                const CUtensorMap *mA = sh ? &tmAs : &tmA;
                const CUtensorMap *mB = sh ? &tmBs : &tmB;
                const CUtensorMap *mB2 = sh ? &tmBs2 : &tmB2;
                const int e = sh ? 0 : group_expert(p, g);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) { fail(s, p, 1); break; }
                    const uint32_t fb = smem_u32(&s.full[stage]);
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smA + stage * A_BYTES, mA, fb, kb * bk_elems<F8>(), a_row);
                    if (MODE == GM_SWIGLU) {
                        tma_load_3d(smB + stage * B_BYTES, mB, fb, kb * bk_elems<F8>(), nt * 128, e);
                        tma_load_3d(smB + stage * B_BYTES + B_BYTES / 2, mB2, fb, kb * bk_elems<F8>(), nt * 128, e);
                    } else {
                        tma_load_3d(smB + stage * B_BYTES, mB, fb, kb * bk_elems<F8>(), nt * BNB, e);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
                // the shared group, when there is one, is the last: its tiles start
                // at tile_start[E] (= total without one), so K needs no search
                const int K = tile >= s.tile_start[p.E] ? p.K_shared : p.K_routed;
                const int nk = (K + bk_elems<F8>() - 1) / bk_elems<F8>();
                if (!mbar_wait(smem_u32(&s.acce[ab]), aphase ^ 1u, p.timeout_ns)) { fail(s, p, 2); break; }
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(ab * BNB);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns)) { fail(s, p, 3); ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = smA + stage * A_BYTES, b0 = smB + stage * B_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        if (F8)
                            mma_e4m3(dtm, sdesc(a0 + k * 32), sdesc(b0 + k * 32), kIdescF8, (kb | k) ? 1u : 0u);
                        else
                            mma_bf16(dtm, sdesc(a0 + k * 32), sdesc(b0 + k * 32), kIdesc, (kb | k) ? 1u : 0u);
                    mma_commit(smem_u32(&s.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(smem_u32(&s.accf[ab]));
                if (++ab == 2) { ab = 0; aphase ^= 1u; }
            }
        }
    } else {
        // ================= epilogue: warps 2..9.  TMEM lane quadrant = warp % 4;
        // warps 2-5 take the first half of the tile's columns, warps 6-9 the second
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r_in_tile = q * 32 + lane;
        const uint32_t stg = base + (uint32_t)kStgOff + (uint32_t)(warp - 2) * STG_BYTES;
        float *scl = reinterpret_cast<float *>(smem + kStgOff + 8 * STG_BYTES + (warp - 2) * SCL_BYTES);
        int ab = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total && !aborted(s); tile += gridDim.x) {
            int g, mt, nt;
            decode(s, G, tile, g, mt, nt);
            const bool sh = g >= p.E;
            const int grow = mt * BM + r_in_tile;
            const bool valid = grow < s.rows[g];
            const int64_t orow = sh ? p.shared_out_row + s.start[g] + grow : (int64_t)s.row0[g] + grow;
            // the row's gate (and, for e4m3 tiles, the scales) are fetched
            // before the accumulator wait, hiding their latency
            float gscale = 1.f;
            if (MODE == GM_DOWN && !sh && valid) gscale = __ldg(p.row_gate + orow);
            const int N = sh ? p.N_shared : p.N_routed;
            float rscale = 0.f, csv[4] = {0.f, 0.f, 0.f, 0.f};
            if (F8)
                preload_scales<MODE>(p, sh, g, nt, half, N, valid, sh ? p.shared_a_row + s.start[g] + grow : orow,
                                     rscale, csv);
            // lane 0 waits, the warp follows its verdict (keeps the warp converged
            // for the .sync.aligned TMEM loads)
            int ok = 1;
            if (lane == 0) ok = mbar_wait(smem_u32(&s.accf[ab]), aphase, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) fail(s, p, 4); break; }
            __syncwarp();
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)(ab * BNB) + ((uint32_t)(q * 32) << 16);
            __nv_bfloat16 *orow_ptr = p.out + orow * p.ldo;
            const float *bias = (!sh && p.bias) ? p.bias + (size_t)group_expert(p, g) * p.N_routed : nullptr;
            const int64_t prow = sh ? orow - p.shared_out_row : orow;   // row in the pre-activation buffer
            epilogue_row<MODE, F8, SAVE>(taddr, half, nt, valid, N, orow_ptr, bias, gscale, &tmO, stg,
                                         (int)(orow - lane), rscale, csv, scl, sh ? &tmPs : &tmP,
                                         (int)(prow - lane),
                                         SAVE ? (sh ? p.pre_s + prow * p.pre_ld_s : p.pre + prow * p.pre_ld)
                                              : nullptr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&s.acce[ab]));
            if (++ab == 2) { ab = 0; aphase ^= 1u; }
        }
        if (lane == 0) tma_store_wait_all();            // the staged stores have landed
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    if (p.tail_mode) asm volatile("griddepcontrol.wait;" ::: "memory");
}


// ============================================================================
// CTA-pair version: one cluster of two CTAs computes a 256-row x 256-column
// accumulator with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16).  Each
// CTA loads its own 128 A rows and half of the B rows (SwiGLU: rank 0 the gate
// rows, rank 1 the up rows), so a CTA moves 32 KiB per 64-deep K step instead
// of 48 KiB; a stage holds two such K steps (three stages of 64 KiB), so one
// barrier round trip covers eight MMAs.  Rank 0 issues the MMAs;
// the full barriers live in rank 0 and collect both CTAs' TMA bytes; rank 0's
// commits arrive on both CTAs' empty and accumulator-full barriers; both
// CTAs' epilogue warps arrive on rank 0's accumulator-empty barriers.
// Pair tiles cover a group's 256-row blocks and a last block of more than 128
// rows; a last block of 1..128 rows runs in the 1-CTA kernel (tail mode), so
// row padding never exceeds that of 128-row tiles.
constexpr int P_STAGES = 3;
constexpr int P_ATOMS = 2;                         // 128-byte K atoms per stage
constexpr uint32_t P_A_BYTES = BM * BK * 2;         // 16 KiB: this CTA's 128 A rows
constexpr uint32_t P_B_BYTES = 128 * BK * 2;        // 16 KiB: this CTA's half of B
constexpr uint32_t P_STAGE_BYTES = P_ATOMS * (P_A_BYTES + P_B_BYTES);
constexpr int PM = 2 * BM;                          // rows per pair tile
constexpr uint32_t kIdescPair = make_idesc_bf16(PM, BNB);
constexpr uint32_t kIdescPairF8 = make_idesc_e4m3(PM, BNB);

struct PairTail {
    uint64_t full[P_STAGES];     // rank 0's are used
    uint64_t empty[P_STAGES];
    uint64_t accf[2];
    uint64_t acce[2];            // rank 0's are used: 8 warps x 2 CTAs
    uint32_t tmem_base;
    int abort_flag;
    int tile_start[kMaxGroups + 1];
    int mtiles[kMaxGroups];
    int rows[kMaxGroups];
    int row0[kMaxGroups];
};

constexpr size_t kPairStgOff = (P_STAGES * P_STAGE_BYTES + sizeof(PairTail) + 1023) / 1024 * 1024;
constexpr size_t kPairSmemBytes = 1024 + kPairStgOff + 8 * STG_BYTES + 8 * SCL_BYTES;
static_assert(kPairSmemBytes <= 227 * 1024, "pair kernel shared memory");

template <class Tail>
__device__ __forceinline__ void decode_pair(const Tail &s, int G, int tile, int &g, int &mt, int &nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int local = tile - s.tile_start[g];
    mt = local % s.mtiles[g];
    nt = local / s.mtiles[g];
}

template <class Tail>
__device__ __forceinline__ bool aborted_pair(const Tail &s) {
    return *reinterpret_cast<const volatile int *>(&s.abort_flag) != 0;
}
template <class Tail>
__device__ __forceinline__ void fail_pair(Tail &s, const GemmParams &p, int where) {
    record_error(p.status, MOE_ERR_TIMEOUT, where);
    *reinterpret_cast<volatile int *>(&s.abort_flag) = 1;
}

template <int MODE, bool F8, bool SAVE = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
tc_grouped_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                     const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                     const __grid_constant__ CUtensorMap tmBs, const __grid_constant__ CUtensorMap tmBs2,
                     const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmP,
                     const __grid_constant__ CUtensorMap tmPs, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    PairTail &s = *reinterpret_cast<PairTail *>(smem + P_STAGES * P_STAGE_BYTES);
    const uint32_t smA = base;                           // P_STAGES x 16 KiB
    const uint32_t smB = base + P_STAGES * P_ATOMS * P_A_BYTES;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = (int)cluster_id_x(), npairs = (int)ncluster_x();
    constexpr int BNO = (MODE == GM_SWIGLU) ? 128 : 256;
    const int G = p.E + (p.has_shared ? 1 : 0);

    // ---- independent of the previous kernel: barriers, TMEM, descriptors
    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < P_STAGES; ++i) { mbar_init(smem_u32(&s.full[i]), 1); mbar_init(smem_u32(&s.empty[i]), 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&s.accf[i]), 1); mbar_init(smem_u32(&s.acce[i]), 16); }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(&s.tmem_base), TMEM_COLS);   // warp 1 of both CTAs
    if (tid == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB2) : "memory");
    }
    pdl_wait_then_release();
    if (tid == 0) s.tile_start[0] = 0;
    for (int g = tid; g < G; g += kThreads) {
        const bool sh = g >= p.E;
        const int rows = sh ? p.T : p.offsets[g + 1] - p.offsets[g];
        const int n = sh ? p.N_shared : p.N_routed;
        const int mt = rows / PM + ((rows % PM) > BM ? 1 : 0);
        s.rows[g] = rows;
        s.row0[g] = sh ? 0 : p.offsets[g];
        s.mtiles[g] = mt > 0 ? mt : 1;
        s.tile_start[g + 1] = mt * ((n + BNO - 1) / BNO);
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
        // ================= TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = pair; tile < total && !aborted_pair(s); tile += npairs) {
                int g, mt, nt;
                decode_pair(s, G, tile, g, mt, nt);
                const bool sh = g >= p.E;
                const int K = sh ? p.K_shared : p.K_routed;
                const int nk = (K + P_ATOMS * bk_elems<F8>() - 1) / (P_ATOMS * bk_elems<F8>());
                const int a_row = (sh ? (int)p.shared_a_row : s.row0[g]) + mt * PM + (int)rank * BM;
                const CUtensorMap *mA = sh ? &tmAs : &tmA;
                const CUtensorMap *mB = (MODE == GM_SWIGLU && rank == 1) ? (sh ? &tmBs2 : &tmB2) : (sh ? &tmBs : &tmB);
                const int b_row = (MODE == GM_SWIGLU) ? nt * 128 : nt * BNB + (int)rank * 128;
                const int e = sh ? 0 : group_expert(p, g);
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) { fail_pair(s, p, 21); break; }
                    const uint32_t fb = mapa_shared(smem_u32(&s.full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&s.full[stage]), 2 * P_STAGE_BYTES);
#pragma unroll
                    for (int at = 0; at < P_ATOMS; ++at) {
                        const int kx = (kb * P_ATOMS + at) * bk_elems<F8>();
                        tma_load_2d_pair(smA + (stage * P_ATOMS + at) * P_A_BYTES, mA, fb, kx, a_row);
                        tma_load_3d_pair(smB + (stage * P_ATOMS + at) * P_B_BYTES, mB, fb, kx, b_row, e);
                    }
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer (rank 0 only)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            for (int tile = pair; tile < total && !aborted_pair(s); tile += npairs) {
                // the shared group, when there is one, is the last: its tiles start
                // at tile_start[E] (= total without one), so K needs no search
                const int K = tile >= s.tile_start[p.E] ? p.K_shared : p.K_routed;
                const int nk = (K + P_ATOMS * bk_elems<F8>() - 1) / (P_ATOMS * bk_elems<F8>());
                if (!mbar_wait(smem_u32(&s.acce[ab]), aphase ^ 1u, p.timeout_ns)) { fail_pair(s, p, 22); break; }
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(ab * BNB);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns)) { fail_pair(s, p, 23); ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < P_ATOMS * (BK / 16); ++kk) {
                        const int at = kk / (BK / 16), k = kk % (BK / 16);
                        const uint32_t a0 = smA + (stage * P_ATOMS + at) * P_A_BYTES;
                        const uint32_t b0 = smB + (stage * P_ATOMS + at) * P_B_BYTES;
                        if (F8)
                            mma_e4m3_pair(dtm, sdesc(a0 + k * 32), sdesc(b0 + k * 32), kIdescPairF8, (kb | kk) ? 1u : 0u);
                        else
                            mma_bf16_pair(dtm, sdesc(a0 + k * 32), sdesc(b0 + k * 32), kIdescPair, (kb | kk) ? 1u : 0u);
                    }
                    mma_commit_pair(smem_u32(&s.empty[stage]), (uint16_t)0x3);
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&s.accf[ab]), (uint16_t)0x3);
                if (++ab == 2) { ab = 0; aphase ^= 1u; }
            }
        }
    } else {
        // ================= epilogue (both CTAs), warps 2..9 as in the 1-CTA kernel
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r_in_tile = q * 32 + lane;
        const uint32_t stg = base + (uint32_t)kPairStgOff + (uint32_t)(warp - 2) * STG_BYTES;
        float *scl = reinterpret_cast<float *>(smem + kPairStgOff + 8 * STG_BYTES + (warp - 2) * SCL_BYTES);
        int ab = 0;
        uint32_t aphase = 0;
        for (int tile = pair; tile < total && !aborted_pair(s); tile += npairs) {
            int g, mt, nt;
            decode_pair(s, G, tile, g, mt, nt);
            const bool sh = g >= p.E;
            const int grow = mt * PM + (int)rank * BM + r_in_tile;
            const bool valid = grow < s.rows[g];
            const int64_t orow = sh ? p.shared_out_row + grow : (int64_t)s.row0[g] + grow;
            float gscale = 1.f;
            if (MODE == GM_DOWN && !sh && valid) gscale = __ldg(p.row_gate + orow);
            const int N = sh ? p.N_shared : p.N_routed;
            float rscale = 0.f, csv[4] = {0.f, 0.f, 0.f, 0.f};
            if (F8) preload_scales<MODE>(p, sh, g, nt, half, N, valid, sh ? p.shared_a_row + grow : orow, rscale, csv);
            int ok = 1;
            if (lane == 0) ok = mbar_wait(smem_u32(&s.accf[ab]), aphase, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) fail_pair(s, p, 24); break; }
            __syncwarp();
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)(ab * BNB) + ((uint32_t)(q * 32) << 16);
            __nv_bfloat16 *orow_ptr = p.out + orow * p.ldo;
            const float *bias = (!sh && p.bias) ? p.bias + (size_t)group_expert(p, g) * p.N_routed : nullptr;
            const int64_t prow = sh ? orow - p.shared_out_row : orow;   // row in the pre-activation buffer
            epilogue_row<MODE, F8, SAVE>(taddr, half, nt, valid, N, orow_ptr, bias, gscale, &tmO, stg,
                                         (int)(orow - lane), rscale, csv, scl, sh ? &tmPs : &tmP,
                                         (int)(prow - lane),
                                         SAVE ? (sh ? p.pre_s + prow * p.pre_ld_s : p.pre + prow * p.pre_ld)
                                              : nullptr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.acce[ab]), 0));
            if (++ab == 2) { ab = 0; aphase ^= 1u; }
        }
        if (lane == 0) tma_store_wait_all();            // the staged stores have landed
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


// The bf16 epilogue of one accumulator row with fewer registers than
// epilogue_row: SwiGLU takes gate and up chunk cc under one TMEM wait, the
// other modes one 32-column chunk per wait.
template <int MODE>
__device__ __forceinline__ void epilogue_row_lean(uint32_t taddr, int half, int nt, bool valid, int N,
                                               __nv_bfloat16 *orow_ptr, const float *bias, float gscale,
                                               const CUtensorMap *tmO, uint32_t stg, int row0) {
    const bool staged = __all_sync(0xffffffffu, valid);
    if (MODE == GM_SWIGLU) {
        const int c0 = half * 2;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            float v[64];
            tmem_ld32x2(taddr + (c0 + cc) * 32, taddr + 128 + (c0 + cc) * 32, v);   // gate, up
            const int col0 = nt * 128 + (c0 + cc) * 32;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * v[32 + i];
            if (staged) {
                if (col0 < N) stage_store32(stg, tmO, col0, row0, v);
            } else if (valid) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (col0 + u * 8 < N) store8(orow_ptr + col0 + u * 8, v + u * 8);
            }
        }
    } else {
        const int c0 = half * 4;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            tmem_ld32(taddr + (c0 + cc) * 32, v);
            {
                const int col0 = nt * BNB + (c0 + cc) * 32;
                if (col0 >= N) continue;                  // uniform over the warp
                float *h = v;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float z = h[i] + ((bias && col0 + i < N) ? __ldg(bias + col0 + i) : 0.f);
                    h[i] = (MODE == GM_GELU) ? gelu_erf(z) : gscale * z;
                }
                if (staged) {
                    stage_store32(stg, tmO, col0, row0, h);
                } else if (valid) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (col0 + u * 8 < N) store8(orow_ptr + col0 + u * 8, h + u * 8);
                }
            }
        }
    }
}

// ============================================================================
// INT4 weight-only experts on CTA pairs: the pair kernel above with its B
// operand decoded on the chip.  The TMA producer brings only A (this CTA's
// 128 rows, two 64-deep bf16 atoms per stage, on the first CTA's barrier as in
// the bf16 pair kernel).  The decode warps of each CTA (four: warp w owns B
// rows 32w .. 32w + 31 of the CTA's half) read their rows' packed codes (64
// bytes a row per stage) and bf16 group scale straight from global memory one
// stage ahead into registers; once the MMA has freed a stage they write its
// two bf16 B atoms in the 128-byte swizzled layout -- bf16(q * s), rounded
// once --, fence them for the tensor core and report to the first CTA, whose
// MMA thread starts once the stage's A has landed and every decode warp of
// the pair has reported.  The decode thus overlaps the A loads instead of
// following them.  Roles: warp 0 TMA, warp 1 MMA (first CTA), warps 2-9
// epilogue (the bf16 pair kernel's with fewer registers, so that 14 warps
// fit), warps 10-13 decode (one per SM sub-partition).
constexpr int W4P_STAGES = 3;
constexpr int W4P_DEC_WARPS = 4;                                // decode warps per CTA: 4 or 8
constexpr int W4P_DEC_ATOMS = P_ATOMS * 4 / W4P_DEC_WARPS;      // B atoms a decode warp writes per stage
constexpr int kW4Threads = (10 + W4P_DEC_WARPS) * 32;
constexpr uint32_t W4P_A_STAGE = P_ATOMS * P_A_BYTES;           // 32 KiB: two A atoms
constexpr uint32_t W4P_B_STAGE = P_ATOMS * P_B_BYTES;           // 32 KiB: two decoded B atoms

// Packed INT4 weights of one GEMM: codes [.., N, K/2] bytes (low nibble = even
// input, nibble = q + 8), scales [.., N, sld] bytes (one bf16 per 128 inputs).
struct W4Ptrs {
    const uint8_t *c, *c2, *cs, *cs2;      // codes: routed, routed SwiGLU up, shared, shared up
    const uint8_t *sc, *sc2, *scs, *scs2;  // scale rows, the same four
    int64_t sld;
};

struct W4PairTail {
    uint64_t full[W4P_STAGES];        // first CTA's: both CTAs' A landed
    uint64_t ready[W4P_STAGES];       // first CTA's: the pair's decode warps wrote B
    uint64_t empty[W4P_STAGES];
    uint64_t accf[2];
    uint64_t acce[2];                 // first CTA's: 8 warps x 2 CTAs
    uint32_t tmem_base;
    int abort_flag;
    int tile_start[kMaxGroups + 1];
    int mtiles[kMaxGroups];
    int rows[kMaxGroups];
    int row0[kMaxGroups];
};
constexpr size_t kW4TailOff = (size_t)W4P_STAGES * (W4P_A_STAGE + W4P_B_STAGE);
constexpr size_t kW4StgOff = (kW4TailOff + sizeof(W4PairTail) + 1023) / 1024 * 1024;
constexpr size_t kW4SmemBytes = 1024 + kW4StgOff + 8 * STG_BYTES;
static_assert(kW4SmemBytes <= 227 * 1024, "INT4 pair kernel shared memory");

// One decode warp's view of a tile: where its row's codes and scales start.
struct W4Row {
    const uint8_t *code;     // this thread's row, stage 0 (null past the weight's rows)
    const uint8_t *scale;
    int nk;                  // stages of the tile
};

template <int MODE>
__device__ __forceinline__ W4Row w4_row(const W4PairTail &s, const GemmParams &p, const W4Ptrs &w, int G, int tile,
                                        uint32_t rank, int n) {
    int g, mt, nt;
    decode_pair(s, G, tile, g, mt, nt);
    const bool sh = g >= p.E;
    const bool up = MODE == GM_SWIGLU && rank == 1;
    const int K = sh ? p.K_shared : p.K_routed;
    const int N = sh ? p.N_shared : p.N_routed;
    const int e = sh ? 0 : group_expert(p, g);
    const int row = ((MODE == GM_SWIGLU) ? nt * 128 : nt * BNB + (int)rank * 128) + n;
    W4Row r;
    r.nk = K / (P_ATOMS * BK);
    if (row < N) {
        const int64_t er = (int64_t)e * N + row;
        r.code = (sh ? (up ? w.cs2 : w.cs) : (up ? w.c2 : w.c)) + er * (K / 2);
        r.scale = (sh ? (up ? w.scs2 : w.scs) : (up ? w.sc2 : w.sc)) + er * w.sld;
    } else {
        r.code = nullptr;
        r.scale = nullptr;
    }
    return r;
}

// Stage kb of a row, atoms atom0 .. atom0 + W4P_DEC_ATOMS - 1: 32 code bytes
// (64 inputs) per atom and the stage's group scale; zeros past the weight's
// rows (decoding to zeros).
__device__ __forceinline__ void w4_fetch(const W4Row &r, int kb, int atom0, uint4 *c, uint32_t &s2) {
    if (r.code) {
        const uint4 *src = reinterpret_cast<const uint4 *>(r.code + (int64_t)kb * 64 + atom0 * 32);
#pragma unroll
        for (int j = 0; j < 2 * W4P_DEC_ATOMS; ++j) c[j] = __ldg(src + j);
        s2 = (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(r.scale) + kb) * 0x10001u;
    } else {
#pragma unroll
        for (int j = 0; j < 2 * W4P_DEC_ATOMS; ++j) c[j] = make_uint4(0u, 0u, 0u, 0u);
        s2 = 0u;
    }
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kW4Threads, 1)
tc_w4_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
                const __grid_constant__ CUtensorMap tmO, const GemmParams p, const W4Ptrs w) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    W4PairTail &s = *reinterpret_cast<W4PairTail *>(smem + kW4TailOff);
    const uint32_t smA = base;                                      // stages x 32 KiB
    const uint32_t smB = base + W4P_STAGES * W4P_A_STAGE;           // stages x 32 KiB

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = (int)cluster_id_x(), npairs = (int)ncluster_x();
    constexpr int BNO = (MODE == GM_SWIGLU) ? 128 : 256;
    constexpr int BKS = P_ATOMS * BK;                               // 128 of K per stage
    const int G = p.E + (p.has_shared ? 1 : 0);

    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < W4P_STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.ready[i]), 2 * W4P_DEC_WARPS);
            mbar_init(smem_u32(&s.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&s.accf[i]), 1); mbar_init(smem_u32(&s.acce[i]), 16); }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(&s.tmem_base), TMEM_COLS);
    if (tid == 0) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
    pdl_wait_then_release();
    if (tid == 0) s.tile_start[0] = 0;
    for (int g = tid; g < G; g += kW4Threads) {
        const bool sh = g >= p.E;
        const int rows = sh ? p.T : p.offsets[g + 1] - p.offsets[g];
        const int n = sh ? p.N_shared : p.N_routed;
        const int mt = rows / PM + ((rows % PM) > BM ? 1 : 0);
        s.rows[g] = rows;
        s.row0[g] = sh ? 0 : p.offsets[g];
        s.mtiles[g] = mt > 0 ? mt : 1;
        s.tile_start[g + 1] = mt * ((n + BNO - 1) / BNO);
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
        // ================= TMA producer of A (both CTAs, bytes on the first CTA's barrier)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int tile = pair; tile < total && !aborted_pair(s); tile += npairs) {
                int g, mt, nt;
                decode_pair(s, G, tile, g, mt, nt);
                const bool sh = g >= p.E;
                const int nk = (sh ? p.K_shared : p.K_routed) / BKS;
                const int a_row = (sh ? (int)p.shared_a_row : s.row0[g]) + mt * PM + (int)rank * BM;
                const CUtensorMap *mA = sh ? &tmAs : &tmA;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) { fail_pair(s, p, 61); break; }
                    const uint32_t fb = mapa_shared(smem_u32(&s.full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&s.full[stage]), 2 * W4P_A_STAGE);
#pragma unroll
                    for (int at = 0; at < P_ATOMS; ++at)
                        tma_load_2d_pair(smA + stage * W4P_A_STAGE + at * P_A_BYTES, mA, fb, kb * BKS + at * BK, a_row);
                    if (++stage == W4P_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer (first CTA only): the stage's A landed and its B decoded
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            for (int tile = pair; tile < total && !aborted_pair(s); tile += npairs) {
                const int K = tile >= s.tile_start[p.E] ? p.K_shared : p.K_routed;
                const int nk = K / BKS;
                if (!mbar_wait(smem_u32(&s.acce[ab]), aphase ^ 1u, p.timeout_ns)) { fail_pair(s, p, 62); break; }
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(ab * BNB);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns) ||
                        !mbar_wait(smem_u32(&s.ready[stage]), phase, p.timeout_ns)) {
                        fail_pair(s, p, 63);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < P_ATOMS * (BK / 16); ++kk) {
                        const int at = kk / (BK / 16), k = kk % (BK / 16);
                        const uint32_t a0 = smA + stage * W4P_A_STAGE + at * P_A_BYTES;
                        const uint32_t b0 = smB + stage * W4P_B_STAGE + at * P_B_BYTES;
                        mma_bf16_pair(dtm, sdesc(a0 + k * 32), sdesc(b0 + k * 32), kIdescPair, (kb | kk) ? 1u : 0u);
                    }
                    mma_commit_pair(smem_u32(&s.empty[stage]), (uint16_t)0x3);
                    if (++stage == W4P_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&s.accf[ab]), (uint16_t)0x3);
                if (++ab == 2) { ab = 0; aphase ^= 1u; }
            }
        }
    } else if (warp >= 10) {
        // ================= decode (both CTAs): warp 10 + w owns B rows 32 (w % 4) .. + 31 and
        // atoms (w / 4) W4P_DEC_ATOMS .. + W4P_DEC_ATOMS - 1 of each stage
        const int dw = warp - 10;
        const int n = (dw & 3) * 32 + lane;
        const int atom0 = (dw >> 2) * W4P_DEC_ATOMS;
        int stage = 0;
        uint32_t phase = 0;
        int tile = pair, kb = 0;
        if (tile < total) {
            W4Row row = w4_row<MODE>(s, p, w, G, tile, rank, n);
            uint4 c[2 * W4P_DEC_ATOMS];
            uint32_t s2;
            w4_fetch(row, 0, atom0, c, s2);
            while (true) {
                // the next stage's codes travel while this one is decoded
                int tile_n = tile, kb_n = kb + 1;
                W4Row row_n = row;
                if (kb_n == row.nk) {
                    tile_n = tile + npairs;
                    kb_n = 0;
                    if (tile_n < total) row_n = w4_row<MODE>(s, p, w, G, tile_n, rank, n);
                }
                uint4 cn[2 * W4P_DEC_ATOMS];
                uint32_t s2n = 0u;
                if (tile_n < total) w4_fetch(row_n, kb_n, atom0, cn, s2n);
                int okw = 1;
                if (lane == 0)
                    okw = (!aborted_pair(s) && mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) ? 1 : 0;
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) { if (lane == 0 && !aborted_pair(s)) fail_pair(s, p, 64); break; }
                const uint32_t bst = smB + stage * W4P_B_STAGE;
                const uint32_t *cw = reinterpret_cast<const uint32_t *>(c);
#pragma unroll
                for (int q = 0; q < 8 * W4P_DEC_ATOMS; ++q) {   // word q: inputs 8q .. of the warp's atoms
                    uint32_t o[4];
                    w4_decode8(cw[q], s2, o);
                    const uint32_t a = bst + (uint32_t)(atom0 + (q >> 3)) * P_B_BYTES + (uint32_t)n * 128 +
                                       ((uint32_t)((q & 7) ^ (n & 7)) << 4);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                 ::"r"(a), "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]) : "memory");
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.ready[stage]), 0));
                if (++stage == W4P_STAGES) { stage = 0; phase ^= 1u; }
                if (tile_n >= total) break;
                tile = tile_n;
                kb = kb_n;
                row = row_n;
#pragma unroll
                for (int j = 0; j < 2 * W4P_DEC_ATOMS; ++j) c[j] = cn[j];
                s2 = s2n;
            }
        }
    } else {
        // ================= epilogue (both CTAs), warps 2..9 as in the bf16 pair kernel
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r_in_tile = q * 32 + lane;
        const uint32_t stg = base + (uint32_t)kW4StgOff + (uint32_t)(warp - 2) * STG_BYTES;
        int ab = 0;
        uint32_t aphase = 0;
        for (int tile = pair; tile < total && !aborted_pair(s); tile += npairs) {
            int g, mt, nt;
            decode_pair(s, G, tile, g, mt, nt);
            const bool sh = g >= p.E;
            const int grow = mt * PM + (int)rank * BM + r_in_tile;
            const bool valid = grow < s.rows[g];
            const int64_t orow = sh ? p.shared_out_row + grow : (int64_t)s.row0[g] + grow;
            float gscale = 1.f;
            if (MODE == GM_DOWN && !sh && valid) gscale = __ldg(p.row_gate + orow);
            const int N = sh ? p.N_shared : p.N_routed;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(smem_u32(&s.accf[ab]), aphase, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) fail_pair(s, p, 67); break; }
            __syncwarp();
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)(ab * BNB) + ((uint32_t)(q * 32) << 16);
            __nv_bfloat16 *orow_ptr = p.out + orow * p.ldo;
            const float *bias = (!sh && p.bias) ? p.bias + (size_t)group_expert(p, g) * p.N_routed : nullptr;
            epilogue_row_lean<MODE>(taddr, half, nt, valid, N, orow_ptr, bias, gscale, &tmO, stg, (int)(orow - lane));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.acce[ab]), 0));
            if (++ab == 2) { ab = 0; aphase ^= 1u; }
        }
        if (lane == 0) tma_store_wait_all();            // the staged stores have landed
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

// ------------------------------------------------------------------ host side
}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// Tensor [outer][mid][inner] (inner contiguous) of bf16 (esize 2) or e4m3
// codes (esize 1), box {one 128-byte row of elements, box_mid(, 1)}.  rank 2
// maps (A operands) ignore `outer`; rank 3 maps (expert-stacked B operands)
// are indexed by expert in the third coordinate.
bool make_map(CUtensorMap *m, int rank, const void *base, uint64_t inner, uint64_t mid, uint64_t outer,
              uint64_t mid_stride_elems, uint64_t outer_stride_elems, uint32_t box_mid, int esize) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    if (outer_stride_elems == 0) outer_stride_elems = mid * mid_stride_elems;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {mid_stride_elems * esize, outer_stride_elems * esize};
    cuuint32_t box[3] = {(cuuint32_t)(128 / esize), box_mid, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapDataType dt = esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUresult r = enc(m, dt, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

// Output map for the staged epilogue stores: bf16 [rows][cols] with row
// stride ld elements, box 32 x 32, 64-byte swizzle.
bool make_store_map(CUtensorMap *m, void *base, uint64_t cols, uint64_t rows, uint64_t ld) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE, bool F8, bool SAVE = false>
cudaError_t launch_gemm(const CUtensorMap &A, const CUtensorMap &As, const CUtensorMap &B, const CUtensorMap &B2,
                        const CUtensorMap &Bs, const CUtensorMap &Bs2, const CUtensorMap &O, const CUtensorMap &P,
                        const CUtensorMap &Ps, const GemmParams &p, int grid, cudaStream_t st, bool pdl) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc_grouped_gemm<MODE, F8, SAVE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_kernel(tc_grouped_gemm<MODE, F8, SAVE>, dim3(grid), dim3(kThreads), kSmemBytes, st, pdl, A, As, B,
                         B2, Bs, Bs2, O, P, Ps, p);
}

template <int MODE, bool F8, bool SAVE = false>
cudaError_t launch_gemm_pair(const CUtensorMap &A, const CUtensorMap &As, const CUtensorMap &B,
                             const CUtensorMap &B2, const CUtensorMap &Bs, const CUtensorMap &Bs2,
                             const CUtensorMap &O, const CUtensorMap &P, const CUtensorMap &Ps, const GemmParams &p,
                             int num_sms, cudaStream_t st, bool pdl) {
    static int grid = 0;
    if (grid == 0) {
        cudaError_t e = cudaFuncSetAttribute(tc_grouped_gemm_pair<MODE, F8, SAVE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmemBytes);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = kPairSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, tc_grouped_gemm_pair<MODE, F8, SAVE>, &cfg);
        if (e != cudaSuccess || nclusters < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        grid = 2 * nclusters;
    }
    return launch_kernel(tc_grouped_gemm_pair<MODE, F8, SAVE>, dim3(grid), dim3(kThreads), kPairSmemBytes, st, pdl, A,
                         As, B, B2, Bs, Bs2, O, P, Ps, p);
}

}  // namespace

// Each GEMM runs as two launches on the stream: the CTA-pair kernel over the
// 256-row blocks of every group (and a last block of > 128 rows), then the
// 1-CTA kernel over the remaining last blocks of 1..128 rows.  With e4m3
// experts the first GEMM reads e4m3 x rows and weights and still writes H in
// bf16; H is then quantized per row (kept routed rows, then the shared rows)
// and the second GEMM reads the e4m3 H.
namespace {

template <bool F8>
cudaError_t run_ffn(const FfnArgs &a, cudaStream_t st) {
    constexpr int es = F8 ? 1 : 2;                 // bytes per A / B element
    const bool swiglu = a.act == MOE_ACT_SWIGLU;
    const bool has_sh = a.S > 0;
    const uint64_t routed_rows = (uint64_t)a.routed_rows;
    const uint64_t all_rows = routed_rows + (has_sh ? (uint64_t)a.T : 0);
    const int grid = a.num_sms > 0 ? a.num_sms : 148;
    const uint64_t timeout_ns = 2000000000ull;

    // ---- GEMM 1: H = act(X W1^T [+ b1])   (A: x_perm / x, B: W1 (+Wu) / Wsg (+Wsu))
    CUtensorMap A1, A1s, B1, B1u, B1s, B1su;
    const uint32_t box1 = swiglu ? 128 : 256;
    if (!make_map(&A1, 2, a.x_perm, a.d, routed_rows, 1, a.d, 0, BM, es)) return cudaErrorInvalidValue;
    if (!make_map(&B1, 3, a.W1, a.d, a.F, a.E, a.d, (uint64_t)a.F * a.d, box1, es)) return cudaErrorInvalidValue;
    if (swiglu) {
        if (!make_map(&B1u, 3, a.Wu, a.d, a.F, a.E, a.d, (uint64_t)a.F * a.d, box1, es)) return cudaErrorInvalidValue;
    } else {
        B1u = B1;
    }
    if (has_sh) {
        if (!make_map(&A1s, 2, a.x, a.d, a.T, 1, a.d, 0, BM, es)) return cudaErrorInvalidValue;
        if (!make_map(&B1s, 3, a.Wsg, a.d, a.S, 1, a.d, 0, box1, es)) return cudaErrorInvalidValue;
        if (swiglu) {
            if (!make_map(&B1su, 3, a.Wsu, a.d, a.S, 1, a.d, 0, box1, es)) return cudaErrorInvalidValue;
        } else {
            B1su = B1s;
        }
    } else {
        A1s = A1; B1s = B1; B1su = B1u;
    }
    GemmParams p1{};
    p1.offsets = a.offsets;
    p1.bias = swiglu ? nullptr : a.b1;
    p1.row_gate = nullptr;
    p1.out = static_cast<__nv_bfloat16 *>(a.H);
    p1.status = a.status;
    p1.E = a.n_groups; p1.E_w = a.E; p1.T = a.T;
    p1.K_routed = a.d; p1.K_shared = a.d;
    p1.N_routed = a.F; p1.N_shared = a.S;
    p1.has_shared = has_sh ? 1 : 0;
    p1.ldo = a.hF;
    p1.shared_a_row = 0;
    p1.shared_out_row = a.shared_base;
    p1.timeout_ns = timeout_ns;
    if (F8) {
        p1.row_scale = a.xperm_scale;
        p1.shared_row_scale = a.x_scale;
        p1.col_scale = a.W1s;
        p1.col_scale2 = swiglu ? a.Wus : nullptr;
        p1.sh_col_scale = a.Wsgs;
        p1.sh_col_scale2 = swiglu ? a.Wsus : nullptr;
    }
    // pair kernel: B boxes of 128 rows (each CTA loads half of the tile's B rows)
    CUtensorMap P1, P1u, P1s, P1su;
    if (swiglu) {
        P1 = B1; P1u = B1u; P1s = B1s; P1su = B1su;
    } else {
        if (!make_map(&P1, 3, a.W1, a.d, a.F, a.E, a.d, (uint64_t)a.F * a.d, 128, es)) return cudaErrorInvalidValue;
        P1u = P1;
        if (has_sh) {
            if (!make_map(&P1s, 3, a.Wsg, a.d, a.S, 1, a.d, 0, 128, es)) return cudaErrorInvalidValue;
        } else {
            P1s = P1;
        }
        P1su = P1s;
    }
    // the first GEMM's output: H [all rows, hF], stored in 32 x 32 blocks
    CUtensorMap O1;
    if (!make_store_map(&O1, a.H, a.hF, all_rows, a.hF)) return cudaErrorInvalidValue;
    cudaError_t err;
    if (!F8 && a.pre) {
        // training forward: the pre-activations too (routed rows, then the shared rows' own buffer)
        const int gw = swiglu ? 2 : 1;
        CUtensorMap Q1, Q1s;
        if (!make_store_map(&Q1, a.pre, (uint64_t)gw * a.F, routed_rows > 0 ? routed_rows : 1, (uint64_t)gw * a.F))
            return cudaErrorInvalidValue;
        if (has_sh) {
            if (!make_store_map(&Q1s, a.pre_s, (uint64_t)gw * a.S, (uint64_t)a.T, (uint64_t)gw * a.S))
                return cudaErrorInvalidValue;
        } else {
            Q1s = Q1;
        }
        p1.pre = static_cast<__nv_bfloat16 *>(a.pre);
        p1.pre_s = static_cast<__nv_bfloat16 *>(a.pre_s);
        p1.pre_ld = (int64_t)gw * a.F;
        p1.pre_ld_s = (int64_t)gw * a.S;
        err = swiglu ? launch_gemm_pair<GM_SWIGLU, false, true>(A1, A1s, P1, P1u, P1s, P1su, O1, Q1, Q1s, p1, grid, st,
                                                                a.pdl)
                     : launch_gemm_pair<GM_GELU, false, true>(A1, A1s, P1, P1u, P1s, P1su, O1, Q1, Q1s, p1, grid, st,
                                                              a.pdl);
        if (err != cudaSuccess) return err;
        p1.tail_mode = 1;
        err = swiglu ? launch_gemm<GM_SWIGLU, false, true>(A1, A1s, B1, B1u, B1s, B1su, O1, Q1, Q1s, p1, grid, st, true)
                     : launch_gemm<GM_GELU, false, true>(A1, A1s, B1, B1u, B1s, B1su, O1, Q1, Q1s, p1, grid, st, true);
        if (err != cudaSuccess) return err;
    } else {
        err = swiglu ? launch_gemm_pair<GM_SWIGLU, F8>(A1, A1s, P1, P1u, P1s, P1su, O1, O1, O1, p1, grid, st, a.pdl)
                     : launch_gemm_pair<GM_GELU, F8>(A1, A1s, P1, P1u, P1s, P1su, O1, O1, O1, p1, grid, st, a.pdl);
        if (err != cudaSuccess) return err;
        p1.tail_mode = 1;
        err = swiglu ? launch_gemm<GM_SWIGLU, F8>(A1, A1s, B1, B1u, B1s, B1su, O1, O1, O1, p1, grid, st, true)
                     : launch_gemm<GM_GELU, F8>(A1, A1s, B1, B1u, B1s, B1su, O1, O1, O1, p1, grid, st, true);
        if (err != cudaSuccess) return err;
    }

    // ---- e4m3: quantize H per row (kept routed rows, then the shared rows)
    if (F8) {
        QuantArgs q{};
        q.in = static_cast<const __nv_bfloat16 *>(a.H);
        q.ld_in = a.hF;
        q.out = a.H8;
        q.ld_out = a.hF;
        q.scale = a.h_scale;
        q.rows = (int64_t)routed_rows;
        q.row0 = 0;
        q.cols = a.F;
        q.rows_limit = a.offsets + a.n_groups;
        q.num_sms = a.num_sms;
        q.pdl = true;
        if ((err = launch_quant_rows(q, st)) != cudaSuccess) return err;
        if (has_sh) {
            q.rows = a.T;
            q.row0 = a.shared_base;
            q.cols = a.S;
            q.rows_limit = nullptr;
            if ((err = launch_quant_rows(q, st)) != cudaSuccess) return err;
        }
    }

    // ---- GEMM 2: Y = gate * (H W2^T [+ b2])   (A: H / H8, B: W2 / Wsd)
    const void *Ain = F8 ? static_cast<const void *>(a.H8) : a.H;
    CUtensorMap A2, A2s, B2m, B2s;
    if (!make_map(&A2, 2, Ain, a.F, all_rows, 1, a.hF, 0, BM, es)) return cudaErrorInvalidValue;
    if (!make_map(&B2m, 3, a.W2, a.F, a.d, a.E, a.F, (uint64_t)a.d * a.F, BNB, es)) return cudaErrorInvalidValue;
    if (has_sh) {
        if (!make_map(&A2s, 2, Ain, a.S, all_rows, 1, a.hF, 0, BM, es)) return cudaErrorInvalidValue;
        if (!make_map(&B2s, 3, a.Wsd, a.S, a.d, 1, a.S, 0, BNB, es)) return cudaErrorInvalidValue;
    } else {
        A2s = A2; B2s = B2m;
    }
    GemmParams p2{};
    p2.offsets = a.offsets;
    p2.bias = swiglu ? nullptr : a.b2;
    p2.row_gate = a.row_gate;
    p2.out = static_cast<__nv_bfloat16 *>(a.y_perm);
    p2.status = a.status;
    p2.E = a.n_groups; p2.E_w = a.E; p2.T = a.T;
    p2.K_routed = a.F; p2.K_shared = a.S;
    p2.N_routed = a.d; p2.N_shared = a.d;
    p2.has_shared = has_sh ? 1 : 0;
    p2.ldo = a.d;
    p2.shared_a_row = a.shared_base;
    p2.shared_out_row = a.shared_base;
    p2.timeout_ns = timeout_ns;
    if (F8) {
        p2.row_scale = a.h_scale;
        p2.shared_row_scale = a.h_scale;
        p2.col_scale = a.W2s;
        p2.sh_col_scale = a.Wsds;
    }
    CUtensorMap P2, P2s;
    if (!make_map(&P2, 3, a.W2, a.F, a.d, a.E, a.F, (uint64_t)a.d * a.F, 128, es)) return cudaErrorInvalidValue;
    if (has_sh) {
        if (!make_map(&P2s, 3, a.Wsd, a.S, a.d, 1, a.S, 0, 128, es)) return cudaErrorInvalidValue;
    } else {
        P2s = P2;
    }
    CUtensorMap O2;                               // y_perm [all rows, d_model]
    if (!make_store_map(&O2, a.y_perm, a.d, all_rows, a.d)) return cudaErrorInvalidValue;
    err = launch_gemm_pair<GM_DOWN, F8>(A2, A2s, P2, P2, P2s, P2s, O2, O2, O2, p2, grid, st, true);
    if (err != cudaSuccess) return err;
    p2.tail_mode = 1;
    return launch_gemm<GM_DOWN, F8>(A2, A2s, B2m, B2m, B2s, B2s, O2, O2, O2, p2, grid, st, true);
}

}  // namespace

namespace {

template <int MODE>
cudaError_t launch_w4_pair_mode(const W4PairArgs &a, const CUtensorMap &O, const GemmParams &p, cudaStream_t st) {
    static int grid = 0;
    if (grid == 0) {
        cudaError_t e = cudaFuncSetAttribute(tc_w4_gemm_pair<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kW4SmemBytes);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (a.num_sms / 2), 1, 1);
        cfg.blockDim = dim3(kW4Threads, 1, 1);
        cfg.dynamicSmemBytes = kW4SmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, tc_w4_gemm_pair<MODE>, &cfg);
        if (e != cudaSuccess || nclusters < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        grid = 2 * nclusters;
    }
    W4Ptrs w{};
    w.c = a.c; w.c2 = a.c2; w.cs = a.cs; w.cs2 = a.cs2;
    w.sc = a.sc; w.sc2 = a.sc2; w.scs = a.scs; w.scs2 = a.scs2;
    w.sld = a.sld;
    return launch_kernel(tc_w4_gemm_pair<MODE>, dim3(grid), dim3(kW4Threads), kW4SmemBytes, st, a.pdl, a.A, a.As, O,
                         p, w);
}

}  // namespace

cudaError_t launch_w4_gemm_pair(const W4PairArgs &a, cudaStream_t st) {
    if (a.K_routed % 128 != 0 || (a.has_shared && a.K_shared % 128 != 0) || a.E + 1 > kMaxGroups)
        return cudaErrorInvalidValue;
    CUtensorMap O;
    if (!make_store_map(&O, a.out, a.out_cols, a.out_rows > 0 ? a.out_rows : 1, (uint64_t)a.ldo))
        return cudaErrorInvalidValue;
    GemmParams p{};
    p.offsets = a.offsets;
    p.bias = a.bias;
    p.row_gate = a.row_gate;
    p.out = a.out;
    p.status = a.status;
    p.E = a.E; p.E_w = a.E; p.T = a.T;
    p.K_routed = a.K_routed; p.K_shared = a.K_shared;
    p.N_routed = a.N_routed; p.N_shared = a.N_shared;
    p.has_shared = a.has_shared;
    p.ldo = a.ldo;
    p.shared_a_row = a.shared_a_row;
    p.shared_out_row = a.shared_out_row;
    p.timeout_ns = 2000000000ull;
    switch (a.mode) {
        case GM_SWIGLU: return launch_w4_pair_mode<GM_SWIGLU>(a, O, p, st);
        case GM_GELU: return launch_w4_pair_mode<GM_GELU>(a, O, p, st);
        case GM_DOWN: return launch_w4_pair_mode<GM_DOWN>(a, O, p, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_ffn_bf16(const FfnArgs &a, cudaStream_t st) {
    if (a.routed_rows == 0 && (a.S == 0 || a.T == 0)) return cudaSuccess;
    return a.f8 ? run_ffn<true>(a, st) : run_ffn<false>(a, st);
}

}  // namespace moe
