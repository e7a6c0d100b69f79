// mx_sm100.cu -- block-scaled (MX) e4m3 experts on sm_100a.
//
// The serving page recommends quantized experts once weight bytes bind
// ("Fine-tuning and serving MoE models", Serving: throughput does not scale
// the way you expect).  This is the block-scaled form, laid out as OCP MX
// FP8: along the contraction dimension every 32 consecutive values share one
// power-of-two scale 2^X, stored as the byte X + 127 (E8M0):
//   amax = max |v| over the 32 values,  X = floor(log2 amax) - 8 clamped to
//   [-127, 127] (-127 for amax = 0 or a subnormal amax),
//   code = e4m3(v * 2^-X), round to nearest even, saturating at 448.
// The multiplication by 2^-X is exact in fp32, so the codes are a function of
// the bf16 inputs alone.
//
//   mx_quant_kernel  bf16 rows -> e4m3 codes + scale bytes (rows of `sld`
//                    bytes), one warp per row, four lanes per 32-value block
//   tc_mx_gemm       grouped GEMM with tcgen05.mma.kind::mxf8f6f4.block_scale:
//                    one CTA per SM, 128 x 128 tiles, K = 128 per stage
//       warp 0     TMA: per stage the A tile (128 rows x 128 codes), the B
//                  tile (128 weight rows, SwiGLU: 64 gate + 64 up rows) and
//                  16-byte-wide boxes of both operands' scale rows holding
//                  the stage's 4 scale bytes per row
//       warps 2-5  one per TMEM lane quadrant: move the stage's scale words
//                  (4 bytes = the 4 blocks of 32 of one row) from shared
//                  memory into the TMEM scale slots -- row 32c + l in column
//                  c of lane l, the same in every quadrant -- with tcgen05.st
//       warp 1     single-thread MMA: per stage four K = 32 instructions,
//                  the j-th reading byte j of the scale words
//       warps 6-9  epilogue, one per lane quadrant: TMEM -> registers, the
//                  fused SwiGLU / GELU + bias / gate, bf16 stores of whole
//                  64-byte row segments through a per-warp staging buffer
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace moe {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();   // ffn_sm100.cu

namespace {

// ------------------------------------------------------------------ quantizer
constexpr int kMxQuantThreads = 256;

__global__ void __launch_bounds__(kMxQuantThreads) mx_quant_kernel(QuantMxArgs a) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    int64_t nrows = a.rows;
    if (a.rows_limit) {
        const int64_t lim = *a.rows_limit;
        nrows = lim < 0 ? 0 : (lim < nrows ? lim : nrows);
    }
    const int64_t wid = ((int64_t)blockIdx.x * kMxQuantThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kMxQuantThreads) >> 5;
    const int nvec = a.cols >> 3;                      // 8 values per lane and step; a multiple of 4
    for (int64_t r = wid; r < nrows; r += nw) {
        const int64_t row = a.row0 + r;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.in + row * a.ld_in);
        uint2 *dst = reinterpret_cast<uint2 *>(a.out + row * a.ld_out);
        uint8_t *srow = a.scale + row * a.ld_scale;
        for (int v0 = 0; v0 < nvec; v0 += 32) {        // the same trip count on every lane
            const int v = v0 + lane;
            const bool on = v < nvec;                  // whole 4-lane blocks are on or off
            float f[8];
            float amax = 0.f;
            if (on) {
                const uint4 u = src[v];
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 p = __bfloat1622float2(h[i]);
                    f[2 * i] = p.x;
                    f[2 * i + 1] = p.y;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            if (!on) continue;
            // X = floor(log2 amax) - 8 from the exponent field; a zero or
            // subnormal amax (field 0) gives X <= -127 - 8, clamped to -127
            const int ef = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
            const int X = ef == 0 ? -127 : max(-127, ef - 127 - 8);
            const float inv = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X, a normal float
            uint32_t w[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(f[4 * hh], inv), __fmul_rn(f[4 * hh + 1], inv)), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fmul_rn(f[4 * hh + 2], inv), __fmul_rn(f[4 * hh + 3], inv)), __NV_SATFINITE,
                    __NV_E4M3);
                w[hh] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            dst[v] = make_uint2(w[0], w[1]);
            if ((lane & 3) == 0) srow[v >> 2] = (uint8_t)(X + 127);
        }
    }
}

// dst[r, :] = src[row_token[r], :] for r < *count: the scale rows of the
// packed rows (bytes per row a multiple of 16).  One warp per row.
__global__ void __launch_bounds__(256) mx_gather_rows_kernel(const uint8_t *src, uint8_t *dst, int64_t ld,
                                                             const int32_t *row_token, const int32_t *count,
                                                             int64_t max_rows) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    int64_t n = *count;
    n = n < 0 ? 0 : (n < max_rows ? n : max_rows);
    const int nvec = (int)(ld / 16);
    const int64_t nw = (int64_t)gridDim.x * 8;
    for (int64_t r = blockIdx.x * 8 + (threadIdx.x >> 5); r < n; r += nw) {
        const uint4 *s = reinterpret_cast<const uint4 *>(src + (int64_t)row_token[r] * ld);
        uint4 *d = reinterpret_cast<uint4 *>(dst + r * ld);
        for (int v = lane; v < nvec; v += 32) d[v] = __ldg(s + v);
    }
}

// ------------------------------------------------------------------ grouped GEMM
// Two kinds share the kernel: MX (e4m3 A and B with E8M0 block scales, K =
// 128 per stage, one 128-byte row of codes) and W4 (bf16 A, INT4 weight-only
// B: K = 64 per stage, one 128-byte row of bf16; the B codes, 32 bytes per
// row, and their bf16 scales arrive by TMA and four warps decode them into the
// stage's bf16 B tile).
enum { KIND_MX = 0, KIND_W4 = 1 };
constexpr int MX_BM = 128, MX_BN = 128;
constexpr int MX_STAGES = 5;
constexpr int kMxThreads = 320;
constexpr uint32_t MX_A_BYTES = MX_BM * 128;            // 16 KiB: 128 rows x 128 bytes
constexpr uint32_t MX_B_BYTES = MX_BN * 128;            // 16 KiB
constexpr uint32_t MX_SA_BYTES = MX_BM * 16;            // MX: 128 rows x 16 scale bytes
constexpr uint32_t MX_SB_BYTES = MX_BN * 16;            // MX: B scale rows; W4: B bf16 scale rows
constexpr uint32_t W4_CODE_BYTES = MX_BN * 32;          // W4: 128 rows x 64 nibbles
template <int KIND> constexpr int kind_bk() { return KIND == KIND_MX ? 128 : 64; }
// Per stage: A | B | (MX) A scales, B scales | (W4) B codes, B scales; the same size for both kinds.
constexpr uint32_t MX_STAGE_BYTES = MX_A_BYTES + MX_B_BYTES + MX_SA_BYTES + MX_SB_BYTES;   // 36 KiB
static_assert(MX_SA_BYTES + MX_SB_BYTES <= W4_CODE_BYTES + MX_SB_BYTES, "W4 stage layout");
constexpr uint32_t W4_STAGE_BYTES = MX_A_BYTES + MX_B_BYTES + W4_CODE_BYTES + MX_SB_BYTES;  // 38 KiB
constexpr uint32_t STAGE_STRIDE = W4_STAGE_BYTES;       // both kinds use the larger stride
constexpr uint32_t MX_TMEM_COLS = 512;
constexpr uint32_t MX_SF_COL0 = 2 * MX_BN;              // scale slots after the two accumulators
constexpr int kMxMaxGroups = 257;
constexpr uint32_t MX_STG_BYTES = 32 * 64;              // per epilogue warp: 32 rows x 64 bytes

enum { MX_SWIGLU = 0, MX_GELU = 1, MX_DOWN = 2 };

// kind::mxf8f6f4 block-scaled instruction descriptor: e4m3 A and B (format
// 0), K-major, E8M0 scales (bit 23), N >> 3 at bit 17, M >> 4 at bit 24, the
// scale byte of A at bits 29-30 and of B at bits 4-5.
__host__ __device__ constexpr uint32_t mx_idesc(uint32_t M, uint32_t N, uint32_t sf_id) {
    return (sf_id << 4) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void mma_mx(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t *w) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};"
                 ::"r"(taddr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
}

struct MxParams {
    const int32_t *offsets;      // [E+1]: routed group g holds rows offsets[g] .. offsets[g+1]
    const float *bias;           // [E, N_routed] or null (GELU b1 / b2)
    const float *row_gate;       // MX_DOWN: [rows] or null
    __nv_bfloat16 *out;
    int64_t ldo;
    int32_t *status;
    uint64_t timeout_ns;
    int E, T, has_shared;        // the shared group, if any, is group E over all T tokens
    int K_routed, K_shared;      // contraction lengths, multiples of 128
    int N_routed, N_shared;      // output columns
    int64_t shared_a_row;        // first A row of the shared group in the shared maps
    int64_t shared_out_row;      // first output row of the shared group
    int tail_mode;               // 1: only a group's last rows when rows % 256 is in 1..128
                                 // (the CTA-pair INT4 kernel runs the rest)
};

struct MxSmem {
    uint64_t full[MX_STAGES];    // TMA bytes of the stage landed
    uint64_t sf_full[MX_STAGES]; // the stage's scale words are in TMEM (4 warps)
    uint64_t empty[MX_STAGES];   // the stage's MMAs completed
    uint64_t accf[2];
    uint64_t acce[2];            // 4 epilogue warps
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int tile_start[kMxMaxGroups + 1];
    int mtiles[kMxMaxGroups];
    int rows[kMxMaxGroups];
    int row0[kMxMaxGroups];
};
constexpr size_t kMxStgOff = ((size_t)MX_STAGES * STAGE_STRIDE + sizeof(MxSmem) + 1023) / 1024 * 1024;
constexpr size_t kMxSmemBytes = 1024 + kMxStgOff + 4 * MX_STG_BYTES;
static_assert(kMxSmemBytes <= 227 * 1024, "MX GEMM shared memory");

__device__ __forceinline__ bool mx_aborted(const MxSmem &s) {
    return *reinterpret_cast<const volatile int *>(&s.abort_flag) != 0;
}
__device__ __forceinline__ void mx_fail(MxSmem &s, const MxParams &p, int where) {
    record_error(p.status, MOE_ERR_TIMEOUT, where);
    *reinterpret_cast<volatile int *>(&s.abort_flag) = 1;
}
__device__ __forceinline__ void mx_decode(const MxSmem &s, int G, int tile, int &g, int &mt, int &nt) {
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

__device__ __forceinline__ float mx_silu(float v) { return __fdividef(v, 1.f + __expf(-v)); }
__device__ __forceinline__ float mx_gelu(float v) { return 0.5f * v * (1.f + erff(v * 0.70710678118654752f)); }

// 32 rows x 32 bf16 columns of the warp (this lane's row in h) to global
// memory: through the staging buffer (16-byte piece c of row r at slot
// c ^ ((r / 2) % 4)), then eight 64-byte row segments per store instruction;
// rows 0..nrows-1 only.
__device__ __forceinline__ void mx_store32(uint32_t stg, const float *h, __nv_bfloat16 *row0_ptr, int64_t ldo,
                                           int nrows) {
    const int lane = threadIdx.x & 31;
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(h[2 * i], h[2 * i + 1]);
        pk[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t a = stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * c]), "r"(pk[4 * c + 1]),
                     "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3]) : "memory");
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = i * 32 + lane, r = j >> 2, c = j & 3;
        if (r < nrows) {
            uint4 v;
            const uint32_t a = stg + r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
            *reinterpret_cast<uint4 *>(row0_ptr + r * ldo + c * 8) = v;
        }
    }
}

template <int MODE, int KIND>
__global__ void __launch_bounds__(kMxThreads, 1)
tc_mx_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
           const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSAs,
           const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
           const __grid_constant__ CUtensorMap tmBs, const __grid_constant__ CUtensorMap tmBs2,
           const __grid_constant__ CUtensorMap tmSB, const __grid_constant__ CUtensorMap tmSB2,
           const __grid_constant__ CUtensorMap tmSBs, const __grid_constant__ CUtensorMap tmSBs2,
           const MxParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (base - raw_addr);
    MxSmem &s = *reinterpret_cast<MxSmem *>(smem + MX_STAGES * STAGE_STRIDE);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int BK = kind_bk<KIND>();
    const int G = p.E + (p.has_shared ? 1 : 0);
    constexpr int OUT_COLS = (MODE == MX_SWIGLU) ? MX_BN / 2 : MX_BN;   // output columns per tile

    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < MX_STAGES; ++i) {
            mbar_init(smem_u32(&s.full[i]), 1);
            mbar_init(smem_u32(&s.sf_full[i]), 4);
            mbar_init(smem_u32(&s.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) { mbar_init(smem_u32(&s.accf[i]), 1); mbar_init(smem_u32(&s.acce[i]), 4); }
        mbar_init(smem_u32(&s.drain), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(&s.tmem_base), MX_TMEM_COLS);
    // Last blocks (tail mode) touch only rows the CTA-pair launch before them
    // leaves alone and read only what the kernel before that wrote, so they
    // start at once and wait for the pair launch only before exiting.
    if (p.tail_mode) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    else pdl_wait_then_release();
    if (tid == 0) s.tile_start[0] = 0;
    for (int g = tid; g < G; g += kMxThreads) {
        const bool sh = g >= p.E;
        int rows = sh ? p.T : p.offsets[g + 1] - p.offsets[g];
        int start = 0;
        if (p.tail_mode) {
            const int rem = rows % (2 * MX_BM);
            start = rows - rem;
            rows = (rem > 0 && rem <= MX_BM) ? rem : 0;
        }
        const int n = sh ? p.N_shared : p.N_routed;
        const int mt = (rows + MX_BM - 1) / MX_BM;
        s.rows[g] = rows;
        s.row0[g] = sh ? start : p.offsets[g] + start;      // the shared group: offset past shared_*_row
        s.mtiles[g] = mt > 0 ? mt : 1;
        s.tile_start[g + 1] = mt * ((n + OUT_COLS - 1) / OUT_COLS);
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
            int last_phase[MX_STAGES];
#pragma unroll
            for (int i = 0; i < MX_STAGES; ++i) last_phase[i] = -1;
            for (int tile = blockIdx.x; tile < total && !mx_aborted(s); tile += gridDim.x) {
                int g, mt, nt;
                mx_decode(s, G, tile, g, mt, nt);
                const bool sh = g >= p.E;
                const int K = sh ? p.K_shared : p.K_routed;
                const int nk = K / BK;
                const int a_row = sh ? (int)p.shared_a_row + s.row0[g] + mt * MX_BM : s.row0[g] + mt * MX_BM;
                const int e = sh ? 0 : g;
                const CUtensorMap *mA = sh ? &tmAs : &tmA, *mSA = sh ? &tmSAs : &tmSA;
                const CUtensorMap *mB = sh ? &tmBs : &tmB, *mB2 = sh ? &tmBs2 : &tmB2;
                const CUtensorMap *mSB = sh ? &tmSBs : &tmSB, *mSB2 = sh ? &tmSBs2 : &tmSB2;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.empty[stage]), phase ^ 1u, p.timeout_ns)) { mx_fail(s, p, 41); break; }
                    const uint32_t fb = smem_u32(&s.full[stage]);
                    const uint32_t a_dst = base + stage * STAGE_STRIDE;
                    const uint32_t b_dst = a_dst + MX_A_BYTES;
                    if (KIND == KIND_W4) {
                        // A (bf16, 64 of K), the B codes (32 bytes of each of 128 rows) and the
                        // 16-byte box of B scale bytes holding the stage's group scale
                        mbar_arrive_expect_tx(fb, MX_A_BYTES + W4_CODE_BYTES + MX_SB_BYTES);
                        const uint32_t c_dst = b_dst + MX_B_BYTES;
                        const uint32_t s_dst = c_dst + W4_CODE_BYTES;
                        const int cx = kb * 32;                       // code bytes: 64 nibbles per stage
                        const int gx = ((kb >> 1) * 2) & ~15;         // scale bytes: group kb / 2, bf16
                        tma_load_2d(a_dst, mA, fb, kb * BK, a_row);
                        if (MODE == MX_SWIGLU) {
                            const int j0 = nt * OUT_COLS;
                            tma_load_3d(c_dst, mB, fb, cx, j0, e);
                            tma_load_3d(c_dst + W4_CODE_BYTES / 2, mB2, fb, cx, j0, e);
                            tma_load_3d(s_dst, mSB, fb, gx, j0, e);
                            tma_load_3d(s_dst + MX_SB_BYTES / 2, mSB2, fb, gx, j0, e);
                        } else {
                            tma_load_3d(c_dst, mB, fb, cx, nt * MX_BN, e);
                            tma_load_3d(s_dst, mSB, fb, gx, nt * MX_BN, e);
                        }
#pragma unroll
                        for (int i = 0; i < MX_STAGES; ++i)
                            if (i == stage) last_phase[i] = (int)phase;
                        if (++stage == MX_STAGES) { stage = 0; phase ^= 1u; }
                        continue;
                    }
                    mbar_arrive_expect_tx(fb, MX_STAGE_BYTES);
                    const uint32_t sa_dst = b_dst + MX_B_BYTES;
                    const uint32_t sb_dst = sa_dst + MX_SA_BYTES;
                    const int kx = kb * BK;
                    const int sx = (kb * 4) & ~15;          // 16-byte box holding the stage's 4 scale bytes
                    tma_load_2d(a_dst, mA, fb, kx, a_row);
                    tma_load_2d(sa_dst, mSA, fb, sx, a_row);
                    if (MODE == MX_SWIGLU) {
                        const int j0 = nt * OUT_COLS;
                        tma_load_3d(b_dst, mB, fb, kx, j0, e);
                        tma_load_3d(b_dst + MX_B_BYTES / 2, mB2, fb, kx, j0, e);
                        tma_load_3d(sb_dst, mSB, fb, sx, j0, e);
                        tma_load_3d(sb_dst + MX_SB_BYTES / 2, mSB2, fb, sx, j0, e);
                    } else {
                        tma_load_3d(b_dst, mB, fb, kx, nt * MX_BN, e);
                        tma_load_3d(sb_dst, mSB, fb, sx, nt * MX_BN, e);
                    }
#pragma unroll
                    for (int i = 0; i < MX_STAGES; ++i)
                        if (i == stage) last_phase[i] = (int)phase;
                    if (++stage == MX_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // no load may still be writing this CTA's shared memory when it exits
#pragma unroll
            for (int i = 0; i < MX_STAGES; ++i)
                if (last_phase[i] >= 0 && !mbar_wait(smem_u32(&s.full[i]), (uint32_t)last_phase[i], p.timeout_ns))
                    mx_fail(s, p, 46);
        }
    } else if (warp == 1) {
        // ================= MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int ab = 0;
            uint32_t aphase = 0;
            for (int tile = blockIdx.x; tile < total && !mx_aborted(s); tile += gridDim.x) {
                const int K = tile >= s.tile_start[p.E] ? p.K_shared : p.K_routed;
                const int nk = K / BK;
                if (!mbar_wait(smem_u32(&s.acce[ab]), aphase ^ 1u, p.timeout_ns)) { mx_fail(s, p, 42); break; }
                tc_fence_after();
                const uint32_t dtm = tmem_base + (uint32_t)(ab * MX_BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(smem_u32(&s.sf_full[stage]), phase, p.timeout_ns)) { mx_fail(s, p, 43); ok = false; break; }
                    tc_fence_after();
                    const uint32_t a0 = base + stage * STAGE_STRIDE, b0 = a0 + MX_A_BYTES;
                    if (KIND == KIND_W4) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_bf16(dtm, sdesc(a0 + j * 32), sdesc(b0 + j * 32), make_idesc_bf16(MX_BM, MX_BN),
                                     (kb | j) ? 1u : 0u);
                    } else {
                        const uint32_t sfa = tmem_base + MX_SF_COL0 + (uint32_t)stage * 8, sfb = sfa + 4;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_mx(dtm, sdesc(a0 + j * 32), sdesc(b0 + j * 32), mx_idesc(MX_BM, MX_BN, (uint32_t)j),
                                   sfa | ((uint32_t)j << 30), sfb | ((uint32_t)j << 30), (kb | j) ? 1u : 0u);
                    }
                    mma_commit(smem_u32(&s.empty[stage]));
                    if (++stage == MX_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit(smem_u32(&s.accf[ab]));
                if (++ab == 2) { ab = 0; aphase ^= 1u; }
            }
            // every MMA issued here has completed before the TMEM is freed
            mma_commit(smem_u32(&s.drain));
            if (!mbar_wait(smem_u32(&s.drain), 0, p.timeout_ns)) mx_fail(s, p, 47);
        }
    } else if (warp < 6) {
        // ================= scale words -> TMEM (warps 2-5, one per lane quadrant)
        const int q = warp & 3;
        int stage = 0;
        uint32_t phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            if (__shfl_sync(0xffffffffu, mx_aborted(s) ? 1 : 0, 0)) break;       // uniform over the warp
            const int K = tile >= s.tile_start[p.E] ? p.K_shared : p.K_routed;
            const int nk = K / BK;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                int okw = 1;
                if (lane == 0) okw = mbar_wait(smem_u32(&s.full[stage]), phase, p.timeout_ns) ? 1 : 0;
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) { if (lane == 0) mx_fail(s, p, 44); ok = false; break; }
                if (KIND == KIND_W4) {
                    // row n of the B tile: 64 nibbles -> bf16(q * s) into the 128-byte swizzled row
                    const int n = (warp - 2) * 32 + lane;
                    const uint32_t b_dst = base + stage * STAGE_STRIDE + MX_A_BYTES;
                    const uint32_t c_src = b_dst + MX_B_BYTES + (uint32_t)n * 32;
                    const uint32_t s_src = b_dst + MX_B_BYTES + W4_CODE_BYTES + (uint32_t)n * 16 +
                                           (uint32_t)(((kb >> 1) * 2) & 15);
                    uint32_t c[8];
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3]) : "r"(c_src));
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(c[4]), "=r"(c[5]), "=r"(c[6]), "=r"(c[7]) : "r"(c_src + 16));
                    unsigned short sb;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(sb) : "r"(s_src));
                    const uint32_t s2 = (uint32_t)sb * 0x10001u;   // the scale in both bf16 halves
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {            // 8 bf16 values per 16-byte chunk
                        // word = inputs 8ch .. 8ch+7, input i in bits 4i .. 4i+3
                        const uint32_t word = c[ch];
                        uint32_t o[4];
                        w4_decode8(word, s2, o);
                        const uint32_t a = b_dst + (uint32_t)n * 128 + ((uint32_t)(ch ^ (n & 7)) << 4);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     ::"r"(a), "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]) : "memory");
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&s.sf_full[stage]));
                    if (++stage == MX_STAGES) { stage = 0; phase ^= 1u; }
                    continue;
                }
                const uint32_t sa = base + stage * STAGE_STRIDE + MX_A_BYTES + MX_B_BYTES;
                const uint32_t sb = sa + MX_SA_BYTES;
                const uint32_t byte = (uint32_t)((kb * 4) & 15);
                uint32_t wa[4], wb[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t off = (uint32_t)(32 * c + lane) * 16u + byte;
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wa[c]) : "r"(sa + off));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wb[c]) : "r"(sb + off));
                }
                const uint32_t slot = tmem_base + ((uint32_t)(q * 32) << 16) + MX_SF_COL0 + (uint32_t)stage * 8;
                tmem_st4(slot, wa);
                tmem_st4(slot + 4, wb);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&s.sf_full[stage]));
                if (++stage == MX_STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ================= epilogue (warps 6-9, one per lane quadrant)
        const int q = warp & 3;
        const uint32_t stg = base + (uint32_t)kMxStgOff + (uint32_t)(warp - 6) * MX_STG_BYTES;
        int ab = 0;
        uint32_t aphase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            if (__shfl_sync(0xffffffffu, mx_aborted(s) ? 1 : 0, 0)) break;       // uniform over the warp
            int g, mt, nt;
            mx_decode(s, G, tile, g, mt, nt);
            const bool sh = g >= p.E;
            const int grow = mt * MX_BM + q * 32 + lane;
            const bool valid = grow < s.rows[g];
            const int nrows = __popc(__ballot_sync(0xffffffffu, valid));
            const int64_t orow = sh ? p.shared_out_row + s.row0[g] + grow : (int64_t)s.row0[g] + grow;
            const int64_t orow0 = orow - lane;
            float gscale = 1.f;
            if (MODE == MX_DOWN && !sh && valid && p.row_gate) gscale = __ldg(p.row_gate + orow);
            const int N = sh ? p.N_shared : p.N_routed;
            const float *bias = (!sh && p.bias) ? p.bias + (size_t)g * p.N_routed : nullptr;
            int ok = 1;
            if (lane == 0) ok = mbar_wait(smem_u32(&s.accf[ab]), aphase, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) { if (lane == 0) mx_fail(s, p, 45); break; }
            __syncwarp();
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t)(ab * MX_BN) + ((uint32_t)(q * 32) << 16);
            if (MODE == MX_SWIGLU) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float v[64];
                    tmem_ld32x2(taddr + cc * 32, taddr + 64 + cc * 32, v);   // gate, up
                    const int col0 = nt * OUT_COLS + cc * 32;
                    if (nrows == 0 || col0 >= N) continue;
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = mx_silu(v[i]) * v[32 + i];
                    mx_store32(stg, v, p.out + orow0 * p.ldo + col0, p.ldo, nrows);
                }
            } else {
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    float v[32];
                    tmem_ld32(taddr + cc * 32, v);
                    const int col0 = nt * OUT_COLS + cc * 32;
                    if (nrows == 0 || col0 >= N) continue;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float z = v[i] + (bias ? __ldg(bias + col0 + i) : 0.f);
                        v[i] = (MODE == MX_GELU) ? mx_gelu(z) : gscale * z;
                    }
                    mx_store32(stg, v, p.out + orow0 * p.ldo + col0, p.ldo, nrows);
                }
            }
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
        tmem_dealloc(tmem_base, MX_TMEM_COLS);
    }
    if (p.tail_mode) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------------ host side
// Code map: e4m3 [outer][mid][inner] (inner = K, 16-byte-aligned rows of ld
// bytes), box {128 codes, box_rows(, 1)}, 128-byte swizzle.
bool mx_code_map(CUtensorMap *m, int rank, const void *base, uint64_t inner, uint64_t mid, uint64_t outer, uint64_t ld,
                 uint32_t box_rows) {
    return make_map(m, rank, base, inner, mid, outer, ld, mid * ld, box_rows, 1);
}
// Byte map: bytes [outer][mid][inner] (rows of ld bytes), box {box_inner
// bytes, box_rows(, 1)}, no swizzle: MX scale rows (box 16), INT4 code rows
// (box 32) and INT4 bf16 scale rows (box 16).
bool byte_map(CUtensorMap *m, int rank, const void *base, uint64_t inner, uint64_t mid, uint64_t outer, uint64_t ld,
              uint32_t box_inner, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {inner, mid, outer};
    cuuint64_t strides[2] = {ld, mid * ld};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
// Scale map: bytes [outer][mid][inner] (inner = K / 32 scale bytes, rows of
// sld bytes), box {16 bytes, box_rows(, 1)}.
bool mx_scale_map(CUtensorMap *m, int rank, const void *base, uint64_t inner, uint64_t mid, uint64_t outer,
                  uint64_t sld, uint32_t box_rows) {
    return byte_map(m, rank, base, inner, mid, outer, sld, 16, box_rows);
}

struct MxMaps {
    CUtensorMap A, As, SA, SAs, B, B2, Bs, Bs2, SB, SB2, SBs, SBs2;
};

template <int MODE, int KIND = KIND_MX>
cudaError_t launch_mx_gemm(const MxMaps &m, const MxParams &p, int num_sms, cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc_mx_gemm<MODE, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kMxSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_kernel(tc_mx_gemm<MODE, KIND>, dim3(num_sms > 0 ? num_sms : 148), dim3(kMxThreads), kMxSmemBytes, st, true,
                         m.A, m.As, m.SA, m.SAs, m.B, m.B2, m.Bs, m.Bs2, m.SB, m.SB2, m.SBs, m.SBs2, p);
}

}  // namespace

cudaError_t launch_mx_gather_rows(const uint8_t *src, uint8_t *dst, int64_t ld, const int32_t *row_token,
                                  const int32_t *count, int64_t max_rows, int num_sms, cudaStream_t st) {
    if (max_rows <= 0) return cudaSuccess;
    if (ld % 16) return cudaErrorInvalidValue;
    const int sms = num_sms > 0 ? num_sms : 148;
    const int64_t want = (max_rows + 7) / 8;
    const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    return launch_kernel(mx_gather_rows_kernel, dim3(grid), dim3(256), 0, st, true, src, dst, ld, row_token, count,
                         max_rows);
}

cudaError_t launch_quant_mx(const QuantMxArgs &a, cudaStream_t st) {
    if (a.rows <= 0 || a.cols <= 0) return cudaSuccess;
    if (a.cols % 32 != 0) return cudaErrorInvalidValue;
    const int sms = a.num_sms > 0 ? a.num_sms : 148;
    const int64_t want = (a.rows + (kMxQuantThreads / 32) - 1) / (kMxQuantThreads / 32);
    const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    return launch_kernel(mx_quant_kernel, dim3(grid), dim3(kMxQuantThreads), 0, st, a.pdl, a);
}

// GEMM 1 (H = act(x W1^T [+ b1]) in bf16), H quantized to MX codes per row,
// GEMM 2 (y_perm = gate * (H W2^T [+ b2])), all on the stream in order.
cudaError_t launch_ffn_mx(const FfnMxArgs &a, cudaStream_t st) {
    if (a.routed_rows == 0 && (a.S == 0 || a.T == 0)) return cudaSuccess;
    if (a.E + 1 > kMxMaxGroups) return cudaErrorInvalidValue;
    const bool swiglu = a.act == MOE_ACT_SWIGLU;
    const bool has_sh = a.S > 0 && a.T > 0;
    const uint64_t routed_rows = (uint64_t)a.routed_rows;
    const uint64_t all_rows = routed_rows + (has_sh ? (uint64_t)a.T : 0);
    const int nsm = a.num_sms > 0 ? a.num_sms : 148;
    const uint64_t sld = (uint64_t)a.sld;
    const uint32_t bbox = swiglu ? 64 : 128;
    cudaError_t err;

    // ---- GEMM 1
    MxMaps m1;
    const uint64_t ar = routed_rows > 0 ? routed_rows : 1;
    if (!mx_code_map(&m1.A, 2, a.x_perm, a.d, ar, 1, a.d, 128) ||
        !mx_scale_map(&m1.SA, 2, a.xs_perm, a.d / 32, ar, 1, sld, 128) ||
        !mx_code_map(&m1.B, 3, a.W1, a.d, a.F, a.E, a.d, bbox) ||
        !mx_scale_map(&m1.SB, 3, a.W1s, a.d / 32, a.F, a.E, sld, bbox))
        return cudaErrorInvalidValue;
    if (swiglu) {
        if (!mx_code_map(&m1.B2, 3, a.Wu, a.d, a.F, a.E, a.d, bbox) ||
            !mx_scale_map(&m1.SB2, 3, a.Wus, a.d / 32, a.F, a.E, sld, bbox))
            return cudaErrorInvalidValue;
    } else {
        m1.B2 = m1.B; m1.SB2 = m1.SB;
    }
    if (has_sh) {
        if (!mx_code_map(&m1.As, 2, a.x, a.d, a.T, 1, a.d, 128) ||
            !mx_scale_map(&m1.SAs, 2, a.xs, a.d / 32, a.T, 1, sld, 128) ||
            !mx_code_map(&m1.Bs, 3, a.Wsg, a.d, a.S, 1, a.d, bbox) ||
            !mx_scale_map(&m1.SBs, 3, a.Wsgs, a.d / 32, a.S, 1, sld, bbox))
            return cudaErrorInvalidValue;
        if (swiglu) {
            if (!mx_code_map(&m1.Bs2, 3, a.Wsu, a.d, a.S, 1, a.d, bbox) ||
                !mx_scale_map(&m1.SBs2, 3, a.Wsus, a.d / 32, a.S, 1, sld, bbox))
                return cudaErrorInvalidValue;
        } else {
            m1.Bs2 = m1.Bs; m1.SBs2 = m1.SBs;
        }
    } else {
        m1.As = m1.A; m1.SAs = m1.SA; m1.Bs = m1.B; m1.Bs2 = m1.B2; m1.SBs = m1.SB; m1.SBs2 = m1.SB2;
    }
    MxParams p1{};
    p1.offsets = a.offsets;
    p1.bias = swiglu ? nullptr : a.b1;
    p1.out = a.H;
    p1.ldo = a.hF;
    p1.status = a.status;
    p1.timeout_ns = 2000000000ull;
    p1.E = a.E; p1.T = a.T; p1.has_shared = has_sh ? 1 : 0;
    p1.K_routed = a.d; p1.K_shared = a.d;
    p1.N_routed = a.F; p1.N_shared = a.S;
    p1.shared_a_row = 0;
    p1.shared_out_row = a.shared_base;
    err = swiglu ? launch_mx_gemm<MX_SWIGLU>(m1, p1, nsm, st) : launch_mx_gemm<MX_GELU>(m1, p1, nsm, st);
    if (err != cudaSuccess) return err;

    // ---- H -> MX codes (the kept routed rows, bounded on the device, then the shared rows)
    QuantMxArgs q{};
    q.in = a.H;
    q.ld_in = a.hF;
    q.out = a.H8;
    q.ld_out = a.hF;
    q.scale = a.Hs;
    q.ld_scale = a.sld;
    q.rows = (int64_t)routed_rows;
    q.row0 = 0;
    q.cols = a.F;
    q.rows_limit = a.offsets + a.E;
    q.num_sms = nsm;
    q.pdl = true;
    if ((err = launch_quant_mx(q, st)) != cudaSuccess) return err;
    if (has_sh) {
        q.rows = a.T;
        q.row0 = a.shared_base;
        q.cols = a.S;
        q.rows_limit = nullptr;
        if ((err = launch_quant_mx(q, st)) != cudaSuccess) return err;
    }

    // ---- GEMM 2
    MxMaps m2;
    const uint64_t hr = all_rows > 0 ? all_rows : 1;
    if (!mx_code_map(&m2.A, 2, a.H8, a.F, hr, 1, a.hF, 128) ||
        !mx_scale_map(&m2.SA, 2, a.Hs, a.F / 32, hr, 1, sld, 128) ||
        !mx_code_map(&m2.B, 3, a.W2, a.F, a.d, a.E, a.F, 128) ||
        !mx_scale_map(&m2.SB, 3, a.W2s, a.F / 32, a.d, a.E, sld, 128))
        return cudaErrorInvalidValue;
    m2.B2 = m2.B; m2.SB2 = m2.SB;
    if (has_sh) {
        if (!mx_code_map(&m2.As, 2, a.H8, a.S, hr, 1, a.hF, 128) ||
            !mx_scale_map(&m2.SAs, 2, a.Hs, a.S / 32, hr, 1, sld, 128) ||
            !mx_code_map(&m2.Bs, 3, a.Wsd, a.S, a.d, 1, a.S, 128) ||
            !mx_scale_map(&m2.SBs, 3, a.Wsds, a.S / 32, a.d, 1, sld, 128))
            return cudaErrorInvalidValue;
    } else {
        m2.As = m2.A; m2.SAs = m2.SA; m2.Bs = m2.B; m2.SBs = m2.SB;
    }
    m2.Bs2 = m2.Bs; m2.SBs2 = m2.SBs;
    MxParams p2{};
    p2.offsets = a.offsets;
    p2.bias = swiglu ? nullptr : a.b2;
    p2.row_gate = a.row_gate;
    p2.out = a.y_perm;
    p2.ldo = a.d;
    p2.status = a.status;
    p2.timeout_ns = 2000000000ull;
    p2.E = a.E; p2.T = a.T; p2.has_shared = has_sh ? 1 : 0;
    p2.K_routed = a.F; p2.K_shared = a.S;
    p2.N_routed = a.d; p2.N_shared = a.d;
    p2.shared_a_row = a.shared_base;
    p2.shared_out_row = a.shared_base;
    return launch_mx_gemm<MX_DOWN>(m2, p2, nsm, st);
}

// INT4 weight-only experts: GEMM 1 (H = act(x W1^T [+ b1]) in bf16 from bf16
// rows and INT4 weights), GEMM 2 (y_perm = gate * (H W2^T [+ b2])).  The
// FfnMxArgs fields carry: x_perm / x bf16 rows, W* packed codes [.., N, K/2],
// W*s bf16 scale bytes [.., N, sld] (one scale per 128 inputs); xs_perm, xs,
// H8 and Hs are unused.
cudaError_t launch_ffn_w4(const FfnMxArgs &a, cudaStream_t st) {
    if (a.routed_rows == 0 && (a.S == 0 || a.T == 0)) return cudaSuccess;
    if (a.E + 1 > kMxMaxGroups) return cudaErrorInvalidValue;
    const bool swiglu = a.act == MOE_ACT_SWIGLU;
    const bool has_sh = a.S > 0 && a.T > 0;
    const uint64_t routed_rows = (uint64_t)a.routed_rows;
    const uint64_t all_rows = routed_rows + (has_sh ? (uint64_t)a.T : 0);
    const int nsm = a.num_sms > 0 ? a.num_sms : 148;
    const uint64_t sld = (uint64_t)a.sld;
    const uint32_t bbox = swiglu ? 64 : 128;
    cudaError_t err;

    // ---- GEMM 1
    MxMaps m1;
    const uint64_t ar = routed_rows > 0 ? routed_rows : 1;
    if (!make_map(&m1.A, 2, a.x_perm, a.d, ar, 1, a.d, 0, 128, 2) ||
        !byte_map(&m1.B, 3, a.W1, a.d / 2, a.F, a.E, a.d / 2, 32, bbox) ||
        !byte_map(&m1.SB, 3, a.W1s, a.d / 64, a.F, a.E, sld, 16, bbox))
        return cudaErrorInvalidValue;
    m1.SA = m1.SB; m1.SAs = m1.SB;                      // no activation scales
    if (swiglu) {
        if (!byte_map(&m1.B2, 3, a.Wu, a.d / 2, a.F, a.E, a.d / 2, 32, bbox) ||
            !byte_map(&m1.SB2, 3, a.Wus, a.d / 64, a.F, a.E, sld, 16, bbox))
            return cudaErrorInvalidValue;
    } else {
        m1.B2 = m1.B; m1.SB2 = m1.SB;
    }
    if (has_sh) {
        if (!make_map(&m1.As, 2, a.x, a.d, a.T, 1, a.d, 0, 128, 2) ||
            !byte_map(&m1.Bs, 3, a.Wsg, a.d / 2, a.S, 1, a.d / 2, 32, bbox) ||
            !byte_map(&m1.SBs, 3, a.Wsgs, a.d / 64, a.S, 1, sld, 16, bbox))
            return cudaErrorInvalidValue;
        if (swiglu) {
            if (!byte_map(&m1.Bs2, 3, a.Wsu, a.d / 2, a.S, 1, a.d / 2, 32, bbox) ||
                !byte_map(&m1.SBs2, 3, a.Wsus, a.d / 64, a.S, 1, sld, 16, bbox))
                return cudaErrorInvalidValue;
        } else {
            m1.Bs2 = m1.Bs; m1.SBs2 = m1.SBs;
        }
    } else {
        m1.As = m1.A; m1.Bs = m1.B; m1.Bs2 = m1.B2; m1.SBs = m1.SB; m1.SBs2 = m1.SB2;
    }
    MxParams p1{};
    p1.offsets = a.offsets;
    p1.bias = swiglu ? nullptr : a.b1;
    p1.out = a.H;
    p1.ldo = a.hF;
    p1.status = a.status;
    p1.timeout_ns = 2000000000ull;
    p1.E = a.E; p1.T = a.T; p1.has_shared = has_sh ? 1 : 0;
    p1.K_routed = a.d; p1.K_shared = a.d;
    p1.N_routed = a.F; p1.N_shared = a.S;
    p1.shared_a_row = 0;
    p1.shared_out_row = a.shared_base;
    // CTA pairs over the 256-row blocks (and a last block of > 128 rows) ...
    W4PairArgs w1{};
    w1.A = m1.A; w1.As = m1.As;
    w1.c = a.W1; w1.sc = a.W1s;
    w1.c2 = swiglu ? a.Wu : a.W1; w1.sc2 = swiglu ? a.Wus : a.W1s;
    w1.cs = has_sh ? a.Wsg : a.W1; w1.scs = has_sh ? a.Wsgs : a.W1s;
    w1.cs2 = has_sh && swiglu ? a.Wsu : w1.cs; w1.scs2 = has_sh && swiglu ? a.Wsus : w1.scs;
    w1.sld = (int64_t)sld;
    w1.offsets = a.offsets;
    w1.bias = p1.bias;
    w1.row_gate = nullptr;
    w1.out = a.H;
    w1.out_cols = (uint64_t)a.hF;
    w1.out_rows = all_rows;
    w1.status = a.status;
    w1.mode = swiglu ? 0 : 1;
    w1.E = a.E; w1.T = a.T; w1.has_shared = p1.has_shared;
    w1.K_routed = a.d; w1.K_shared = a.d;
    w1.N_routed = a.F; w1.N_shared = a.S;
    w1.ldo = a.hF;
    w1.shared_a_row = 0;
    w1.shared_out_row = a.shared_base;
    w1.num_sms = nsm;
    w1.pdl = true;
    if ((err = launch_w4_gemm_pair(w1, st)) != cudaSuccess) return err;
    // ... then one CTA per SM over the last blocks of 1..128 rows
    p1.tail_mode = 1;
    err = swiglu ? launch_mx_gemm<MX_SWIGLU, KIND_W4>(m1, p1, nsm, st)
                 : launch_mx_gemm<MX_GELU, KIND_W4>(m1, p1, nsm, st);
    if (err != cudaSuccess) return err;

    // ---- GEMM 2 (A: H in bf16)
    MxMaps m2;
    const uint64_t hr = all_rows > 0 ? all_rows : 1;
    if (!make_map(&m2.A, 2, a.H, a.F, hr, 1, a.hF, 0, 128, 2) ||
        !byte_map(&m2.B, 3, a.W2, a.F / 2, a.d, a.E, a.F / 2, 32, 128) ||
        !byte_map(&m2.SB, 3, a.W2s, a.F / 64, a.d, a.E, sld, 16, 128))
        return cudaErrorInvalidValue;
    m2.SA = m2.SB; m2.SAs = m2.SB; m2.B2 = m2.B; m2.SB2 = m2.SB;
    if (has_sh) {
        if (!make_map(&m2.As, 2, a.H, a.S, hr, 1, a.hF, 0, 128, 2) ||
            !byte_map(&m2.Bs, 3, a.Wsd, a.S / 2, a.d, 1, a.S / 2, 32, 128) ||
            !byte_map(&m2.SBs, 3, a.Wsds, a.S / 64, a.d, 1, sld, 16, 128))
            return cudaErrorInvalidValue;
    } else {
        m2.As = m2.A; m2.Bs = m2.B; m2.SBs = m2.SB;
    }
    m2.Bs2 = m2.Bs; m2.SBs2 = m2.SBs;
    MxParams p2{};
    p2.offsets = a.offsets;
    p2.bias = swiglu ? nullptr : a.b2;
    p2.row_gate = a.row_gate;
    p2.out = a.y_perm;
    p2.ldo = a.d;
    p2.status = a.status;
    p2.timeout_ns = 2000000000ull;
    p2.E = a.E; p2.T = a.T; p2.has_shared = has_sh ? 1 : 0;
    p2.K_routed = a.F; p2.K_shared = a.S;
    p2.N_routed = a.d; p2.N_shared = a.d;
    p2.shared_a_row = a.shared_base;
    p2.shared_out_row = a.shared_base;
    W4PairArgs w2{};
    w2.A = m2.A; w2.As = m2.As;
    w2.c = a.W2; w2.sc = a.W2s;
    w2.cs = has_sh ? a.Wsd : a.W2; w2.scs = has_sh ? a.Wsds : a.W2s;
    w2.c2 = w2.c; w2.sc2 = w2.sc; w2.cs2 = w2.cs; w2.scs2 = w2.scs;
    w2.sld = (int64_t)sld;
    w2.offsets = a.offsets;
    w2.bias = p2.bias;
    w2.row_gate = a.row_gate;
    w2.out = a.y_perm;
    w2.out_cols = (uint64_t)a.d;
    w2.out_rows = all_rows;
    w2.status = a.status;
    w2.mode = 2;
    w2.E = a.E; w2.T = a.T; w2.has_shared = p2.has_shared;
    w2.K_routed = a.F; w2.K_shared = a.S;
    w2.N_routed = a.d; w2.N_shared = a.d;
    w2.ldo = a.d;
    w2.shared_a_row = a.shared_base;
    w2.shared_out_row = a.shared_base;
    w2.num_sms = nsm;
    w2.pdl = true;
    if ((err = launch_w4_gemm_pair(w2, st)) != cudaSuccess) return err;
    p2.tail_mode = 1;
    return launch_mx_gemm<MX_DOWN, KIND_W4>(m2, p2, nsm, st);
}

}  // namespace moe
