// permute_noalloc.cu -- moe_permute for callers that cannot allocate device
// memory.
//
// moe_permute needs a little scratch (per-chunk expert counts and their
// prefix sums) and takes it from the caller's workspace.  Some callers have
// no way to provide one: a plug-in running inside a host framework that owns
// the whole device-memory budget and forbids its libraries from calling
// cudaMalloc, or a latency-critical caller that cannot afford cudaMalloc's
// implicit device-wide synchronisation and has no pool to draw from.  For
// them this file keeps that scratch in a fixed array in the library's own
// device memory (a file-scope __device__ array, loaded with the module: every
// GPU that loads libmoe holds these bytes until the process exits) and runs
// the same three kernels as moe_permute on it.
//
// Limits and behaviour:
//   - E * ceil(T / 64) <= MOE_PERMUTE_NOALLOC_MAX_CELLS (262,144, i.e. E = 256
//     with T <= 65,536), 2 MiB + 256 bytes of static device memory; larger
//     problems are rejected with MOE_ERR_UNSUPPORTED before any launch.
//   - The first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current and caches it; make that
//     first call before any stream capture.  The cached address belongs to the
//     device's current context: after cudaDeviceReset on that device the
//     library must be reloaded (the module, and so the array, may then sit at
//     another address).
//   - All calls share the one array: calls that overlap on the GPU (two
//     streams, or two host threads) race on it.  Each call rewrites every
//     count it reads, and clears the status header it owns first.
//   - There is no workspace, so a device-detected bad expert id cannot be read
//     back: such an assignment is dropped (row -1) exactly as in moe_permute,
//     but not reported.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

#define MOE_PERMUTE_NOALLOC_MAX_CELLS (256 * 1024)

namespace {

constexpr size_t kHeader = 256;
constexpr size_t kCells = MOE_PERMUTE_NOALLOC_MAX_CELLS;
constexpr size_t kScratchBytes = kHeader + 2 * kCells * sizeof(int32_t);

// status header | per-chunk counts [E][nchunks] | per-chunk bases [E][nchunks]
static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {nullptr};

moe_status reject(moe_status s, const char *why) {
    moe::set_error_detail("moe_permute_noalloc", why);
    return s;
}

// Device address of the static scratch on the current device (looked up once
// per device, with that device current).
moe_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return reject(MOE_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices) return reject(MOE_ERR_UNSUPPORTED, "device index above 63");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_permute_scratch);
        if (e != cudaSuccess || ptr == nullptr) return reject(MOE_ERR_CUDA, cudaGetErrorString(e));
        g_scratch_addr[dev] = ptr;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_config *cfg, const void *x, const int32_t *idx,
                                          const float *gate, int32_t *counts, int32_t *kept, int32_t *offsets,
                                          int32_t *row_of, int32_t *row_token, float *row_gate, void *x_perm,
                                          int32_t *n_dropped, moe_stream_t stream) {
    // Argument checks mirror moe_permute's (messages via moe_last_error_detail).
    moe_status s = moe::validate_config(cfg);
    if (s != MOE_OK) return s;
    if (!counts || !kept || !offsets) return reject(MOE_ERR_INVALID_ARG, "NULL counts, kept or offsets");
    // x_perm may be NULL (row tables only), as in moe_permute
    if (cfg->T > 0 && (!x || !idx || !gate || !row_of || !row_token || !row_gate))
        return reject(MOE_ERR_INVALID_ARG, "NULL input or output array");
    auto mis = [](const void *p, uintptr_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(x, 16) || mis(x_perm, 16) || mis(idx, 4) || mis(gate, 4) || mis(counts, 4) || mis(kept, 4) ||
        mis(offsets, 4) || mis(row_of, 4) || mis(row_token, 4) || mis(row_gate, 4) || mis(n_dropped, 4))
        return reject(MOE_ERR_INVALID_ARG, "misaligned pointer");
    const int nchunks = moe::dispatch_chunks(cfg->T);
    if ((size_t)cfg->E * (size_t)nchunks > kCells)
        return reject(MOE_ERR_UNSUPPORTED, "E * ceil(T/64) exceeds the 262144-cell static scratch");

    void *base = nullptr;
    s = scratch_address(&base);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(base, 0, kHeader, st);
    if (e != cudaSuccess) return reject(MOE_ERR_CUDA, cudaGetErrorString(e));

    char *b = static_cast<char *>(base);
    const size_t plane = (size_t)cfg->E * (size_t)nchunks * sizeof(int32_t);
    moe::DispatchArgs a{};
    a.x = x; a.idx = idx; a.gate = gate;
    a.chunk_cnt = reinterpret_cast<int32_t *>(b + kHeader);
    a.chunk_base = reinterpret_cast<int32_t *>(b + kHeader + plane);
    a.counts = counts; a.kept = kept; a.offsets = offsets;
    a.row_of = row_of; a.row_token = row_token; a.row_gate = row_gate; a.x_perm = x_perm;
    a.n_dropped = n_dropped;
    a.status = reinterpret_cast<int32_t *>(b);
    a.T = cfg->T; a.d = cfg->d_model; a.E = cfg->E; a.k = cfg->top_k;
    a.capacity = moe_capacity(cfg);
    e = moe::launch_dispatch(a, cfg->dtype == MOE_BF16 ? 2 : 4, st);
    if (e != cudaSuccess) return reject(MOE_ERR_CUDA, cudaGetErrorString(e));
    return MOE_OK;
}
