// moe_api.cu -- the extern "C" boundary of libmoe: argument checks, workspace
// layout and the launch sequence.  See include/moe.h for the contract.
#include <math.h>

#include <algorithm>
#include <mutex>
#include <vector>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "kernels.cuh"

namespace {

// One CTA waits on a barrier nothing arrives on; the bounded wait gives up
// after limit_ns and the timeout lands in the status word.
__global__ void wait_timeout_kernel(int32_t *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    moe::mbar_init(moe::smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!moe::mbar_wait(moe::smem_u32(&bar), 0, limit_ns)) moe::record_error(status, MOE_ERR_TIMEOUT, 77);
}

thread_local char g_detail[256] = "";

moe_status fail(moe_status s, const char *fmt, const char *what = "") {
    snprintf(g_detail, sizeof g_detail, fmt, what);
    return s;
}

moe_status cuda_fail(cudaError_t e, const char *where) {
    snprintf(g_detail, sizeof g_detail, "%s: %s", where, cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Layout {
    size_t router_w, logits, psum, chunk_cnt, chunk_base, kept, contrib, offsets, row_of, row_token, row_gate, x_perm, H, y_perm;
    // e4m3 experts (bf16 layers): codes and row scales of x, the packed rows'
    // scales (the codes themselves go to x_perm), codes and scales of H
    size_t x8, x8_scale, xperm_scale, H8, h_scale;
    size_t total;
};

int64_t perm_rows(const moe_config *c) {
    return (int64_t)c->T * c->top_k + (c->d_ff_shared > 0 ? (int64_t)c->T : 0);
}

Layout layout(const moe_config *c) {
    Layout L{};
    const size_t esz = c->dtype == MOE_BF16 ? 2 : 4;
    const size_t Tk = (size_t)c->T * c->top_k;
    const size_t rows = (size_t)perm_rows(c);
    const size_t hF = (size_t)(c->d_ff > c->d_ff_shared ? c->d_ff : c->d_ff_shared);
    const bool bf16 = c->dtype == MOE_BF16;
    const size_t nblk = (size_t)moe::router_blocks(c->T, bf16);
    const size_t nch = (size_t)moe::dispatch_chunks(c->T);
    size_t o = sizeof(moe::WsHeader);
    L.router_w = o;   o = align256(o + (bf16 ? moe::router_split_bytes(c->d_model, c->E) : 0));
    L.logits = o;     o = align256(o + (bf16 ? (size_t)moe::router_logit_splits_max(c->T) * c->T * c->E * 4 : 0));
    L.psum = o;       o = align256(o + nblk * c->E * 4);
    L.chunk_cnt = o;  o = align256(o + nch * c->E * 4);
    L.chunk_base = o; o = align256(o + nch * c->E * 4);
    L.kept = o;       o = align256(o + (size_t)c->E * 4);
    L.contrib = o;    o = align256(o + (size_t)c->E * 8);
    L.offsets = o;    o = align256(o + (size_t)(c->E + 1) * 4);
    L.row_of = o;     o = align256(o + Tk * 4);
    L.row_token = o;  o = align256(o + Tk * 4);
    L.row_gate = o;   o = align256(o + Tk * 4);
    L.x_perm = o;     o = align256(o + Tk * c->d_model * esz);
    L.H = o;          o = align256(o + rows * hF * esz);
    L.y_perm = o;     o = align256(o + rows * c->d_model * esz);
    const size_t f8 = bf16 ? 1 : 0;
    L.x8 = o;         o = align256(o + f8 * (size_t)c->T * c->d_model);
    L.x8_scale = o;   o = align256(o + f8 * (size_t)c->T * 4);
    L.xperm_scale = o; o = align256(o + f8 * Tk * 4);
    L.H8 = o;         o = align256(o + f8 * rows * hF);
    L.h_scale = o;    o = align256(o + f8 * rows * 4);
    L.total = o;
    return L;
}

moe_status check_cfg(const moe_config *c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL%s");
    if (c->T < 0) return fail(MOE_ERR_INVALID_ARG, "T < 0%s");
    if (c->E < 1) return fail(MOE_ERR_INVALID_ARG, "E < 1%s");
    if (c->E > 256) return fail(MOE_ERR_UNSUPPORTED, "E > 256%s");
    if (c->top_k < 1 || c->top_k > c->E) return fail(MOE_ERR_INVALID_ARG, "top_k outside 1..E%s");
    if (c->top_k > 32) return fail(MOE_ERR_UNSUPPORTED, "top_k > 32%s");
    if (c->d_model < 1 || c->d_ff < 1 || c->d_ff_shared < 0) return fail(MOE_ERR_INVALID_ARG, "non-positive width%s");
    if (c->d_model % 8 || c->d_ff % 8 || c->d_ff_shared % 8)
        return fail(MOE_ERR_UNSUPPORTED, "d_model, d_ff and d_ff_shared must be multiples of 8%s");
    if (c->d_model > 65536 || c->d_ff > 65536 || c->d_ff_shared > 65536)
        return fail(MOE_ERR_UNSUPPORTED, "widths above 65536%s");
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "bad dtype%s");
    if (c->act != MOE_ACT_GELU_BIAS && c->act != MOE_ACT_SWIGLU) return fail(MOE_ERR_INVALID_ARG, "bad act%s");
    if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID) return fail(MOE_ERR_INVALID_ARG, "bad score%s");
    if (c->renorm != 0 && c->renorm != 1) return fail(MOE_ERR_INVALID_ARG, "renorm must be 0 or 1%s");
    if (!isfinite(c->capacity_factor)) return fail(MOE_ERR_INVALID_ARG, "capacity_factor not finite%s");
    if (perm_rows(c) >= ((int64_t)1 << 31) - 256) return fail(MOE_ERR_UNSUPPORTED, "T * (top_k + 1) too large%s");
    return MOE_OK;
}

moe_status check_ws(const moe_config *c, void *ws, size_t ws_bytes) {
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL%s");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned%s");
    if (ws_bytes < layout(c).total) return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_workspace_size()%s");
    return MOE_OK;
}

#define NEED(p) \
    do { if (!(p)) return fail(MOE_ERR_INVALID_ARG, "NULL pointer: %s", #p); } while (0)
// 16-byte vector loads / TMA need 16-byte aligned rows; 4-byte arrays need 4.
#define ALIGNED(p, a) \
    do { if ((p) && (reinterpret_cast<uintptr_t>(p) % (a))) \
        return fail(MOE_ERR_INVALID_ARG, "misaligned pointer: %s", #p); } while (0)

// e4m3 experts: bf16 layers only; every e4m3 row (x, weights, H) must be a
// multiple of 16 bytes for the tensor maps.
moe_status check_fp8_cfg(const moe_config *c) {
    if (c->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "FP8 experts need a bf16 layer%s");
    if (c->d_model % 16 || c->d_ff % 16 || c->d_ff_shared % 16)
        return fail(MOE_ERR_UNSUPPORTED, "FP8 experts need d_model, d_ff, d_ff_shared multiples of 16%s");
    return MOE_OK;
}

// MX experts: bf16 layers, K dimensions in whole 128-value stages, at most
// 256 routed groups, scale rows of sld bytes (a multiple of 16 that holds
// d_model / 32, d_ff / 32 and d_ff_shared / 32 bytes).
moe_status check_mx_cfg(const moe_config *c, int32_t sld) {
    if (c->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "MX experts need a bf16 layer%s");
    if (c->d_model % 128 || c->d_ff % 128 || c->d_ff_shared % 128)
        return fail(MOE_ERR_UNSUPPORTED, "MX experts need d_model, d_ff, d_ff_shared multiples of 128%s");
    if (c->E > 256) return fail(MOE_ERR_UNSUPPORTED, "MX experts: at most 256 experts%s");
    const int need = std::max(c->d_model, std::max(c->d_ff, c->d_ff_shared)) / 32;
    if (sld < need || sld % 16) return fail(MOE_ERR_INVALID_ARG, "sld below the widest K / 32 or not a multiple of 16%s");
    return MOE_OK;
}

// MX workspace: H in bf16, its codes and scale rows (the grouped FFN), then
// x's codes and scale rows and the packed rows' scale rows (moe_forward_mx).
// INT4 experts: bf16 layers, K dimensions in whole 128-input groups, at most
// 256 routed groups, bf16 scale rows of sld bytes (a multiple of 16 that holds
// 2 * K / 128 bytes for every K).
moe_status check_w4_cfg(const moe_config *c, int32_t sld) {
    if (c->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "INT4 experts need a bf16 layer%s");
    if (c->d_model % 128 || c->d_ff % 128 || c->d_ff_shared % 128)
        return fail(MOE_ERR_UNSUPPORTED, "INT4 experts need d_model, d_ff, d_ff_shared multiples of 128%s");
    if (c->E > 256) return fail(MOE_ERR_UNSUPPORTED, "INT4 experts: at most 256 experts%s");
    const int need = std::max(c->d_model, std::max(c->d_ff, c->d_ff_shared)) / 64;
    if (sld < need || sld % 16) return fail(MOE_ERR_INVALID_ARG, "sld below 2 * K / 128 or not a multiple of 16%s");
    return MOE_OK;
}

moe_status check_w4_weights(const moe_config *c, const moe_w4_experts *w) {
    NEED(w->W1); NEED(w->W1_scale); NEED(w->W2); NEED(w->W2_scale);
    if (c->act == MOE_ACT_SWIGLU) { NEED(w->Wu); NEED(w->Wu_scale); }
    if (c->d_ff_shared > 0) {
        NEED(w->Wsh_g); NEED(w->Wsh_g_scale); NEED(w->Wsh_d); NEED(w->Wsh_d_scale);
        if (c->act == MOE_ACT_SWIGLU) { NEED(w->Wsh_u); NEED(w->Wsh_u_scale); }
    }
    ALIGNED(w->W1, 16); ALIGNED(w->Wu, 16); ALIGNED(w->W2, 16); ALIGNED(w->Wsh_g, 16); ALIGNED(w->Wsh_u, 16);
    ALIGNED(w->Wsh_d, 16); ALIGNED(w->W1_scale, 16); ALIGNED(w->Wu_scale, 16); ALIGNED(w->W2_scale, 16);
    ALIGNED(w->Wsh_g_scale, 16); ALIGNED(w->Wsh_u_scale, 16); ALIGNED(w->Wsh_d_scale, 16);
    return MOE_OK;
}

struct MxLayout {
    size_t H, H8, Hs, x8, xs, xs_perm, total;
    int hF;
};
MxLayout mx_layout(const moe_config *c, int32_t sld) {
    MxLayout L{};
    const size_t Tk = (size_t)c->T * c->top_k;
    const size_t rows = Tk + (c->d_ff_shared > 0 ? (size_t)c->T : 0);
    L.hF = std::max(c->d_ff, c->d_ff_shared);
    size_t o = sizeof(moe::WsHeader);
    L.H = o;        o = align256(o + rows * L.hF * 2);
    L.H8 = o;       o = align256(o + rows * L.hF);
    L.Hs = o;       o = align256(o + rows * (size_t)sld);
    L.x8 = o;       o = align256(o + (size_t)c->T * c->d_model);
    L.xs = o;       o = align256(o + (size_t)c->T * (size_t)sld);
    L.xs_perm = o;  o = align256(o + Tk * (size_t)sld);
    L.total = o;
    return L;
}

// Frozen routers (moe_router_freeze): the workspace whose router scratch
// holds the split of a given W_r (pointer, d_model, E).  Router launches on
// that workspace with the same W_r skip the split; a launch with other
// weights re-splits and drops the entry; moe_workspace_init drops it too.
struct FrozenRouter {
    const void *ws;
    const float *Wr;
    int d, E;
};
std::mutex g_frozen_mu;
std::vector<FrozenRouter> g_frozen;

bool router_split_ready(const void *ws, const float *Wr, int d, int E) {
    std::lock_guard<std::mutex> lock(g_frozen_mu);
    for (size_t i = 0; i < g_frozen.size(); ++i) {
        if (g_frozen[i].ws != ws) continue;
        if (g_frozen[i].Wr == Wr && g_frozen[i].d == d && g_frozen[i].E == E) return true;
        g_frozen.erase(g_frozen.begin() + (long)i);     // this launch overwrites the split
        return false;
    }
    return false;
}
void set_frozen(const void *ws, const float *Wr, int d, int E) {
    std::lock_guard<std::mutex> lock(g_frozen_mu);
    for (auto &f : g_frozen)
        if (f.ws == ws) { f.Wr = Wr; f.d = d; f.E = E; return; }
    g_frozen.push_back(FrozenRouter{ws, Wr, d, E});
}
void forget_frozen(const void *ws) {
    std::lock_guard<std::mutex> lock(g_frozen_mu);
    for (size_t i = 0; i < g_frozen.size(); ++i)
        if (g_frozen[i].ws == ws) { g_frozen.erase(g_frozen.begin() + (long)i); return; }
}

moe_status check_fp8_weights(const moe_config *c, const moe_fp8_experts *w) {
    NEED(w);
    NEED(w->W1); NEED(w->W1_scale); NEED(w->W2); NEED(w->W2_scale);
    ALIGNED(w->W1, 16); ALIGNED(w->Wu, 16); ALIGNED(w->W2, 16);
    ALIGNED(w->Wsh_g, 16); ALIGNED(w->Wsh_u, 16); ALIGNED(w->Wsh_d, 16);
    ALIGNED(w->W1_scale, 4); ALIGNED(w->Wu_scale, 4); ALIGNED(w->W2_scale, 4);
    ALIGNED(w->Wsh_g_scale, 4); ALIGNED(w->Wsh_u_scale, 4); ALIGNED(w->Wsh_d_scale, 4);
    if (c->act == MOE_ACT_SWIGLU) { NEED(w->Wu); NEED(w->Wu_scale); }
    if (c->d_ff_shared > 0) {
        NEED(w->Wsh_g); NEED(w->Wsh_g_scale); NEED(w->Wsh_d); NEED(w->Wsh_d_scale);
        if (c->act == MOE_ACT_SWIGLU) { NEED(w->Wsh_u); NEED(w->Wsh_u_scale); }
    }
    return MOE_OK;
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

template <typename T>
T *at(void *ws, size_t off) { return reinterpret_cast<T *>(static_cast<char *>(ws) + off); }

int32_t *status_word(void *ws) { return reinterpret_cast<int32_t *>(ws); }

moe_status check_weights(const moe_config *c, const void *W1, const void *Wu, const void *W2,
                         const void *x, const void *Wsg, const void *Wsu, const void *Wsd) {
    NEED(W1); NEED(W2);
    ALIGNED(W1, 16); ALIGNED(Wu, 16); ALIGNED(W2, 16); ALIGNED(x, 16);
    ALIGNED(Wsg, 16); ALIGNED(Wsu, 16); ALIGNED(Wsd, 16);
    if (c->act == MOE_ACT_SWIGLU) NEED(Wu);
    if (c->d_ff_shared > 0) {
        NEED(x); NEED(Wsg); NEED(Wsd);
        if (c->act == MOE_ACT_SWIGLU) NEED(Wsu);
    }
    return MOE_OK;
}

moe::FfnArgs ffn_args(const moe_config *c, const void *x_perm, const int32_t *offsets, const float *row_gate,
                      const void *W1, const float *b1, const void *Wu, const void *W2, const float *b2,
                      const void *x, const void *Wsg, const void *Wsu, const void *Wsd, void *y_perm, void *ws) {
    const Layout L = layout(c);
    moe::FfnArgs a{};
    a.x_perm = x_perm; a.x = x; a.offsets = offsets; a.row_gate = row_gate;
    a.W1 = W1; a.Wu = Wu; a.W2 = W2; a.b1 = b1; a.b2 = b2;
    a.Wsg = Wsg; a.Wsu = Wsu; a.Wsd = Wsd;
    a.H = at<char>(ws, L.H);
    a.y_perm = y_perm;
    a.status = status_word(ws);
    a.T = c->T; a.d = c->d_model; a.E = c->E; a.k = c->top_k; a.F = c->d_ff; a.S = c->d_ff_shared;
    a.n_groups = c->E;
    a.routed_rows = (int64_t)c->T * c->top_k;
    a.act = c->act;
    a.hF = c->d_ff > c->d_ff_shared ? c->d_ff : c->d_ff_shared;
    a.shared_base = (int64_t)c->T * c->top_k;
    a.num_sms = num_sms();
    return a;
}

// The e4m3 fields of the FFN arguments (x_perm / x hold codes).
void set_fp8(moe::FfnArgs &a, const moe_config *c, const moe_fp8_experts *w, const float *xperm_scale,
             const float *x_scale, void *ws) {
    const Layout L = layout(c);
    a.f8 = true;
    a.xperm_scale = xperm_scale;
    a.x_scale = x_scale;
    a.W1s = w->W1_scale; a.Wus = w->Wu_scale; a.W2s = w->W2_scale;
    a.Wsgs = w->Wsh_g_scale; a.Wsus = w->Wsh_u_scale; a.Wsds = w->Wsh_d_scale;
    a.H8 = at<uint8_t>(ws, L.H8);
    a.h_scale = at<float>(ws, L.h_scale);
}

// ---- expert parallelism: the grouped FFN over rows gathered from n_src sources
moe_status check_ep_cfg(const moe_config *c, int32_t n_src, int64_t max_rows) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL%s");
    if (c->E < 1) return fail(MOE_ERR_INVALID_ARG, "E (local experts) < 1%s");
    if (n_src < 1) return fail(MOE_ERR_INVALID_ARG, "n_src < 1%s");
    if ((int64_t)n_src * c->E > 256) return fail(MOE_ERR_UNSUPPORTED, "n_src * E (row groups) > 256%s");
    if (c->d_model < 1 || c->d_ff < 1) return fail(MOE_ERR_INVALID_ARG, "non-positive width%s");
    if (c->d_model % 8 || c->d_ff % 8) return fail(MOE_ERR_UNSUPPORTED, "d_model and d_ff must be multiples of 8%s");
    if (c->d_model > 65536 || c->d_ff > 65536) return fail(MOE_ERR_UNSUPPORTED, "widths above 65536%s");
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "bad dtype%s");
    if (c->act != MOE_ACT_GELU_BIAS && c->act != MOE_ACT_SWIGLU) return fail(MOE_ERR_INVALID_ARG, "bad act%s");
    if (max_rows < 0) return fail(MOE_ERR_INVALID_ARG, "max_rows < 0%s");
    if (max_rows >= ((int64_t)1 << 31) - 256) return fail(MOE_ERR_UNSUPPORTED, "max_rows too large%s");
    return MOE_OK;
}
size_t ep_h_offset() { return sizeof(moe::WsHeader); }
size_t ep_ws_bytes(const moe_config *c, int64_t max_rows) {
    const size_t esz = c->dtype == MOE_BF16 ? 2 : 4;
    return align256(ep_h_offset() + (size_t)max_rows * c->d_ff * esz);
}
moe::FfnMxArgs w4_args(const moe_config *cfg, const void *x_perm, const int32_t *offsets, const float *row_gate,
                       const moe_w4_experts *w, const float *b1, const float *b2, const void *x, void *y_perm,
                       void *ws) {
    const Layout L = layout(cfg);
    moe::FfnMxArgs a{};
    a.x_perm = static_cast<const uint8_t *>(x_perm); a.x = static_cast<const uint8_t *>(x);
    a.offsets = offsets; a.row_gate = row_gate;
    a.W1 = w->W1; a.W1s = w->W1_scale; a.Wu = w->Wu; a.Wus = w->Wu_scale; a.W2 = w->W2; a.W2s = w->W2_scale;
    a.b1 = b1; a.b2 = b2;
    a.Wsg = w->Wsh_g; a.Wsgs = w->Wsh_g_scale; a.Wsu = w->Wsh_u; a.Wsus = w->Wsh_u_scale;
    a.Wsd = w->Wsh_d; a.Wsds = w->Wsh_d_scale;
    a.H = at<__nv_bfloat16>(ws, L.H);
    a.y_perm = static_cast<__nv_bfloat16 *>(y_perm);
    a.status = status_word(ws);
    a.T = cfg->T; a.d = cfg->d_model; a.E = cfg->E; a.F = cfg->d_ff; a.S = cfg->d_ff_shared; a.act = cfg->act;
    a.routed_rows = (int64_t)cfg->T * cfg->top_k;
    a.hF = std::max(cfg->d_ff, cfg->d_ff_shared);
    a.shared_base = (int64_t)cfg->T * cfg->top_k;
    a.sld = w->sld;
    a.num_sms = num_sms();
    return a;
}

}  // namespace

namespace moe {
moe_status validate_config(const moe_config *cfg) { return check_cfg(cfg); }

namespace {
struct SavedPreacts {
    const void *bwd_ws;
    const void *fwd_ws;
    moe_config cfg;
};
std::mutex g_pre_mu;
std::vector<SavedPreacts> g_pre;
bool same_cfg(const moe_config &a, const moe_config &b) { return memcmp(&a, &b, sizeof(moe_config)) == 0; }
}  // namespace

void note_saved_preacts(const void *bwd_ws, const void *fwd_ws, const moe_config &cfg) {
    std::lock_guard<std::mutex> lock(g_pre_mu);
    g_pre.push_back(SavedPreacts{bwd_ws, fwd_ws, cfg});
}
bool take_saved_preacts(const void *bwd_ws, const void *fwd_ws, const moe_config &cfg) {
    std::lock_guard<std::mutex> lock(g_pre_mu);
    bool hit = false;
    for (size_t i = 0; i < g_pre.size();) {
        if (g_pre[i].bwd_ws == bwd_ws) {
            hit = hit || (g_pre[i].fwd_ws == fwd_ws && same_cfg(g_pre[i].cfg, cfg));
            g_pre.erase(g_pre.begin() + (long)i);
        } else {
            ++i;
        }
    }
    return hit;
}
void forget_saved_preacts(const void *ws) {
    std::lock_guard<std::mutex> lock(g_pre_mu);
    for (size_t i = 0; i < g_pre.size();) {
        if (g_pre[i].bwd_ws == ws || g_pre[i].fwd_ws == ws) g_pre.erase(g_pre.begin() + (long)i);
        else ++i;
    }
}

void set_error_detail(const char *where, const char *what) {
    snprintf(g_detail, sizeof g_detail, "%s: %s", where, what);
}
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_config *cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return layout(cfg).total;
}

int32_t moe_capacity(const moe_config *cfg) {
    if (check_cfg(cfg) != MOE_OK) return -1;
    if (!(cfg->capacity_factor > 0.f)) return -1;
    const double c = floor((double)cfg->capacity_factor * (double)cfg->top_k * (double)cfg->T / (double)cfg->E);
    return c > 2147483647.0 ? 2147483647 : (int32_t)c;
}

int32_t moe_router_blocks(const moe_config *cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return moe::router_blocks(cfg->T, cfg->dtype == MOE_BF16);
}

int64_t moe_perm_rows(const moe_config *cfg) {
    if (check_cfg(cfg) != MOE_OK) return 0;
    return perm_rows(cfg);
}

const char *moe_last_error_detail(void) { return g_detail; }

moe_status moe_workspace_init(void *ws, size_t ws_bytes, moe_stream_t stream) {
    if (!ws || ws_bytes < sizeof(moe::WsHeader)) return fail(MOE_ERR_WORKSPACE, "workspace missing or < 256 bytes%s");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned%s");
    forget_frozen(ws);
    moe::forget_saved_preacts(ws);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(moe::WsHeader), reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_workspace_init");
}

moe_status moe_router_freeze(const moe_config *cfg, const float *Wr, void *ws, size_t ws_bytes,
                             moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(Wr);
    ALIGNED(Wr, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    if (cfg->dtype != MOE_BF16) return MOE_OK;      // fp32 layers keep every product in fp32: nothing to split
    moe::RouterArgs a{};
    a.Wr = Wr; a.d = cfg->d_model; a.E = cfg->E;
    a.wsplit = at<char>(ws, layout(cfg).router_w);
    a.pdl = false;
    cudaError_t e = moe::launch_router_split(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "router_freeze");
    set_frozen(ws, Wr, cfg->d_model, cfg->E);
    return MOE_OK;
}

moe_status moe_router_topk(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                           const float *sel_bias, int32_t *idx, float *gate, float *logits_out, float *psum,
                           void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    if (cfg->T > 0) { NEED(x); NEED(Wr); NEED(idx); NEED(gate); NEED(psum); }
    ALIGNED(x, 16); ALIGNED(Wr, 4); ALIGNED(logit_bias, 4); ALIGNED(sel_bias, 4); ALIGNED(idx, 4);
    ALIGNED(gate, 4); ALIGNED(logits_out, 4); ALIGNED(psum, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::RouterArgs a{x, Wr, logit_bias, sel_bias, idx, gate, logits_out, psum,
                      cfg->T, cfg->d_model, cfg->E, cfg->top_k, cfg->score, cfg->renorm,
                      at<char>(ws, layout(cfg).router_w), at<float>(ws, layout(cfg).logits), status_word(ws),
                      num_sms()};
    a.split_ready = cfg->dtype == MOE_BF16 && router_split_ready(ws, Wr, cfg->d_model, cfg->E);
    cudaError_t e = moe::launch_router(a, cfg->dtype == MOE_BF16, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "router");
}

moe_status moe_permute(const moe_config *cfg, const void *x, const int32_t *idx, const float *gate,
                       int32_t *counts, int32_t *kept, int32_t *offsets, int32_t *row_of, int32_t *row_token,
                       float *row_gate, void *x_perm, int32_t *n_dropped, void *ws, size_t ws_bytes,
                       moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(counts); NEED(kept); NEED(offsets);
    if (cfg->T > 0) { NEED(x); NEED(idx); NEED(gate); NEED(row_of); NEED(row_token); NEED(row_gate); }
    ALIGNED(x, 16); ALIGNED(x_perm, 16); ALIGNED(idx, 4); ALIGNED(gate, 4); ALIGNED(counts, 4); ALIGNED(kept, 4);
    ALIGNED(offsets, 4); ALIGNED(row_of, 4); ALIGNED(row_token, 4); ALIGNED(row_gate, 4); ALIGNED(n_dropped, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    const Layout L = layout(cfg);
    moe::DispatchArgs a{};
    a.x = x; a.idx = idx; a.gate = gate;
    a.chunk_cnt = at<int32_t>(ws, L.chunk_cnt);
    a.chunk_base = at<int32_t>(ws, L.chunk_base);
    a.counts = counts; a.kept = kept; a.offsets = offsets;
    a.row_of = row_of; a.row_token = row_token; a.row_gate = row_gate; a.x_perm = x_perm;
    a.n_dropped = n_dropped;
    a.status = status_word(ws);
    a.T = cfg->T; a.d = cfg->d_model; a.E = cfg->E; a.k = cfg->top_k;
    a.capacity = moe_capacity(cfg);
    cudaError_t e = moe::launch_dispatch(a, cfg->dtype == MOE_BF16 ? 2 : 4, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "permute");
}

moe_status moe_grouped_ffn(const moe_config *cfg, const void *x_perm, const int32_t *offsets, const float *row_gate,
                           const void *W1, const float *b1, const void *Wu, const void *W2, const float *b2,
                           const void *x, const void *Wsh_g, const void *Wsh_u, const void *Wsh_d, void *y_perm,
                           void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    if (cfg->T > 0) {
        NEED(x_perm); NEED(offsets); NEED(row_gate); NEED(y_perm);
        if ((s = check_weights(cfg, W1, Wu, W2, x, Wsh_g, Wsh_u, Wsh_d)) != MOE_OK) return s;
    }
    ALIGNED(x_perm, 16); ALIGNED(y_perm, 16); ALIGNED(offsets, 4); ALIGNED(row_gate, 4); ALIGNED(b1, 4);
    ALIGNED(b2, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    moe::FfnArgs a = ffn_args(cfg, x_perm, offsets, row_gate, W1, b1, Wu, W2, b2, x, Wsh_g, Wsh_u, Wsh_d, y_perm, ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cfg->dtype == MOE_BF16 ? moe::launch_ffn_bf16(a, st) : moe::launch_ffn_f32(a, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "grouped_ffn");
}

moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *row_of, void *y, void *ws,
                       size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    if (cfg->T > 0) { NEED(y_perm); NEED(row_of); NEED(y); }
    ALIGNED(y_perm, 16); ALIGNED(y, 16); ALIGNED(row_of, 4);
    if (!ws || ws_bytes < sizeof(moe::WsHeader)) return fail(MOE_ERR_WORKSPACE, "workspace missing%s");
    moe::CombineArgs a{y_perm, row_of, y, status_word(ws), cfg->T, cfg->d_model, cfg->top_k,
                       cfg->d_ff_shared > 0 ? 1 : 0, (int64_t)cfg->T * cfg->top_k, num_sms()};
    cudaError_t e = moe::launch_combine(a, cfg->dtype == MOE_BF16, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "combine");
}

moe_status moe_balance_stats(const moe_config *cfg, const int32_t *counts, const float *psum, float *f, float *P,
                             double *loss, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(counts); NEED(f); NEED(P); NEED(loss);
    if (cfg->T > 0) NEED(psum);
    ALIGNED(counts, 4); ALIGNED(psum, 4); ALIGNED(f, 4); ALIGNED(P, 4); ALIGNED(loss, 8);
    moe::BalanceArgs a{counts, psum, f, P, loss, cfg->T, cfg->E, cfg->top_k,
                       moe::router_blocks(cfg->T, cfg->dtype == MOE_BF16)};
    cudaError_t e = moe::launch_balance(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "balance");
}

// The layer's forward pass; pre / pre_s non-null: the training form, which
// also leaves the expert pre-activations there (bf16 layers).
static moe_status forward_impl(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                               const float *sel_bias, const void *W1, const float *b1, const void *Wu, const void *W2,
                               const float *b2, const void *Wsh_g, const void *Wsh_u, const void *Wsh_d, void *y,
                               int32_t *idx, float *gate, int32_t *counts, float *f, float *P, double *loss,
                               float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream,
                               void *pre, void *pre_s) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(counts); NEED(f); NEED(P); NEED(loss);
    if (cfg->T > 0) {
        NEED(x); NEED(Wr); NEED(y); NEED(idx); NEED(gate);
        if ((s = check_weights(cfg, W1, Wu, W2, x, Wsh_g, Wsh_u, Wsh_d)) != MOE_OK) return s;
    }
    ALIGNED(x, 16); ALIGNED(y, 16); ALIGNED(Wr, 4); ALIGNED(logit_bias, 4); ALIGNED(sel_bias, 4);
    ALIGNED(b1, 4); ALIGNED(b2, 4); ALIGNED(idx, 4); ALIGNED(gate, 4); ALIGNED(counts, 4); ALIGNED(f, 4);
    ALIGNED(P, 4); ALIGNED(loss, 8); ALIGNED(logits_out, 4); ALIGNED(n_dropped, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    const Layout L = layout(cfg);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = cfg->dtype == MOE_BF16;
    float *psum = at<float>(ws, L.psum);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *row_of = at<int32_t>(ws, L.row_of);
    float *row_gate = at<float>(ws, L.row_gate);
    void *y_perm = at<char>(ws, L.y_perm);
    cudaError_t e;

    moe::RouterArgs ra{x, Wr, logit_bias, sel_bias, idx, gate, logits_out, psum,
                       cfg->T, cfg->d_model, cfg->E, cfg->top_k, cfg->score, cfg->renorm,
                       at<char>(ws, L.router_w), at<float>(ws, L.logits), status_word(ws), num_sms()};
    ra.split_ready = bf16 && router_split_ready(ws, Wr, cfg->d_model, cfg->E);
    if ((e = moe::launch_router(ra, bf16, st)) != cudaSuccess) return cuda_fail(e, "router");

    moe::DispatchArgs da{};
    da.x = x; da.idx = idx; da.gate = gate;
    da.chunk_cnt = at<int32_t>(ws, L.chunk_cnt);
    da.chunk_base = at<int32_t>(ws, L.chunk_base);
    da.counts = counts; da.kept = at<int32_t>(ws, L.kept); da.offsets = offsets;
    da.row_of = row_of; da.row_token = at<int32_t>(ws, L.row_token); da.row_gate = row_gate;
    da.x_perm = at<char>(ws, L.x_perm);
    da.n_dropped = n_dropped;
    da.status = status_word(ws);
    da.T = cfg->T; da.d = cfg->d_model; da.E = cfg->E; da.k = cfg->top_k;
    da.capacity = moe_capacity(cfg);
    // the balance statistics ride on the dispatch scan
    da.psum = psum; da.f = f; da.P = P; da.loss = loss;
    da.contrib = at<double>(ws, L.contrib);
    da.nblk = moe::router_blocks(cfg->T, bf16);
    da.pdl = true;                                 // every launch after the first overlaps its predecessor
    if ((e = moe::launch_dispatch(da, bf16 ? 2 : 4, st)) != cudaSuccess) return cuda_fail(e, "permute");

    moe::FfnArgs fa = ffn_args(cfg, da.x_perm, offsets, row_gate, W1, b1, Wu, W2, b2, x, Wsh_g, Wsh_u, Wsh_d,
                               y_perm, ws);
    fa.pdl = true;
    fa.pre = pre;
    fa.pre_s = pre_s;
    e = bf16 ? moe::launch_ffn_bf16(fa, st) : moe::launch_ffn_f32(fa, st);
    if (e != cudaSuccess) return cuda_fail(e, "grouped_ffn");

    moe::CombineArgs ca{y_perm, row_of, y, status_word(ws), cfg->T, cfg->d_model, cfg->top_k,
                        cfg->d_ff_shared > 0 ? 1 : 0, (int64_t)cfg->T * cfg->top_k, num_sms(), true};
    if ((e = moe::launch_combine(ca, bf16, st)) != cudaSuccess) return cuda_fail(e, "combine");
    return MOE_OK;
}

moe_status moe_forward(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                       const float *sel_bias, const void *W1, const float *b1, const void *Wu, const void *W2,
                       const float *b2, const void *Wsh_g, const void *Wsh_u, const void *Wsh_d, void *y,
                       int32_t *idx, float *gate, int32_t *counts, float *f, float *P, double *loss,
                       float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream) {
    return forward_impl(cfg, x, Wr, logit_bias, sel_bias, W1, b1, Wu, W2, b2, Wsh_g, Wsh_u, Wsh_d, y, idx, gate,
                        counts, f, P, loss, logits_out, n_dropped, ws, ws_bytes, stream, nullptr, nullptr);
}

moe_status moe_forward_train(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                             const float *sel_bias, const void *W1, const float *b1, const void *Wu, const void *W2,
                             const float *b2, const void *Wsh_g, const void *Wsh_u, const void *Wsh_d, void *y,
                             int32_t *idx, float *gate, int32_t *counts, float *f, float *P, double *loss,
                             float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes, void *bwd_ws,
                             size_t bwd_ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    const size_t need = moe_backward_workspace_size(cfg);
    if (need == 0) return fail(MOE_ERR_UNSUPPORTED, "training forward: the layer has no backward pass%s");
    if (!bwd_ws || (reinterpret_cast<uintptr_t>(bwd_ws) & 255u))
        return fail(MOE_ERR_WORKSPACE, "backward workspace NULL or not 256-byte aligned%s");
    if (bwd_ws_bytes < need) return fail(MOE_ERR_WORKSPACE, "backward workspace smaller than moe_backward_workspace_size()%s");
    void *GU = nullptr, *GUs = nullptr;
    if (!moe::bwd_preact_buffers(cfg, bwd_ws, &GU, &GUs))
        return fail(MOE_ERR_UNSUPPORTED, "training forward: the layer has no backward pass%s");
    moe::forget_saved_preacts(bwd_ws);
    s = forward_impl(cfg, x, Wr, logit_bias, sel_bias, W1, b1, Wu, W2, b2, Wsh_g, Wsh_u, Wsh_d, y, idx, gate, counts,
                     f, P, loss, logits_out, n_dropped, ws, ws_bytes, stream, GU, GUs);
    if (s == MOE_OK) moe::note_saved_preacts(bwd_ws, ws, *cfg);
    return s;
}

size_t moe_ep_workspace_size(const moe_config *cfg, int32_t n_src, int64_t max_rows) {
    if (check_ep_cfg(cfg, n_src, max_rows) != MOE_OK) return 0;
    return ep_ws_bytes(cfg, max_rows);
}

moe_status moe_ep_grouped_ffn(const moe_config *cfg, int32_t n_src, const int32_t *group_offsets, int64_t max_rows,
                              const void *x_rows, const float *row_gate, const void *W1, const float *b1,
                              const void *Wu, const void *W2, const float *b2, void *y_rows, void *ws,
                              size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_ep_cfg(cfg, n_src, max_rows);
    if (s != MOE_OK) return s;
    NEED(group_offsets);
    if (max_rows > 0) {
        NEED(x_rows); NEED(row_gate); NEED(y_rows); NEED(W1); NEED(W2);
        if (cfg->act == MOE_ACT_SWIGLU) NEED(Wu);
    }
    ALIGNED(x_rows, 16); ALIGNED(y_rows, 16); ALIGNED(W1, 16); ALIGNED(Wu, 16); ALIGNED(W2, 16);
    ALIGNED(group_offsets, 4); ALIGNED(row_gate, 4); ALIGNED(b1, 4); ALIGNED(b2, 4);
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL%s");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned%s");
    if (ws_bytes < ep_ws_bytes(cfg, max_rows))
        return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_ep_workspace_size()%s");
    if (max_rows == 0) return MOE_OK;
    moe::FfnArgs a{};
    a.x_perm = x_rows; a.x = nullptr; a.offsets = group_offsets; a.row_gate = row_gate;
    a.W1 = W1; a.Wu = Wu; a.W2 = W2; a.b1 = b1; a.b2 = b2;
    a.H = at<char>(ws, ep_h_offset());
    a.y_perm = y_rows;
    a.status = status_word(ws);
    a.T = 0; a.d = cfg->d_model; a.E = cfg->E; a.k = 1; a.F = cfg->d_ff; a.S = 0;
    a.n_groups = n_src * cfg->E;
    a.routed_rows = max_rows;
    a.act = cfg->act;
    a.hF = cfg->d_ff;
    a.shared_base = max_rows;
    a.num_sms = num_sms();
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cfg->dtype == MOE_BF16 ? moe::launch_ffn_bf16(a, st) : moe::launch_ffn_f32(a, st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "ep_grouped_ffn");
}

moe_status moe_workspace_view(const moe_config *cfg, void *ws, size_t ws_bytes, moe_ws_view *out) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(out);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    const Layout L = layout(cfg);
    out->kept = at<int32_t>(ws, L.kept);
    out->offsets = at<int32_t>(ws, L.offsets);
    out->row_of = at<int32_t>(ws, L.row_of);
    out->row_token = at<int32_t>(ws, L.row_token);
    out->row_gate = at<float>(ws, L.row_gate);
    out->x_perm = at<char>(ws, L.x_perm);
    out->H = at<char>(ws, L.H);
    out->y_perm = at<char>(ws, L.y_perm);
    out->h_stride = cfg->d_ff > cfg->d_ff_shared ? cfg->d_ff : cfg->d_ff_shared;
    return MOE_OK;
}

moe_status moe_bias_update(const moe_config *cfg, const int32_t *counts, float *sel_bias, float gamma,
                           moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(counts); NEED(sel_bias);
    ALIGNED(counts, 4); ALIGNED(sel_bias, 4);
    if (!isfinite(gamma)) return fail(MOE_ERR_INVALID_ARG, "gamma not finite%s");
    cudaError_t e = moe::launch_bias_update(counts, sel_bias, (double)gamma, cfg->T, cfg->top_k, cfg->E,
                                            reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "bias_update");
}

moe_status moe_routing_health(const moe_config *cfg, const int32_t *counts, const float *P, double *out,
                              moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(counts); NEED(P); NEED(out);
    ALIGNED(counts, 4); ALIGNED(P, 4); ALIGNED(out, 8);
    cudaError_t e = moe::launch_routing_health(counts, P, out, cfg->T, cfg->top_k, cfg->E,
                                               reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "routing_health");
}

moe_status moe_check_wait_timeout(void *ws, uint64_t limit_ns, moe_stream_t stream) {
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL%s");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned%s");
    if (limit_ns < 1000ull || limit_ns > 10000000000ull)
        return fail(MOE_ERR_INVALID_ARG, "limit_ns outside 1 us .. 10 s%s");
    wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status_word(ws), limit_ns);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "check_wait_timeout");
}

moe_status moe_get_device_status(void *ws, moe_stream_t stream, int32_t *status_out) {
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL%s");
    if (!status_out) return fail(MOE_ERR_INVALID_ARG, "status_out is NULL%s");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "moe_get_device_status sync");
    int32_t h[2] = {0, 0};
    e = cudaMemcpy(h, ws, sizeof h, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "moe_get_device_status read");
    e = cudaMemset(ws, 0, sizeof h);
    if (e != cudaSuccess) return cuda_fail(e, "moe_get_device_status clear");
    *status_out = h[0];
    if (h[0] != 0) snprintf(g_detail, sizeof g_detail, "device status %d, detail %d", h[0], h[1]);
    return MOE_OK;
}

moe_status moe_quantize_rows_e4m3(const void *in, int64_t rows, int32_t cols, int64_t ld_in, uint8_t *codes,
                                  int64_t ld_out, float *scale, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return fail(MOE_ERR_INVALID_ARG, "negative rows or cols%s");
    if (rows == 0 || cols == 0) return MOE_OK;
    NEED(in); NEED(codes); NEED(scale);
    if (cols % 8) return fail(MOE_ERR_UNSUPPORTED, "cols must be a multiple of 8%s");
    if (ld_in < cols || ld_in % 8) return fail(MOE_ERR_INVALID_ARG, "ld_in < cols or not a multiple of 8%s");
    if (ld_out < cols || ld_out % 8) return fail(MOE_ERR_INVALID_ARG, "ld_out < cols or not a multiple of 8%s");
    ALIGNED(in, 16); ALIGNED(codes, 8); ALIGNED(scale, 4);
    moe::QuantArgs q{};
    q.in = static_cast<const __nv_bfloat16 *>(in);
    q.ld_in = ld_in;
    q.out = codes;
    q.ld_out = ld_out;
    q.scale = scale;
    q.rows = rows;
    q.cols = cols;
    q.num_sms = num_sms();
    cudaError_t e = moe::launch_quant_rows(q, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "quantize_rows");
}

moe_status moe_grouped_ffn_fp8(const moe_config *cfg, const uint8_t *x8_perm, const float *x8_perm_scale,
                               const int32_t *offsets, const float *row_gate, const moe_fp8_experts *w,
                               const float *b1, const float *b2, const uint8_t *x8, const float *x8_scale,
                               void *y_perm, void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    if ((s = check_fp8_cfg(cfg)) != MOE_OK) return s;
    NEED(w);
    if (cfg->T > 0) {
        NEED(x8_perm); NEED(x8_perm_scale); NEED(offsets); NEED(row_gate); NEED(y_perm);
        if ((s = check_fp8_weights(cfg, w)) != MOE_OK) return s;
        if (cfg->d_ff_shared > 0) { NEED(x8); NEED(x8_scale); }
    }
    ALIGNED(x8_perm, 16); ALIGNED(x8, 16); ALIGNED(y_perm, 16); ALIGNED(x8_perm_scale, 4); ALIGNED(x8_scale, 4);
    ALIGNED(offsets, 4); ALIGNED(row_gate, 4); ALIGNED(b1, 4); ALIGNED(b2, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    if (cfg->T == 0) return MOE_OK;
    moe::FfnArgs a = ffn_args(cfg, x8_perm, offsets, row_gate, w->W1, b1, w->Wu, w->W2, b2, x8, w->Wsh_g, w->Wsh_u,
                              w->Wsh_d, y_perm, ws);
    set_fp8(a, cfg, w, x8_perm_scale, x8_scale, ws);
    cudaError_t e = moe::launch_ffn_bf16(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "grouped_ffn_fp8");
}

moe_status moe_forward_fp8(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                           const float *sel_bias, const moe_fp8_experts *w, const float *b1, const float *b2,
                           void *y, int32_t *idx, float *gate, int32_t *counts, float *f, float *P, double *loss,
                           float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    if ((s = check_fp8_cfg(cfg)) != MOE_OK) return s;
    NEED(counts); NEED(f); NEED(P); NEED(loss); NEED(w);
    if (cfg->T > 0) {
        NEED(x); NEED(Wr); NEED(y); NEED(idx); NEED(gate);
        if ((s = check_fp8_weights(cfg, w)) != MOE_OK) return s;
    }
    ALIGNED(x, 16); ALIGNED(y, 16); ALIGNED(Wr, 4); ALIGNED(logit_bias, 4); ALIGNED(sel_bias, 4);
    ALIGNED(b1, 4); ALIGNED(b2, 4); ALIGNED(idx, 4); ALIGNED(gate, 4); ALIGNED(counts, 4); ALIGNED(f, 4);
    ALIGNED(P, 4); ALIGNED(loss, 8); ALIGNED(logits_out, 4); ALIGNED(n_dropped, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    const Layout L = layout(cfg);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *psum = at<float>(ws, L.psum);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *row_of = at<int32_t>(ws, L.row_of);
    float *row_gate = at<float>(ws, L.row_gate);
    void *y_perm = at<char>(ws, L.y_perm);
    uint8_t *x8 = at<uint8_t>(ws, L.x8);
    float *x8_scale = at<float>(ws, L.x8_scale);
    float *xperm_scale = at<float>(ws, L.xperm_scale);
    cudaError_t e;

    moe::RouterArgs ra{x, Wr, logit_bias, sel_bias, idx, gate, logits_out, psum,
                       cfg->T, cfg->d_model, cfg->E, cfg->top_k, cfg->score, cfg->renorm,
                       at<char>(ws, L.router_w), at<float>(ws, L.logits), status_word(ws), num_sms()};
    ra.split_ready = router_split_ready(ws, Wr, cfg->d_model, cfg->E);
    if ((e = moe::launch_router(ra, true, st)) != cudaSuccess) return cuda_fail(e, "router");

    moe::QuantArgs q{};                           // x -> e4m3 codes + row scales
    q.in = static_cast<const __nv_bfloat16 *>(x);
    q.ld_in = cfg->d_model;
    q.out = x8;
    q.ld_out = cfg->d_model;
    q.scale = x8_scale;
    q.rows = cfg->T;
    q.cols = cfg->d_model;
    q.num_sms = num_sms();
    q.pdl = true;
    if ((e = moe::launch_quant_rows(q, st)) != cudaSuccess) return cuda_fail(e, "quantize_x");

    moe::DispatchArgs da{};
    da.x = x8; da.idx = idx; da.gate = gate;
    da.chunk_cnt = at<int32_t>(ws, L.chunk_cnt);
    da.chunk_base = at<int32_t>(ws, L.chunk_base);
    da.counts = counts; da.kept = at<int32_t>(ws, L.kept); da.offsets = offsets;
    da.row_of = row_of; da.row_token = at<int32_t>(ws, L.row_token); da.row_gate = row_gate;
    da.x_perm = at<char>(ws, L.x_perm);
    da.x_scale = x8_scale;
    da.row_scale = xperm_scale;
    da.n_dropped = n_dropped;
    da.status = status_word(ws);
    da.T = cfg->T; da.d = cfg->d_model; da.E = cfg->E; da.k = cfg->top_k;
    da.capacity = moe_capacity(cfg);
    da.psum = psum; da.f = f; da.P = P; da.loss = loss;
    da.contrib = at<double>(ws, L.contrib);
    da.nblk = moe::router_blocks(cfg->T, true);
    da.pdl = true;
    if ((e = moe::launch_dispatch(da, 1, st)) != cudaSuccess) return cuda_fail(e, "permute");

    moe::FfnArgs fa = ffn_args(cfg, da.x_perm, offsets, row_gate, w->W1, b1, w->Wu, w->W2, b2, x8, w->Wsh_g,
                               w->Wsh_u, w->Wsh_d, y_perm, ws);
    set_fp8(fa, cfg, w, xperm_scale, x8_scale, ws);
    fa.pdl = true;
    if ((e = moe::launch_ffn_bf16(fa, st)) != cudaSuccess) return cuda_fail(e, "grouped_ffn_fp8");

    moe::CombineArgs ca{y_perm, row_of, y, status_word(ws), cfg->T, cfg->d_model, cfg->top_k,
                        cfg->d_ff_shared > 0 ? 1 : 0, (int64_t)cfg->T * cfg->top_k, num_sms(), true};
    if ((e = moe::launch_combine(ca, true, st)) != cudaSuccess) return cuda_fail(e, "combine");
    return MOE_OK;
}

// ---- block-scaled (MX) e4m3 experts

moe_status moe_quantize_rows_mx(const void *in, int64_t rows, int32_t cols, int64_t ld_in, uint8_t *codes,
                                int64_t ld_out, uint8_t *scales, int64_t ld_scale, moe_stream_t stream) {
    if (rows < 0 || cols < 0) return fail(MOE_ERR_INVALID_ARG, "negative rows or cols%s");
    if (rows == 0 || cols == 0) return MOE_OK;
    NEED(in); NEED(codes); NEED(scales);
    if (cols % 32) return fail(MOE_ERR_UNSUPPORTED, "cols must be a multiple of 32%s");
    if (ld_in < cols || ld_in % 8) return fail(MOE_ERR_INVALID_ARG, "ld_in < cols or not a multiple of 8%s");
    if (ld_out < cols || ld_out % 8) return fail(MOE_ERR_INVALID_ARG, "ld_out < cols or not a multiple of 8%s");
    if (ld_scale < cols / 32) return fail(MOE_ERR_INVALID_ARG, "ld_scale < cols / 32%s");
    ALIGNED(in, 16); ALIGNED(codes, 8);
    moe::QuantMxArgs q{};
    q.in = static_cast<const __nv_bfloat16 *>(in);
    q.ld_in = ld_in;
    q.out = codes;
    q.ld_out = ld_out;
    q.scale = scales;
    q.ld_scale = ld_scale;
    q.rows = rows;
    q.cols = cols;
    q.num_sms = num_sms();
    cudaError_t e = moe::launch_quant_mx(q, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "quantize_rows_mx");
}

size_t moe_grouped_ffn_mx_workspace_size(const moe_config *cfg, int32_t sld) {
    if (check_cfg(cfg) != MOE_OK || check_mx_cfg(cfg, sld) != MOE_OK) return 0;
    return mx_layout(cfg, sld).total;
}

moe_status moe_grouped_ffn_mx(const moe_config *cfg, const uint8_t *x8_perm, const uint8_t *xs_perm,
                              const int32_t *offsets, const float *row_gate, const moe_mx_experts *w, const float *b1,
                              const float *b2, const uint8_t *x8, const uint8_t *xs, void *y_perm, void *ws,
                              size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(w);
    if ((s = check_mx_cfg(cfg, w->sld)) != MOE_OK) return s;
    const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
    const bool shared = cfg->d_ff_shared > 0;
    if (cfg->T > 0) {
        NEED(x8_perm); NEED(xs_perm); NEED(offsets); NEED(row_gate); NEED(y_perm);
        NEED(w->W1); NEED(w->W1_scale); NEED(w->W2); NEED(w->W2_scale);
        if (swiglu) { NEED(w->Wu); NEED(w->Wu_scale); }
        if (shared) {
            NEED(x8); NEED(xs); NEED(w->Wsh_g); NEED(w->Wsh_g_scale); NEED(w->Wsh_d); NEED(w->Wsh_d_scale);
            if (swiglu) { NEED(w->Wsh_u); NEED(w->Wsh_u_scale); }
        }
    }
    ALIGNED(x8_perm, 16); ALIGNED(xs_perm, 16); ALIGNED(x8, 16); ALIGNED(xs, 16); ALIGNED(y_perm, 16);
    ALIGNED(offsets, 4); ALIGNED(row_gate, 4); ALIGNED(b1, 4); ALIGNED(b2, 4);
    ALIGNED(w->W1, 16); ALIGNED(w->Wu, 16); ALIGNED(w->W2, 16); ALIGNED(w->Wsh_g, 16); ALIGNED(w->Wsh_u, 16);
    ALIGNED(w->Wsh_d, 16); ALIGNED(w->W1_scale, 16); ALIGNED(w->Wu_scale, 16); ALIGNED(w->W2_scale, 16);
    ALIGNED(w->Wsh_g_scale, 16); ALIGNED(w->Wsh_u_scale, 16); ALIGNED(w->Wsh_d_scale, 16);
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL%s");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned%s");
    const MxLayout L = mx_layout(cfg, w->sld);
    if (ws_bytes < L.total) return fail(MOE_ERR_WORKSPACE, "workspace smaller than moe_grouped_ffn_mx_workspace_size()%s");
    if (cfg->T == 0) return MOE_OK;
    moe::FfnMxArgs a{};
    a.x_perm = x8_perm; a.xs_perm = xs_perm; a.x = x8; a.xs = xs;
    a.offsets = offsets; a.row_gate = row_gate;
    a.W1 = w->W1; a.W1s = w->W1_scale; a.Wu = w->Wu; a.Wus = w->Wu_scale; a.W2 = w->W2; a.W2s = w->W2_scale;
    a.b1 = b1; a.b2 = b2;
    a.Wsg = w->Wsh_g; a.Wsgs = w->Wsh_g_scale; a.Wsu = w->Wsh_u; a.Wsus = w->Wsh_u_scale;
    a.Wsd = w->Wsh_d; a.Wsds = w->Wsh_d_scale;
    a.H = at<__nv_bfloat16>(ws, L.H);
    a.H8 = at<uint8_t>(ws, L.H8);
    a.Hs = at<uint8_t>(ws, L.Hs);
    a.y_perm = static_cast<__nv_bfloat16 *>(y_perm);
    a.status = status_word(ws);
    a.T = cfg->T; a.d = cfg->d_model; a.E = cfg->E; a.F = cfg->d_ff; a.S = cfg->d_ff_shared; a.act = cfg->act;
    a.routed_rows = (int64_t)cfg->T * cfg->top_k;
    a.hF = L.hF;
    a.shared_base = (int64_t)cfg->T * cfg->top_k;
    a.sld = w->sld;
    a.num_sms = num_sms();
    cudaError_t e = moe::launch_ffn_mx(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "grouped_ffn_mx");
}

moe_status moe_forward_mx(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                          const float *sel_bias, const moe_mx_experts *w, const float *b1, const float *b2, void *y,
                          int32_t *idx, float *gate, int32_t *counts, float *f, float *P, double *loss,
                          float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes, void *mx_ws,
                          size_t mx_ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(w);
    if ((s = check_mx_cfg(cfg, w->sld)) != MOE_OK) return s;
    NEED(counts); NEED(f); NEED(P); NEED(loss);
    const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
    const bool shared = cfg->d_ff_shared > 0;
    if (cfg->T > 0) {
        NEED(x); NEED(Wr); NEED(y); NEED(idx); NEED(gate);
        NEED(w->W1); NEED(w->W1_scale); NEED(w->W2); NEED(w->W2_scale);
        if (swiglu) { NEED(w->Wu); NEED(w->Wu_scale); }
        if (shared) {
            NEED(w->Wsh_g); NEED(w->Wsh_g_scale); NEED(w->Wsh_d); NEED(w->Wsh_d_scale);
            if (swiglu) { NEED(w->Wsh_u); NEED(w->Wsh_u_scale); }
        }
    }
    ALIGNED(x, 16); ALIGNED(y, 16); ALIGNED(Wr, 4); ALIGNED(logit_bias, 4); ALIGNED(sel_bias, 4);
    ALIGNED(b1, 4); ALIGNED(b2, 4); ALIGNED(idx, 4); ALIGNED(gate, 4); ALIGNED(counts, 4); ALIGNED(f, 4);
    ALIGNED(P, 4); ALIGNED(loss, 8); ALIGNED(logits_out, 4); ALIGNED(n_dropped, 4);
    ALIGNED(w->W1, 16); ALIGNED(w->Wu, 16); ALIGNED(w->W2, 16); ALIGNED(w->Wsh_g, 16); ALIGNED(w->Wsh_u, 16);
    ALIGNED(w->Wsh_d, 16); ALIGNED(w->W1_scale, 16); ALIGNED(w->Wu_scale, 16); ALIGNED(w->W2_scale, 16);
    ALIGNED(w->Wsh_g_scale, 16); ALIGNED(w->Wsh_u_scale, 16); ALIGNED(w->Wsh_d_scale, 16);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    if (!mx_ws) return fail(MOE_ERR_WORKSPACE, "MX workspace is NULL%s");
    if (reinterpret_cast<uintptr_t>(mx_ws) & 255u) return fail(MOE_ERR_WORKSPACE, "MX workspace not 256-byte aligned%s");
    const MxLayout M = mx_layout(cfg, w->sld);
    if (mx_ws_bytes < M.total) return fail(MOE_ERR_WORKSPACE, "MX workspace smaller than moe_grouped_ffn_mx_workspace_size()%s");
    const Layout L = layout(cfg);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *psum = at<float>(ws, L.psum);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *row_of = at<int32_t>(ws, L.row_of);
    int32_t *row_token = at<int32_t>(ws, L.row_token);
    float *row_gate = at<float>(ws, L.row_gate);
    void *y_perm = at<char>(ws, L.y_perm);
    uint8_t *x8 = at<uint8_t>(mx_ws, M.x8);
    uint8_t *xs = at<uint8_t>(mx_ws, M.xs);
    uint8_t *xs_perm = at<uint8_t>(mx_ws, M.xs_perm);
    cudaError_t e;

    moe::RouterArgs ra{x, Wr, logit_bias, sel_bias, idx, gate, logits_out, psum,
                       cfg->T, cfg->d_model, cfg->E, cfg->top_k, cfg->score, cfg->renorm,
                       at<char>(ws, L.router_w), at<float>(ws, L.logits), status_word(ws), num_sms()};
    ra.split_ready = router_split_ready(ws, Wr, cfg->d_model, cfg->E);
    if ((e = moe::launch_router(ra, true, st)) != cudaSuccess) return cuda_fail(e, "router");

    moe::QuantMxArgs q{};                         // x -> MX codes + scale rows
    q.in = static_cast<const __nv_bfloat16 *>(x);
    q.ld_in = cfg->d_model;
    q.out = x8;
    q.ld_out = cfg->d_model;
    q.scale = xs;
    q.ld_scale = w->sld;
    q.rows = cfg->T;
    q.cols = cfg->d_model;
    q.num_sms = num_sms();
    q.pdl = true;
    if ((e = moe::launch_quant_mx(q, st)) != cudaSuccess) return cuda_fail(e, "quantize_x_mx");

    moe::DispatchArgs da{};
    da.x = x8; da.idx = idx; da.gate = gate;
    da.chunk_cnt = at<int32_t>(ws, L.chunk_cnt);
    da.chunk_base = at<int32_t>(ws, L.chunk_base);
    da.counts = counts; da.kept = at<int32_t>(ws, L.kept); da.offsets = offsets;
    da.row_of = row_of; da.row_token = row_token; da.row_gate = row_gate;
    da.x_perm = at<char>(ws, L.x_perm);
    da.n_dropped = n_dropped;
    da.status = status_word(ws);
    da.T = cfg->T; da.d = cfg->d_model; da.E = cfg->E; da.k = cfg->top_k;
    da.capacity = moe_capacity(cfg);
    da.psum = psum; da.f = f; da.P = P; da.loss = loss;
    da.contrib = at<double>(ws, L.contrib);
    da.nblk = moe::router_blocks(cfg->T, true);
    da.pdl = true;
    if ((e = moe::launch_dispatch(da, 1, st)) != cudaSuccess) return cuda_fail(e, "permute");
    if (cfg->T > 0 &&
        (e = moe::launch_mx_gather_rows(xs, xs_perm, w->sld, row_token, offsets + cfg->E,
                                        (int64_t)cfg->T * cfg->top_k, num_sms(), st)) != cudaSuccess)
        return cuda_fail(e, "gather_scales_mx");

    if (cfg->T > 0) {
        moe::FfnMxArgs a{};
        a.x_perm = at<uint8_t>(ws, L.x_perm); a.xs_perm = xs_perm; a.x = x8; a.xs = xs;
        a.offsets = offsets; a.row_gate = row_gate;
        a.W1 = w->W1; a.W1s = w->W1_scale; a.Wu = w->Wu; a.Wus = w->Wu_scale; a.W2 = w->W2; a.W2s = w->W2_scale;
        a.b1 = b1; a.b2 = b2;
        a.Wsg = w->Wsh_g; a.Wsgs = w->Wsh_g_scale; a.Wsu = w->Wsh_u; a.Wsus = w->Wsh_u_scale;
        a.Wsd = w->Wsh_d; a.Wsds = w->Wsh_d_scale;
        a.H = at<__nv_bfloat16>(mx_ws, M.H);
        a.H8 = at<uint8_t>(mx_ws, M.H8);
        a.Hs = at<uint8_t>(mx_ws, M.Hs);
        a.y_perm = static_cast<__nv_bfloat16 *>(y_perm);
        a.status = status_word(ws);
        a.T = cfg->T; a.d = cfg->d_model; a.E = cfg->E; a.F = cfg->d_ff; a.S = cfg->d_ff_shared; a.act = cfg->act;
        a.routed_rows = (int64_t)cfg->T * cfg->top_k;
        a.hF = M.hF;
        a.shared_base = (int64_t)cfg->T * cfg->top_k;
        a.sld = w->sld;
        a.num_sms = num_sms();
        if ((e = moe::launch_ffn_mx(a, st)) != cudaSuccess) return cuda_fail(e, "grouped_ffn_mx");
    }

    moe::CombineArgs ca{y_perm, row_of, y, status_word(ws), cfg->T, cfg->d_model, cfg->top_k,
                        shared ? 1 : 0, (int64_t)cfg->T * cfg->top_k, num_sms(), true};
    if ((e = moe::launch_combine(ca, true, st)) != cudaSuccess) return cuda_fail(e, "combine");
    return MOE_OK;
}


moe_status moe_grouped_ffn_w4(const moe_config *cfg, const void *x_perm, const int32_t *offsets,
                              const float *row_gate, const moe_w4_experts *w, const float *b1, const float *b2,
                              const void *x, void *y_perm, void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(w);
    if ((s = check_w4_cfg(cfg, w->sld)) != MOE_OK) return s;
    if (cfg->T > 0) {
        NEED(x_perm); NEED(offsets); NEED(row_gate); NEED(y_perm);
        if ((s = check_w4_weights(cfg, w)) != MOE_OK) return s;
        if (cfg->d_ff_shared > 0) NEED(x);
    }
    ALIGNED(x_perm, 16); ALIGNED(x, 16); ALIGNED(y_perm, 16); ALIGNED(offsets, 4); ALIGNED(row_gate, 4);
    ALIGNED(b1, 4); ALIGNED(b2, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    if (cfg->T == 0) return MOE_OK;
    moe::FfnMxArgs a = w4_args(cfg, x_perm, offsets, row_gate, w, b1, b2, x, y_perm, ws);
    cudaError_t e = moe::launch_ffn_w4(a, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "grouped_ffn_w4");
}

moe_status moe_forward_w4(const moe_config *cfg, const void *x, const float *Wr, const float *logit_bias,
                          const float *sel_bias, const moe_w4_experts *w, const float *b1, const float *b2, void *y,
                          int32_t *idx, float *gate, int32_t *counts, float *f, float *P, double *loss,
                          float *logits_out, int32_t *n_dropped, void *ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status s = check_cfg(cfg);
    if (s != MOE_OK) return s;
    NEED(w);
    if ((s = check_w4_cfg(cfg, w->sld)) != MOE_OK) return s;
    NEED(counts); NEED(f); NEED(P); NEED(loss);
    if (cfg->T > 0) {
        NEED(x); NEED(Wr); NEED(y); NEED(idx); NEED(gate);
        if ((s = check_w4_weights(cfg, w)) != MOE_OK) return s;
    }
    ALIGNED(x, 16); ALIGNED(y, 16); ALIGNED(Wr, 4); ALIGNED(logit_bias, 4); ALIGNED(sel_bias, 4);
    ALIGNED(b1, 4); ALIGNED(b2, 4); ALIGNED(idx, 4); ALIGNED(gate, 4); ALIGNED(counts, 4); ALIGNED(f, 4);
    ALIGNED(P, 4); ALIGNED(loss, 8); ALIGNED(logits_out, 4); ALIGNED(n_dropped, 4);
    if ((s = check_ws(cfg, ws, ws_bytes)) != MOE_OK) return s;
    moe::forget_saved_preacts(ws);        // the packed rows / hidden activation change
    const Layout L = layout(cfg);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *psum = at<float>(ws, L.psum);
    int32_t *offsets = at<int32_t>(ws, L.offsets);
    int32_t *row_of = at<int32_t>(ws, L.row_of);
    float *row_gate = at<float>(ws, L.row_gate);
    void *y_perm = at<char>(ws, L.y_perm);
    cudaError_t e;

    moe::RouterArgs ra{x, Wr, logit_bias, sel_bias, idx, gate, logits_out, psum,
                       cfg->T, cfg->d_model, cfg->E, cfg->top_k, cfg->score, cfg->renorm,
                       at<char>(ws, L.router_w), at<float>(ws, L.logits), status_word(ws), num_sms()};
    ra.split_ready = router_split_ready(ws, Wr, cfg->d_model, cfg->E);
    if ((e = moe::launch_router(ra, true, st)) != cudaSuccess) return cuda_fail(e, "router");

    moe::DispatchArgs da{};
    da.x = x; da.idx = idx; da.gate = gate;
    da.chunk_cnt = at<int32_t>(ws, L.chunk_cnt);
    da.chunk_base = at<int32_t>(ws, L.chunk_base);
    da.counts = counts; da.kept = at<int32_t>(ws, L.kept); da.offsets = offsets;
    da.row_of = row_of; da.row_token = at<int32_t>(ws, L.row_token); da.row_gate = row_gate;
    da.x_perm = at<char>(ws, L.x_perm);
    da.n_dropped = n_dropped;
    da.status = status_word(ws);
    da.T = cfg->T; da.d = cfg->d_model; da.E = cfg->E; da.k = cfg->top_k;
    da.capacity = moe_capacity(cfg);
    da.psum = psum; da.f = f; da.P = P; da.loss = loss;
    da.contrib = at<double>(ws, L.contrib);
    da.nblk = moe::router_blocks(cfg->T, true);
    da.pdl = true;
    if ((e = moe::launch_dispatch(da, 2, st)) != cudaSuccess) return cuda_fail(e, "permute");

    if (cfg->T > 0) {
        moe::FfnMxArgs a = w4_args(cfg, da.x_perm, offsets, row_gate, w, b1, b2, x, y_perm, ws);
        if ((e = moe::launch_ffn_w4(a, st)) != cudaSuccess) return cuda_fail(e, "grouped_ffn_w4");
    }
    moe::CombineArgs ca{y_perm, row_of, y, status_word(ws), cfg->T, cfg->d_model, cfg->top_k,
                        cfg->d_ff_shared > 0 ? 1 : 0, (int64_t)cfg->T * cfg->top_k, num_sms(), true};
    if ((e = moe::launch_combine(ca, true, st)) != cudaSuccess) return cuda_fail(e, "combine");
    return MOE_OK;
}

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case MOE_ERR_CUDA: return "CUDA call failed";
        case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
        case MOE_ERR_DEVICE_BOUNDS: return "device index out of range";
    }
    return "unknown status";
}

}  // extern "C"
