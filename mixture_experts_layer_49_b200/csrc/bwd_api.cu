// bwd_api.cu -- moe_backward: the layer's backward pass, launched on one
// stream after the forward pass that filled the forward workspace.  See
// include/moe.h for the contract; the kernels are in bwd_sm100.cu
// (contractions) and bwd_aux.cu (the rest).
#include <stdio.h>

#include "common.cuh"
#include "kernels.cuh"

namespace {

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

struct BwdLayout {
    size_t GU, dGU, dZ, dXr, part, dh, dh16, wr16, dXrt, sh_off, GUs, dGUs, dXs, parts, colpart;
    size_t total;
};

int part_cols(int F) { return 2 * ((F + 255) / 256); }
int pad64(int v) { return (v + 63) / 64 * 64; }

BwdLayout bwd_layout(const moe_config *c) {
    BwdLayout L{};
    const size_t rows = (size_t)c->T * c->top_k;
    const size_t F = (size_t)c->d_ff, S = (size_t)c->d_ff_shared, d = (size_t)c->d_model, T = (size_t)c->T;
    const size_t gw = c->act == MOE_ACT_SWIGLU ? 2 : 1;          // G | U, or the GELU input
    const size_t E64 = (size_t)pad64(c->E);
    size_t o = 256;
    L.GU = o;     o = al256(o + rows * gw * F * 2);
    L.dGU = o;    o = al256(o + rows * gw * F * 2);
    L.dZ = o;     o = al256(o + rows * d * 2);
    L.dXr = o;    o = al256(o + rows * d * 2);
    L.part = o;   o = al256(o + rows * (size_t)part_cols(c->d_ff) * 4);
    L.dh = o;     o = al256(o + T * (size_t)c->E * 4);
    L.dh16 = o;   o = al256(o + T * E64 * 2);
    L.wr16 = o;   o = al256(o + d * E64 * 2);
    L.dXrt = o;   o = al256(o + T * d * 4);
    L.sh_off = o; o = al256(o + 2 * 4);
    L.GUs = o;    o = al256(o + T * gw * S * 2);
    L.dGUs = o;   o = al256(o + T * gw * S * 2);
    L.dXs = o;    o = al256(o + (S > 0 ? T * d * 4 : 0));
    L.parts = o;  o = al256(o + (S > 0 ? T * (size_t)part_cols(c->d_ff_shared) * 4 : 0));
    L.colpart = o; o = al256(o + (T + 255) / 256 * (size_t)c->E * 4);
    L.total = o;
    return L;
}

moe_status bfail(moe_status s, const char *what) {
    moe::set_error_detail("moe_backward", what);
    return s;
}

moe_status check_bwd_cfg(const moe_config *c) {
    moe_status s = moe::validate_config(c);
    if (s != MOE_OK) return s;
    if (c->dtype != MOE_BF16) return bfail(MOE_ERR_UNSUPPORTED, "the backward pass runs for bf16 layers");
    if (c->d_model % 64 || c->d_ff % 64 || c->d_ff_shared % 64)
        return bfail(MOE_ERR_UNSUPPORTED, "the backward pass needs d_model, d_ff, d_ff_shared multiples of 64");
    return MOE_OK;
}

template <typename T>
T *at(void *ws, size_t off) { return reinterpret_cast<T *>(static_cast<char *>(ws) + off); }

bool map2(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t ld, uint32_t box_rows) {
    return moe::make_map(m, 2, base, inner, rows, 1, ld, 0, box_rows, 2);
}
bool map3(CUtensorMap *m, const void *base, uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_mid) {
    return moe::make_map(m, 3, base, inner, mid, outer, inner, inner * mid, box_mid, 2);
}

moe::BwdGemmParams gemm(const int32_t *offsets, int G, int kgroup, int M, int N, int K, int mode, int32_t *status) {
    moe::BwdGemmParams p{};
    p.offsets = offsets;
    p.G = G;
    p.kgroup = kgroup;
    p.M = M; p.N = N; p.K = K;
    p.b_per_group = kgroup ? 0 : 1;
    p.mode = mode;
    p.status = status;
    p.timeout_ns = 2000000000ull;
    return p;
}

}  // namespace

namespace moe {

// Where moe_backward keeps the expert pre-activations inside its workspace
// (G | U rows [T*k, 2F] or W_1 x + b_1 rows [T*k, F]; the shared expert's
// [T, 2S] or [T, S]); false on an unsupported config.
bool bwd_preact_buffers(const moe_config *cfg, void *ws, void **GU, void **GUs) {
    if (check_bwd_cfg(cfg) != MOE_OK) return false;
    const BwdLayout L = bwd_layout(cfg);
    *GU = static_cast<char *>(ws) + L.GU;
    *GUs = static_cast<char *>(ws) + L.GUs;
    return true;
}

}  // namespace moe

extern "C" {

size_t moe_backward_workspace_size(const moe_config *cfg) {
    if (check_bwd_cfg(cfg) != MOE_OK) return 0;
    return bwd_layout(cfg).total;
}

moe_status moe_backward(const moe_config *cfg, const void *x, const float *Wr, const void *W1, const float *b1,
                        const void *Wu, const void *W2, const float *b2, const void *Wsh_g, const void *Wsh_u,
                        const void *Wsh_d, const int32_t *idx, const float *gate, const float *logits,
                        const int32_t *counts, const void *dy, float alpha, void *dx, float *dWr, float *dlogit_bias,
                        float *dW1, float *db1, float *dWu, float *dW2, float *db2, float *dWsh_g, float *dWsh_u,
                        float *dWsh_d, void *fwd_ws, size_t fwd_ws_bytes, void *ws, size_t ws_bytes,
                        moe_stream_t stream) {
    moe_status s = check_bwd_cfg(cfg);
    if (s != MOE_OK) return s;
    const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
    const bool shared = cfg->d_ff_shared > 0;
    auto need = [](const void *p) { return p != nullptr; };
    if (!need(W1) || !need(W2) || (swiglu && !need(Wu)) || !need(dW2) || !need(dW1) || (swiglu && !need(dWu)))
        return bfail(MOE_ERR_INVALID_ARG, "NULL expert weight or weight-gradient pointer");
    if (shared && (!need(Wsh_g) || !need(Wsh_d) || (swiglu && !need(Wsh_u)) || !need(dWsh_g) || !need(dWsh_d) ||
                   (swiglu && !need(dWsh_u))))
        return bfail(MOE_ERR_INVALID_ARG, "NULL shared-expert weight or gradient pointer");
    if (cfg->T > 0 && (!need(x) || !need(Wr) || !need(idx) || !need(gate) || !need(logits) || !need(counts) ||
                       !need(dy) || !need(dx) || !need(dWr)))
        return bfail(MOE_ERR_INVALID_ARG, "NULL input, forward output or gradient pointer");
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return bfail(MOE_ERR_WORKSPACE, "workspace NULL or misaligned");
    if (ws_bytes < bwd_layout(cfg).total) return bfail(MOE_ERR_WORKSPACE, "workspace smaller than moe_backward_workspace_size()");
    moe_ws_view v;
    if ((s = moe_workspace_view(cfg, fwd_ws, fwd_ws_bytes, &v)) != MOE_OK) return s;
    auto mis16 = [](const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u); };
    if (mis16(x) || mis16(W1) || mis16(Wu) || mis16(W2) || mis16(Wsh_g) || mis16(Wsh_u) || mis16(Wsh_d) || mis16(dy) ||
        mis16(dx) || mis16(dW1) || mis16(dWu) || mis16(dW2) || mis16(dWsh_g) || mis16(dWsh_u) || mis16(dWsh_d))
        return bfail(MOE_ERR_INVALID_ARG, "misaligned pointer (16 bytes needed)");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int T = cfg->T, d = cfg->d_model, E = cfg->E, k = cfg->top_k, F = cfg->d_ff, S = cfg->d_ff_shared;
    const BwdLayout L = bwd_layout(cfg);
    int32_t *status = reinterpret_cast<int32_t *>(fwd_ws);
    int nsm = 0, dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0) nsm = 148;
    auto cuda = [](cudaError_t e, const char *where) {
        if (e == cudaSuccess) return MOE_OK;
        char msg[200];
        snprintf(msg, sizeof msg, "%s: %s", where, cudaGetErrorString(e));
        moe::set_error_detail("moe_backward", msg);
        return MOE_ERR_CUDA;
    };
    if (T == 0) {                                  // nothing routed: every gradient is zero
        cudaError_t e = cudaSuccess;
        auto zero = [&](void *p, size_t n) { if (p && e == cudaSuccess) e = cudaMemsetAsync(p, 0, n, st); };
        zero(dWr, (size_t)d * E * 4); zero(dlogit_bias, (size_t)E * 4);
        zero(dW1, (size_t)E * F * d * 4); zero(db1, (size_t)E * F * 4); zero(dWu, (size_t)E * F * d * 4);
        zero(dW2, (size_t)E * d * F * 4); zero(db2, (size_t)E * d * 4);
        if (shared) { zero(dWsh_g, (size_t)S * d * 4); zero(dWsh_u, (size_t)S * d * 4); zero(dWsh_d, (size_t)d * S * 4); }
        return cuda(e, "zero gradients");
    }

    const int rows = T * k;
    const int gw = swiglu ? 2 : 1;
    const int E64 = pad64(E);
    __nv_bfloat16 *GU = at<__nv_bfloat16>(ws, L.GU), *dGU = at<__nv_bfloat16>(ws, L.dGU);
    __nv_bfloat16 *dZ = at<__nv_bfloat16>(ws, L.dZ);
    __nv_bfloat16 *dXr = at<__nv_bfloat16>(ws, L.dXr);
    float *part = at<float>(ws, L.part), *dh = at<float>(ws, L.dh);
    __nv_bfloat16 *dh16 = at<__nv_bfloat16>(ws, L.dh16), *wr16 = at<__nv_bfloat16>(ws, L.wr16);
    float *dXrt = at<float>(ws, L.dXrt);
    int32_t *sh_off = at<int32_t>(ws, L.sh_off);
    __nv_bfloat16 *GUs = at<__nv_bfloat16>(ws, L.GUs), *dGUs = at<__nv_bfloat16>(ws, L.dGUs);
    float *dXs = at<float>(ws, L.dXs), *parts = at<float>(ws, L.parts);
    const __nv_bfloat16 *H = static_cast<const __nv_bfloat16 *>(v.H);
    const int64_t hF = v.h_stride;
    cudaError_t e;
    CUtensorMap mA, mB, mB2;

    // ---- the shared group's row range {0, T}; the padded router operands
    {
        if ((e = moe::launch_set_pair(sh_off, 0, T, st)) != cudaSuccess) return cuda(e, "shared offsets");
        if (E64 != E) {
            if ((e = cudaMemsetAsync(dh16, 0, (size_t)T * E64 * 2, st)) != cudaSuccess) return cuda(e, "pad dh");
            if ((e = cudaMemsetAsync(wr16, 0, (size_t)d * E64 * 2, st)) != cudaSuccess) return cuda(e, "pad Wr");
        }
        if ((e = moe::launch_to_bf16(Wr, wr16, d, E, E64, st)) != cudaSuccess) return cuda(e, "Wr to bf16");
    }

    moe::BwdAuxArgs aux{};
    aux.offsets = v.offsets; aux.row_token = v.row_token; aux.row_gate = v.row_gate; aux.row_of = v.row_of;
    aux.idx = idx; aux.gate = gate; aux.logits = logits; aux.counts = counts; aux.dy = dy;
    aux.b2 = swiglu ? nullptr : b2;
    aux.part = part; aux.part_ld = part_cols(F);
    aux.dZ = dZ; aux.dh = dh; aux.dh_bf16 = dh16; aux.dh_ld = E64;
    aux.dX_rows = dXr; aux.dX_shared = shared ? dXs : nullptr; aux.dX_router = dXrt; aux.dx = dx;
    aux.alpha = alpha;
    aux.T = T; aux.d = d; aux.E = E; aux.k = k; aux.score = cfg->score; aux.renorm = cfg->renorm; aux.num_sms = nsm;

    // ---- 1. dZ = gate * dy[token] for every packed row
    if ((e = moe::launch_scale_rows(aux, rows, st)) != cudaSuccess) return cuda(e, "scale rows");

    // ---- 2. pre-activations again: G | U (SwiGLU) or W1 x + b1 (GELU), routed and shared --
    // unless moe_forward_train on fwd_ws already left them in this workspace
    const bool saved = moe::take_saved_preacts(ws, fwd_ws, *cfg);
    for (int part_i = 0; part_i < (saved ? 0 : gw); ++part_i) {
        const void *Wsrc = part_i == 0 ? W1 : Wu;
        if (!map2(&mA, v.x_perm, d, rows, d, 128) || !map3(&mB, Wsrc, d, F, E, moe::kBwdBoxRowsB)) return cuda(cudaErrorInvalidValue, "maps");
        moe::BwdGemmParams p = gemm(v.offsets, E, 0, 0, F, d, moe::BW_STORE_BF16, status);
        p.out = GU + part_i * F; p.ldo = (int64_t)gw * F;
        p.bias = (!swiglu) ? b1 : nullptr; p.bias_group_stride = F;
        if ((e = moe::launch_bwd_gemm(mA, mB, mB, false, false, p, nsm, st)) != cudaSuccess) return cuda(e, "recompute");
        if (shared) {
            const void *Ws = part_i == 0 ? Wsh_g : Wsh_u;
            if (!map2(&mA, x, d, T, d, 128) || !map3(&mB, Ws, d, S, 1, moe::kBwdBoxRowsB)) return cuda(cudaErrorInvalidValue, "maps");
            moe::BwdGemmParams q = gemm(sh_off, 1, 0, 0, S, d, moe::BW_STORE_BF16, status);
            q.out = GUs + part_i * S; q.ldo = (int64_t)gw * S;
            if ((e = moe::launch_bwd_gemm(mA, mB, mB, false, false, q, nsm, st)) != cudaSuccess) return cuda(e, "recompute shared");
        }
    }

    // ---- 3. down-projection dgrad: dH = dZ W_d (MN-major W_d), fused with the
    // activation's backward (dG | dU or dA) and the partial <H, dH> per row
    {
        if (!map2(&mA, dZ, d, rows, d, 128) || !map3(&mB, W2, F, d, E, 64)) return cuda(cudaErrorInvalidValue, "maps");
        moe::BwdGemmParams p = gemm(v.offsets, E, 0, 0, F, d, moe::BW_DGRAD2, status);
        p.part = part; p.part_ld = part_cols(F);
        p.H = H; p.ldh = hF; p.GU = GU; p.ldgu = (int64_t)gw * F; p.dGU = dGU; p.F = F; p.act = cfg->act;
        if ((e = moe::launch_bwd_gemm(mA, mB, mB, false, true, p, nsm, st)) != cudaSuccess) return cuda(e, "dgrad down");
        if (shared) {
            if (!map2(&mA, dy, d, T, d, 128) || !map3(&mB, Wsh_d, S, d, 1, 64)) return cuda(cudaErrorInvalidValue, "maps");
            moe::BwdGemmParams q = gemm(sh_off, 1, 0, 0, S, d, moe::BW_DGRAD2, status);
            q.part = parts; q.part_ld = part_cols(S);
            q.H = H + (int64_t)rows * hF; q.ldh = hF; q.GU = GUs; q.ldgu = (int64_t)gw * S; q.dGU = dGUs; q.F = S;
            q.act = cfg->act;
            if ((e = moe::launch_bwd_gemm(mA, mB, mB, false, true, q, nsm, st)) != cudaSuccess) return cuda(e, "dgrad down shared");
        }
    }

    // ---- 4. up-projection dgrad: dX = dG W_g + dU W_u (or dA W_1), bf16 rows
    {
        if (!map2(&mA, dGU, (uint64_t)gw * F, rows, (uint64_t)gw * F, 128) || !map3(&mB, W1, d, F, E, 64) ||
            !map3(&mB2, swiglu ? Wu : W1, d, F, E, 64))
            return cuda(cudaErrorInvalidValue, "maps");
        moe::BwdGemmParams p = gemm(v.offsets, E, 0, 0, d, gw * F, moe::BW_STORE_BF16, status);
        p.k_split = swiglu ? F : 0;
        p.out = dXr; p.ldo = d;
        if ((e = moe::launch_bwd_gemm(mA, mB, mB2, false, true, p, nsm, st)) != cudaSuccess) return cuda(e, "dgrad up");
        if (shared) {
            if (!map2(&mA, dGUs, (uint64_t)gw * S, T, (uint64_t)gw * S, 128) || !map3(&mB, Wsh_g, d, S, 1, 64) ||
                !map3(&mB2, swiglu ? Wsh_u : Wsh_g, d, S, 1, 64))
                return cuda(cudaErrorInvalidValue, "maps");
            moe::BwdGemmParams q = gemm(sh_off, 1, 0, 0, d, gw * S, moe::BW_STORE_F32, status);
            q.k_split = swiglu ? S : 0;
            q.out = dXs; q.ldo = d;
            if ((e = moe::launch_bwd_gemm(mA, mB, mB2, false, true, q, nsm, st)) != cudaSuccess) return cuda(e, "dgrad up shared");
        }
    }

    // ---- 5. router: gate gradients -> logits (+ balance loss); 6. its input gradient
    if ((e = moe::launch_router_bwd(aux, st)) != cudaSuccess) return cuda(e, "router backward");
    {
        if (!map2(&mA, dh16, E64, T, E64, 128) || !map3(&mB, wr16, E64, d, 1, moe::kBwdBoxRowsB)) return cuda(cudaErrorInvalidValue, "maps");
        moe::BwdGemmParams p = gemm(sh_off, 1, 0, 0, d, E64, moe::BW_STORE_F32, status);
        p.out = dXrt; p.ldo = d;
        if ((e = moe::launch_bwd_gemm(mA, mB, mB, false, false, p, nsm, st)) != cudaSuccess) return cuda(e, "router dgrad");
    }
    // ---- 7. dx
    if ((e = moe::launch_dx_combine(aux, st)) != cudaSuccess) return cuda(e, "dx combine");

    // ---- 8. weight gradients: the contraction runs over each expert's rows
    {
        // dW_d[e] = dZ_e^T H_e   [d, F]
        if (!map2(&mA, dZ, d, rows, d, 64) || !map2(&mB, H, F, rows, hF, 64)) return cuda(cudaErrorInvalidValue, "maps");
        moe::BwdGemmParams p = gemm(v.offsets, E, 1, d, F, 0, moe::BW_STORE_F32, status);
        p.out = dW2; p.ldo = F; p.out_group_stride = (int64_t)d * F;
        if ((e = moe::launch_bwd_gemm(mA, mB, mB, true, true, p, nsm, st)) != cudaSuccess) return cuda(e, "wgrad down");
        // dW_g[e] = dG_e^T X_e, dW_u[e] = dU_e^T X_e   [F, d]
        for (int part_i = 0; part_i < gw; ++part_i) {
            if (!map2(&mA, dGU + part_i * F, F, rows, (uint64_t)gw * F, 64) || !map2(&mB, v.x_perm, d, rows, d, 64))
                return cuda(cudaErrorInvalidValue, "maps");
            moe::BwdGemmParams q = gemm(v.offsets, E, 1, F, d, 0, moe::BW_STORE_F32, status);
            q.out = part_i == 0 ? dW1 : dWu; q.ldo = d; q.out_group_stride = (int64_t)F * d;
            if ((e = moe::launch_bwd_gemm(mA, mB, mB, true, true, q, nsm, st)) != cudaSuccess) return cuda(e, "wgrad up");
        }
        if (shared) {
            if (!map2(&mA, dy, d, T, d, 64) || !map2(&mB, H + (int64_t)rows * hF, S, T, hF, 64))
                return cuda(cudaErrorInvalidValue, "maps");
            moe::BwdGemmParams q = gemm(sh_off, 1, 1, d, S, 0, moe::BW_STORE_F32, status);
            q.out = dWsh_d; q.ldo = S;
            if ((e = moe::launch_bwd_gemm(mA, mB, mB, true, true, q, nsm, st)) != cudaSuccess) return cuda(e, "wgrad shared");
            for (int part_i = 0; part_i < gw; ++part_i) {
                if (!map2(&mA, dGUs + part_i * S, S, T, (uint64_t)gw * S, 64) || !map2(&mB, x, d, T, d, 64))
                    return cuda(cudaErrorInvalidValue, "maps");
                moe::BwdGemmParams r = gemm(sh_off, 1, 1, S, d, 0, moe::BW_STORE_F32, status);
                r.out = part_i == 0 ? dWsh_g : dWsh_u; r.ldo = d;
                if ((e = moe::launch_bwd_gemm(mA, mB, mB, true, true, r, nsm, st)) != cudaSuccess) return cuda(e, "wgrad shared");
            }
        }
        // dW_r = x^T dh   [d, E]
        if (!map2(&mA, x, d, T, d, 64) || !map2(&mB, dh16, E64, T, E64, 64)) return cuda(cudaErrorInvalidValue, "maps");
        moe::BwdGemmParams q = gemm(sh_off, 1, 1, d, E, 0, moe::BW_STORE_F32, status);
        q.out = dWr; q.ldo = E;
        if ((e = moe::launch_bwd_gemm(mA, mB, mB, true, true, q, nsm, st)) != cudaSuccess) return cuda(e, "router wgrad");
    }
    // ---- 9. bias gradients (GELU experts) and the logit offset's
    if (!swiglu) {
        moe::ColSumArgs c2{dZ, 0, d, v.offsets, E, 0, d, db2};
        if (db2 && (e = moe::launch_column_sums(c2, st)) != cudaSuccess) return cuda(e, "db2");
        moe::ColSumArgs c1{dGU, 0, F, v.offsets, E, 0, F, db1};
        if (db1 && (e = moe::launch_column_sums(c1, st)) != cudaSuccess) return cuda(e, "db1");
    }
    if (dlogit_bias) {
        if ((e = moe::launch_col_sums_2pass(dh, T, E, E, at<float>(ws, L.colpart), dlogit_bias, st)) != cudaSuccess)
            return cuda(e, "dbeta");
    }
    return MOE_OK;
}

}  // extern "C"
