// C ABI of the latent-MoE block: argument checks, workspace carve-up and
// dispatch to the kernels.  Declarations and conventions: include/lmoe.h.

#include <algorithm>
#include <cstring>

#include "lmoe_prefill.cuh"

using namespace lmoe;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_cfg(const lmoe_cfg* c) {
    if (c == nullptr) return LMOE_ERR_ARG;
    if (c->hidden <= 0 || c->latent <= 0 || c->n_experts <= 0 || c->top_k <= 0 || c->n_groups <= 0 ||
        c->ffn <= 0 || c->shared_ffn <= 0)
        return LMOE_ERR_ARG;
    if (c->hidden % 128 || c->latent % 128 || c->ffn % 64 || c->shared_ffn % 64) return LMOE_ERR_UNSUPPORTED;
    if (c->hidden > 960 * 32) return LMOE_ERR_UNSUPPORTED;
    if (c->top_k > kMaxTopK || c->top_k > c->n_experts || c->n_experts > kMaxExpertsTopk) return LMOE_ERR_UNSUPPORTED;
    if (c->n_groups > kMaxGroups || c->n_groups > 255) return LMOE_ERR_UNSUPPORTED;
    if (c->du_fmt != LMOE_Q8_0 && c->du_fmt != LMOE_Q4_0) return LMOE_ERR_UNSUPPORTED;
    if (c->router_dtype != LMOE_F32 && c->router_dtype != LMOE_BF16) return LMOE_ERR_UNSUPPORTED;
    if (c->expert_fmt != LMOE_EXPERTS_NVFP4 && c->expert_fmt != LMOE_EXPERTS_Q3K) return LMOE_ERR_UNSUPPORTED;
    if (c->expert_fmt == LMOE_EXPERTS_Q3K && c->latent % 256) return LMOE_ERR_UNSUPPORTED;
    if (c->act_fmt != LMOE_ACT_FP16 && c->act_fmt != LMOE_ACT_NVFP4) return LMOE_ERR_UNSUPPORTED;
    if (c->act_fmt == LMOE_ACT_NVFP4 && (c->expert_fmt != LMOE_EXPERTS_NVFP4 || c->latent % 128 || c->ffn % 128 ||
                                         c->latent > 2048 || c->ffn > 2048))
        return LMOE_ERR_UNSUPPORTED;
    return LMOE_OK;
}

size_t du_matrix_bytes(const lmoe_cfg& c) {
    return (size_t)c.latent * c.hidden / 32 * (c.du_fmt == LMOE_Q8_0 ? 34 : 18);
}

size_t record_bytes(const lmoe_cfg& c) {
    const size_t lf = (size_t)c.latent * c.ffn;
    if (c.expert_fmt == LMOE_EXPERTS_Q3K) return 2 * (lf / 256 * 110) + lf / 32 * 18;
    return 3 * lf / 2 + 3 * lf / 16 + 16;
}

// Token count from which the tensor-core path runs (bf16 router only).
constexpr int kPrefillMinT = 64;

// (the router GEMM tiles the experts by 128)
bool use_prefill(const lmoe_cfg& c, int T) {
    return T >= kPrefillMinT && c.router_dtype == LMOE_BF16 && c.n_experts % 128 == 0 && c.n_groups <= 62;
}

// Workspace of the few-token path (first) and of the tensor-core path; both
// start after the control block, so one allocation serves either.
struct WsLayout {
    size_t ctrl, idx, w, logits, n_unique, uexp, ucnt, uoff, ugrp, slot_pair, pair_slot, slot_tok, slot_w, pgrp, ghit,
        tghit, wpart, wtick;
    size_t wtick_bytes;
    size_t x16, h16, zsh, zsh16, o16w, z16, s16, ypart, xio, yio, xa, xb;
    // tensor-core path
    size_t p_zero_begin, p_tgmask, p_cnt, p_fill, p_dhit, p_n_etiles, p_zero_end;
    size_t p_n_unique, p_off, p_uexp, p_ucnt, p_uoff, p_etile, p_slot_pair, p_wslot, p_pair_slot, p_idx, p_w, p_logits;
    size_t p_xh, p_xr, p_xr_lo, p_hperm, p_zperm, p_operm, p_s, p_zsh, p_aq, p_asf, p_aG, p_upart;
    size_t total;
};

WsLayout ws_layout(const lmoe_cfg& c, int T) {
    WsLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~(size_t)255;
        return o;
    };
    L.ctrl = take(sizeof(Ctrl));
    L.xio = take((size_t)T * c.hidden * 2);
    L.yio = take((size_t)T * c.hidden * 2);
    L.xa = take((size_t)T * c.hidden * 2);
    L.xb = take((size_t)T * c.hidden * 2);
    const size_t common = off;
    // few-token path (used below kPrefillMinT tokens)
    {
        const int Td = use_prefill(c, T) ? kPrefillMinT - 1 : T;
        const size_t TK = (size_t)Td * c.top_k;
        L.idx = take(TK * 4);
        L.w = take(TK * 4);
        L.logits = take((size_t)Td * c.n_experts * 4);
        L.n_unique = take(4);
        L.uexp = take(TK * 4);
        L.ucnt = take(TK * 4);
        L.uoff = take(TK * 4);
        L.ugrp = take(TK * 4);
        L.slot_pair = take(TK * 4);
        L.pair_slot = take(TK * 4);
        L.slot_tok = take(TK * 4);
        L.slot_w = take(TK * 4);
        L.pgrp = take(TK * 4);
        L.ghit = take((size_t)c.n_groups * 4);
        L.tghit = take((size_t)Td * c.n_groups);
        L.x16 = take((size_t)Td * c.hidden * 2);
        L.h16 = take((size_t)Td * c.n_groups * c.latent * 2);
        L.zsh = take((size_t)Td * c.shared_ffn * 4);
        L.zsh16 = take((size_t)Td * c.shared_ffn * 2);
        L.o16w = take(TK * c.latent * 2);
        L.z16 = take(TK * c.ffn * 2);
        L.s16 = take((size_t)Td * c.n_groups * c.latent * 2);
        L.ypart = take((size_t)(c.n_groups + 1) * Td * c.hidden * 4);
        const int Ts = std::min(Td, 8);
        L.wpart = take(stream_ws_part_bytes(c.hidden, c.latent, c.ffn, c.shared_ffn, c.n_groups, c.n_experts, c.top_k, Ts,
                                            c.du_fmt));
        L.wtick_bytes = stream_ws_tick_bytes(c.hidden, c.latent, c.ffn, c.shared_ffn, c.n_groups, c.n_experts, c.top_k, Ts,
                                             c.du_fmt);
        L.wtick = take(L.wtick_bytes);
    }
    const size_t end_decode = off;
    if (use_prefill(c, T)) {
        off = common;
        const size_t TK = (size_t)T * c.top_k;
        const size_t ttiles = (T + kNtDense - 1) / kNtDense;
        L.p_zero_begin = off;
        L.p_tgmask = take((size_t)T * c.n_groups * 4);
        L.p_cnt = take((size_t)c.n_experts * 4);
        L.p_fill = take((size_t)c.n_experts * 4);
        L.p_dhit = take(ttiles * c.n_groups);
        L.p_n_etiles = take(4);
        L.p_zero_end = off;
        L.p_n_unique = take(4);
        L.p_off = take((size_t)c.n_experts * 4);
        const size_t nu = std::min((size_t)c.n_experts, TK);
        L.p_uexp = take(nu * 4);
        L.p_ucnt = take(nu * 4);
        L.p_uoff = take(nu * 4);
        L.p_etile = take((nu + TK / kNtExpert + 1) * 16);
        L.p_slot_pair = take(TK * 4);
        L.p_wslot = take(TK * 4);
        L.p_pair_slot = take(TK * 4);
        L.p_idx = take(TK * 4);
        L.p_w = take(TK * 4);
        L.p_logits = take((size_t)T * c.n_experts * 4);
        L.p_xh = take((size_t)T * c.hidden * 2);
        L.p_xr = take((size_t)T * c.hidden * 2);
        L.p_xr_lo = take((size_t)T * c.hidden * 2);
        L.p_hperm = take(TK * c.latent * 2);
        L.p_zperm = take(TK * c.ffn * 2);
        L.p_operm = take(TK * c.latent * 2);
        L.p_s = take((size_t)T * c.n_groups * c.latent * 2);
        L.p_zsh = take((size_t)2 * T * c.shared_ffn * 2);
        L.p_upart = take((size_t)kMaxUPieces * kNtDense * 128 * 4);   // U's split pieces
        if (c.act_fmt == LMOE_ACT_NVFP4) {
            const size_t Kmax = std::max(c.latent, c.ffn);
            L.p_aq = take(TK * Kmax / 2);
            L.p_asf = take(TK * Kmax / 16);
            L.p_aG = take(TK * 4);
        }
    }
    L.total = std::max(off, end_decode);
    return L;
}

FwdParams base_params(const lmoe_cfg& c, int T, void* ws, const WsLayout& L) {
    FwdParams p;
    std::memset(&p, 0, sizeof(p));
    p.H = c.hidden; p.L = c.latent; p.E = c.n_experts; p.K = c.top_k; p.G = c.n_groups;
    p.F = c.ffn; p.Fs = c.shared_ffn; p.du_fmt = c.du_fmt; p.router_bf16 = c.router_dtype == LMOE_BF16;
    p.efmt = c.expert_fmt;
    p.act = c.act_fmt;
    p.T = T;
    char* b = static_cast<char*>(ws);
    p.ctrl = reinterpret_cast<Ctrl*>(b + L.ctrl);
    p.r.idx = reinterpret_cast<int32_t*>(b + L.idx);
    p.r.w = reinterpret_cast<float*>(b + L.w);
    p.r.logits = reinterpret_cast<float*>(b + L.logits);
    p.r.n_unique = reinterpret_cast<int32_t*>(b + L.n_unique);
    p.r.uexp = reinterpret_cast<int32_t*>(b + L.uexp);
    p.r.ucnt = reinterpret_cast<int32_t*>(b + L.ucnt);
    p.r.uoff = reinterpret_cast<int32_t*>(b + L.uoff);
    p.r.ugrp = reinterpret_cast<int32_t*>(b + L.ugrp);
    p.r.slot_pair = reinterpret_cast<int32_t*>(b + L.slot_pair);
    p.r.pair_slot = reinterpret_cast<int32_t*>(b + L.pair_slot);
    p.r.slot_tok = reinterpret_cast<int32_t*>(b + L.slot_tok);
    p.r.slot_w = reinterpret_cast<float*>(b + L.slot_w);
    p.r.pgrp = reinterpret_cast<int32_t*>(b + L.pgrp);
    p.r.ghit = reinterpret_cast<int32_t*>(b + L.ghit);
    p.r.tghit = reinterpret_cast<uint8_t*>(b + L.tghit);
    p.x16 = reinterpret_cast<__half*>(b + L.x16);
    p.h16 = reinterpret_cast<__half*>(b + L.h16);
    p.zsh = reinterpret_cast<float*>(b + L.zsh);
    p.zsh16 = reinterpret_cast<__half*>(b + L.zsh16);
    p.o16w = reinterpret_cast<__half*>(b + L.o16w);
    p.z16 = reinterpret_cast<__half*>(b + L.z16);
    p.s16 = reinterpret_cast<__half*>(b + L.s16);
    p.ypart = reinterpret_cast<float*>(b + L.ypart);
    p.wpart = reinterpret_cast<float*>(b + L.wpart);
    p.wtick = reinterpret_cast<int*>(b + L.wtick);
    p.wtick_bytes = L.wtick_bytes;
    p.du_bytes_D = du_matrix_bytes(c);
    p.du_bytes_U = du_matrix_bytes(c);
    p.rec_bytes = record_bytes(c);
    p.eps = 0.f;
    return p;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA; }

// Reset the CTA tickets (the status word is kept until it is read).
cudaError_t reset_tickets(void* ws, cudaStream_t st) {
    return cudaMemsetAsync(static_cast<char*>(ws) + offsetof(Ctrl, route_ticket), 0,
                           sizeof(Ctrl) - offsetof(Ctrl, route_ticket), st);
}

int check_block_ptrs(const void* x, const void* router_w, const uint8_t* expert_group, const void* D, const void* U,
                     const void* experts, const lmoe_shared* shared, const void* y) {
    if (!x || !router_w || !expert_group || !D || !U || !experts || !shared || !y) return LMOE_ERR_ARG;
    if (!shared->gate || !shared->up || !shared->down) return LMOE_ERR_ARG;
    const void* p16[] = {x, router_w, D, U, experts, shared->gate, shared->up, shared->down, y};
    for (const void* q : p16)
        if (!aligned(q, 16)) return LMOE_ERR_ARG;
    return LMOE_OK;
}

// Fill the tensor-core path's parameters from the few-token ones and run it.
int run_prefill(const lmoe_cfg& c, const FwdParams& f, const WsLayout& L, void* ws, cudaStream_t st) {
    PrefillParams p;
    std::memset(&p, 0, sizeof(p));
    char* b = static_cast<char*>(ws);
    p.H = f.H; p.L = f.L; p.E = f.E; p.K = f.K; p.G = f.G; p.F = f.F; p.Fs = f.Fs; p.du_fmt = f.du_fmt; p.T = f.T;
    p.efmt = f.efmt;
    p.act = f.act;
    p.x = f.x;
    p.router_w_bf16 = static_cast<const uint16_t*>(f.router_w);
    p.router_b = f.router_b;
    p.group = f.group;
    p.D = f.D; p.U = f.U; p.experts = f.experts;
    p.sg = f.sg; p.su = f.su; p.sd = f.sd;
    p.residual = f.residual;
    p.gamma = f.gamma;
    p.eps = f.eps;
    p.inject_idx = f.inject_idx;
    p.inject_w = f.inject_w;
    p.du_bytes = f.du_bytes_D;
    p.rec_bytes = f.rec_bytes;
    p.y = f.y;
    p.out_idx = f.out_idx;
    p.out_w = f.out_w;
    p.ctrl = f.ctrl;
    p.logits = reinterpret_cast<float*>(b + L.p_logits);
    p.idx = reinterpret_cast<int32_t*>(b + L.p_idx);
    p.w = reinterpret_cast<float*>(b + L.p_w);
    p.tgmask = reinterpret_cast<uint32_t*>(b + L.p_tgmask);
    p.cnt = reinterpret_cast<int32_t*>(b + L.p_cnt);
    p.fill = reinterpret_cast<int32_t*>(b + L.p_fill);
    p.dhit = reinterpret_cast<uint8_t*>(b + L.p_dhit);
    p.n_etiles = reinterpret_cast<int32_t*>(b + L.p_n_etiles);
    p.n_unique = reinterpret_cast<int32_t*>(b + L.p_n_unique);
    p.off = reinterpret_cast<int32_t*>(b + L.p_off);
    p.uexp = reinterpret_cast<int32_t*>(b + L.p_uexp);
    p.ucnt = reinterpret_cast<int32_t*>(b + L.p_ucnt);
    p.uoff = reinterpret_cast<int32_t*>(b + L.p_uoff);
    p.etile = reinterpret_cast<int4*>(b + L.p_etile);
    p.slot_pair = reinterpret_cast<int32_t*>(b + L.p_slot_pair);
    p.wslot = reinterpret_cast<float*>(b + L.p_wslot);
    p.pair_slot = reinterpret_cast<int32_t*>(b + L.p_pair_slot);
    p.xh = reinterpret_cast<__half*>(b + L.p_xh);
    if (f.gamma) {
        p.xr = reinterpret_cast<uint16_t*>(b + L.p_xr);
        p.xr_lo = reinterpret_cast<uint16_t*>(b + L.p_xr_lo);
    }
    p.hperm = reinterpret_cast<__half*>(b + L.p_hperm);
    p.zperm = reinterpret_cast<__half*>(b + L.p_zperm);
    p.operm = reinterpret_cast<__half*>(b + L.p_operm);
    p.s = reinterpret_cast<__half*>(b + L.p_s);
    p.zsh = reinterpret_cast<uint16_t*>(b + L.p_zsh);
    p.upart = reinterpret_cast<float*>(b + L.p_upart);
    if (f.act == LMOE_ACT_NVFP4) {
        p.aq = reinterpret_cast<uint8_t*>(b + L.p_aq);
        p.asf = reinterpret_cast<uint32_t*>(b + L.p_asf);
        p.aG = reinterpret_cast<float*>(b + L.p_aG);
    }
    (void)c;
    stage_reset();
    return cuda_status(run_prefill_path(p, st, b + L.p_zero_begin, L.p_zero_end - L.p_zero_begin, stage_mark));
}

int forward_impl(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b,
                 const uint8_t* expert_group, const void* D, const void* U, const void* experts,
                 const lmoe_shared* shared, const void* residual, const int32_t* inject_idx, const float* inject_w,
                 int32_t* out_idx, float* out_w, void* y, int T, void* ws, size_t ws_bytes, cudaStream_t st,
                 const void* gamma, float eps) {
    int s = check_cfg(cfg);
    if (s != LMOE_OK) return s;
    if (T < 0) return LMOE_ERR_ARG;
    s = check_block_ptrs(x, router_w, expert_group, D, U, experts, shared, y);
    if (s != LMOE_OK) return s;
    if ((router_b && !aligned(router_b, 4)) || (residual && !aligned(residual, 16)) ||
        (inject_idx && !aligned(inject_idx, 4)) || (inject_w && !aligned(inject_w, 4)) ||
        (out_idx && !aligned(out_idx, 4)) || (out_w && !aligned(out_w, 4)) || (gamma && !aligned(gamma, 16)))
        return LMOE_ERR_ARG;
    if ((inject_idx == nullptr) != (inject_w == nullptr)) return LMOE_ERR_ARG;
    if (T == 0) return LMOE_OK;
    if (!ws || !aligned(ws, 256)) return LMOE_ERR_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (L.total > ws_bytes) return LMOE_ERR_WORKSPACE;
    FwdParams p = base_params(*cfg, T, ws, L);
    p.x = static_cast<const uint16_t*>(x);
    p.router_w = router_w;
    p.router_b = router_b;
    p.group = expert_group;
    p.D = static_cast<const uint8_t*>(D);
    p.U = static_cast<const uint8_t*>(U);
    p.experts = static_cast<const uint8_t*>(experts);
    p.sg = static_cast<const uint16_t*>(shared->gate);
    p.su = static_cast<const uint16_t*>(shared->up);
    p.sd = static_cast<const uint16_t*>(shared->down);
    p.residual = static_cast<const uint16_t*>(residual);
    p.gamma = static_cast<const uint16_t*>(gamma);
    p.eps = eps;
    p.inject_idx = inject_idx;
    p.inject_w = inject_w;
    p.out_idx = out_idx;
    p.out_w = out_w;
    p.y = static_cast<uint16_t*>(y);
    if (cfg->act_fmt == LMOE_ACT_NVFP4) {
        FwdParams q = p;
        q.T = std::min(T, 8);
        if (!nvf4_usable(q)) return LMOE_ERR_UNSUPPORTED;
    }
    if (use_prefill(*cfg, T)) return run_prefill(*cfg, p, L, ws, st);
    if ((cfg->expert_fmt == LMOE_EXPERTS_Q3K || cfg->act_fmt == LMOE_ACT_NVFP4) && T > 8) {
        // the Q3_K build between 9 and 63 tokens, and NVFP4 expert inputs
        // above 8 tokens: the few-token step on passes of at most 8 tokens
        // (the kernels of 9-63 tokens read NVFP4 records with fp16 inputs
        // only)
        for (int t0 = 0; t0 < T; t0 += 8) {
            FwdParams q = p;
            q.T = std::min(8, T - t0);
            q.x = p.x + (size_t)t0 * p.H;
            q.y = p.y + (size_t)t0 * p.H;
            if (p.residual) q.residual = p.residual + (size_t)t0 * p.H;
            if (p.inject_idx) { q.inject_idx = p.inject_idx + (size_t)t0 * p.K; q.inject_w = p.inject_w + (size_t)t0 * p.K; }
            if (p.out_idx) q.out_idx = p.out_idx + (size_t)t0 * p.K;
            if (p.out_w) q.out_w = p.out_w + (size_t)t0 * p.K;
            if (reset_tickets(ws, st) != cudaSuccess) return LMOE_ERR_CUDA;
            const cudaError_t e = run_gemv_path(q, st, false);
            if (e != cudaSuccess) return LMOE_ERR_CUDA;
        }
        return LMOE_OK;
    }
    cudaError_t e = reset_tickets(ws, st);
    if (e != cudaSuccess) return LMOE_ERR_CUDA;
    return cuda_status(run_gemv_path(p, st, false));
}

}  // namespace

extern "C" {

int lmoe_cfg_check(const lmoe_cfg* cfg) { return check_cfg(cfg); }

size_t lmoe_expert_record_bytes(const lmoe_cfg* cfg) { return check_cfg(cfg) == LMOE_OK ? record_bytes(*cfg) : 0; }

size_t lmoe_du_bytes(const lmoe_cfg* cfg) {
    return check_cfg(cfg) == LMOE_OK ? du_matrix_bytes(*cfg) * cfg->n_groups : 0;
}

size_t lmoe_workspace_bytes(const lmoe_cfg* cfg, int T_max) {
    if (check_cfg(cfg) != LMOE_OK || T_max < 0) return 0;
    return ws_layout(*cfg, T_max < 1 ? 1 : T_max).total;
}

int lmoe_route(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b, int T,
               int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
    int s = check_cfg(cfg);
    if (s != LMOE_OK) return s;
    if (T < 0 || !x || !router_w || !topk_idx || !topk_w) return LMOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
        (router_b && !aligned(router_b, 4)))
        return LMOE_ERR_ARG;
    if (T == 0) return LMOE_OK;
    if (!ws || !aligned(ws, 256)) return LMOE_ERR_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (L.total > ws_bytes) return LMOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    FwdParams p = base_params(*cfg, T, ws, L);
    p.x = static_cast<const uint16_t*>(x);
    p.router_w = router_w;
    p.router_b = router_b;
    p.out_idx = topk_idx;
    p.out_w = topk_w;
    if (use_prefill(*cfg, T)) {
        PrefillParams q;
        std::memset(&q, 0, sizeof(q));
        char* b = static_cast<char*>(ws);
        q.H = p.H; q.E = p.E; q.K = p.K; q.T = T;
        q.x = p.x;
        q.router_w_bf16 = static_cast<const uint16_t*>(router_w);
        q.router_b = router_b;
        q.ctrl = p.ctrl;
        q.logits = reinterpret_cast<float*>(b + L.p_logits);
        q.idx = reinterpret_cast<int32_t*>(b + L.p_idx);
        q.w = reinterpret_cast<float*>(b + L.p_w);
        q.out_idx = topk_idx;
        q.out_w = topk_w;
        return cuda_status(run_prefill_route(q, st));
    }
    cudaError_t e = reset_tickets(ws, st);
    if (e != cudaSuccess) return LMOE_ERR_CUDA;
    return cuda_status(run_gemv_path(p, st, true));
}

int lmoe_forward(const lmoe_cfg* cfg, const void* x, const void* router_w, const uint8_t* expert_group,
                 const void* D, const void* U, const void* experts, const lmoe_shared* shared, void* y, int T,
                 void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(cfg, x, router_w, nullptr, expert_group, D, U, experts, shared, nullptr, nullptr, nullptr,
                        nullptr, nullptr, y, T, ws, ws_bytes, static_cast<cudaStream_t>(stream), nullptr, 0.f);
}

int lmoe_forward_ex(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b,
                    const uint8_t* expert_group, const void* D, const void* U, const void* experts,
                    const lmoe_shared* shared, const void* residual, const int32_t* inject_idx, const float* inject_w,
                    int32_t* out_idx, float* out_w, void* y, int T, void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(cfg, x, router_w, router_b, expert_group, D, U, experts, shared, residual, inject_idx,
                        inject_w, out_idx, out_w, y, T, ws, ws_bytes, static_cast<cudaStream_t>(stream), nullptr,
                        0.f);
}

int lmoe_forward_host(const lmoe_cfg* cfg, const void* x_host, const void* router_w, const float* router_b,
                      const uint8_t* expert_group, const void* D, const void* U, const void* experts,
                      const lmoe_shared* shared, void* y_host, int T, void* ws, size_t ws_bytes, void* stream) {
    int s = check_cfg(cfg);
    if (s != LMOE_OK) return s;
    if (!x_host || !y_host || T < 0) return LMOE_ERR_ARG;
    if (T == 0) return LMOE_OK;
    if (!ws || !aligned(ws, 256)) return LMOE_ERR_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (L.total > ws_bytes) return LMOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    const size_t bytes = (size_t)T * cfg->hidden * 2;
    if (cudaMemcpyAsync(b + L.xio, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return LMOE_ERR_CUDA;
    s = forward_impl(cfg, b + L.xio, router_w, router_b, expert_group, D, U, experts, shared, nullptr, nullptr,
                     nullptr, nullptr, nullptr, b + L.yio, T, ws, ws_bytes, st, nullptr, 0.f);
    if (s != LMOE_OK) return s;
    if (cudaMemcpyAsync(y_host, b + L.yio, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return LMOE_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(st));
}

int lmoe_stack_forward(const lmoe_cfg* cfg, int n_layers, const lmoe_layer* layers, const void* x, void* y, int T,
                       float rms_eps, void* ws, size_t ws_bytes, void* stream) {
    int s = check_cfg(cfg);
    if (s != LMOE_OK) return s;
    if (n_layers < 1 || !layers || !x || !y || T < 0 || !(rms_eps >= 0.f)) return LMOE_ERR_ARG;
    for (int l = 0; l < n_layers; ++l)
        if (!layers[l].norm_gamma) return LMOE_ERR_ARG;
    if (T == 0) return LMOE_OK;
    if (!ws || !aligned(ws, 256)) return LMOE_ERR_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (L.total > ws_bytes) return LMOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* b = static_cast<char*>(ws);
    const void* cur = x;
    for (int l = 0; l < n_layers; ++l) {
        void* out = l == n_layers - 1 ? y : (void*)(b + ((l & 1) ? L.xb : L.xa));
        const lmoe_layer& ly = layers[l];
        s = forward_impl(cfg, cur, ly.router_w, ly.router_b, ly.expert_group, ly.D, ly.U, ly.experts, &ly.shared,
                         cur, nullptr, nullptr, nullptr, nullptr, out, T, ws, ws_bytes, st, ly.norm_gamma, rms_eps);
        if (s != LMOE_OK) return s;
        cur = out;
    }
    return LMOE_OK;
}

int lmoe_last_device_status(void* ws, size_t ws_bytes, void* stream) {
    if (!ws || ws_bytes < sizeof(Ctrl)) return LMOE_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LMOE_ERR_CUDA;
    if (cudaMemcpy(&host, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LMOE_ERR_CUDA;
    if (cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return LMOE_ERR_CUDA;
    return host;
}

const char* lmoe_status_str(int s) {
    switch (s) {
        case LMOE_OK: return "ok";
        case LMOE_ERR_ARG: return "invalid argument (null, size or alignment)";
        case LMOE_ERR_UNSUPPORTED: return "unsupported shape or format";
        case LMOE_ERR_CUDA: return "CUDA runtime error";
        case LMOE_ERR_WORKSPACE: return "workspace too small";
        case LMOE_ERR_TIMEOUT: return "a bounded device wait gave up";
        case LMOE_ERR_DEVICE_CHECK: return "a kernel found an invalid input";
        default: return "unknown status";
    }
}

int lmoe_profile_stage_events(void* const* events, int n) {
    if (n < 0 || n > kMaxStageEvents || (n > 0 && !events)) return LMOE_ERR_ARG;
    set_stage_events(events, n);
    return LMOE_OK;
}

int lmoe_dproj_ablation(const lmoe_cfg* cfg, const void* x, const void* D, int act_fmt, uint32_t group_mask, float* h,
                        int T, void* ws, size_t ws_bytes, void* stream) {
    int s = check_cfg(cfg);
    if (s != LMOE_OK) return s;
    if (!x || !D || !h || T < 0 || (act_fmt != 0 && act_fmt != 1)) return LMOE_ERR_ARG;
    if (!aligned(x, 16) || !aligned(D, 16) || !aligned(h, 4)) return LMOE_ERR_ARG;
    if (cfg->n_groups > 32) return LMOE_ERR_UNSUPPORTED;
    if (T == 0) return LMOE_OK;
    if (!ws || !aligned(ws, 256)) return LMOE_ERR_ARG;
    const WsLayout L = ws_layout(*cfg, T);
    if (L.total > ws_bytes) return LMOE_ERR_WORKSPACE;
    // the Q8_1 rows use the workspace's two spare activation buffers
    if (dproj_ablation_ws_bytes(T, cfg->hidden) > L.idx - L.xa) return LMOE_ERR_WORKSPACE;
    return cuda_status(run_dproj_ablation(static_cast<const uint16_t*>(x), static_cast<const uint8_t*>(D), T,
                                          cfg->hidden, cfg->latent, cfg->n_groups, cfg->du_fmt, act_fmt, group_mask,
                                          du_matrix_bytes(*cfg), h, static_cast<char*>(ws) + L.xa,
                                          static_cast<cudaStream_t>(stream)));
}

int lmoe_debug_decode(int fmt, const void* blob, int rows, int cols, float ts, float* out, void* stream) {
    if (!blob || !out || rows <= 0 || cols <= 0 || cols % 64 || !aligned(blob, 16)) return LMOE_ERR_ARG;
    if (fmt != LMOE_Q8_0 && fmt != LMOE_Q4_0 && fmt != 1 && fmt != 2 && fmt != 3) return LMOE_ERR_UNSUPPORTED;
    if (fmt == 2 && cols % 256) return LMOE_ERR_ARG;
    return cuda_status(run_debug_decode(fmt, blob, rows, cols, ts, out, static_cast<cudaStream_t>(stream)));
}

int lmoe_debug_act_quant(const void* src, int n, int cols, void* codes, void* scales, float* G, void* stream) {
    if (!src || !codes || !scales || !G || n <= 0 || cols <= 0 || cols % 64 || !aligned(src, 16) || !aligned(codes, 16) ||
        !aligned(scales, 4) || !aligned(G, 4))
        return LMOE_ERR_ARG;
    return cuda_status(run_act_quant(static_cast<const __half*>(src), n, cols, static_cast<uint8_t*>(codes),
                                     static_cast<uint32_t*>(scales), G, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
