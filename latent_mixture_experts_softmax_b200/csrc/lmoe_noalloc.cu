// Router entry point that allocates nothing.
//
// Some callers cannot call cudaMalloc: code embedded in a host framework
// that owns every device allocation, or a latency-critical path where an
// allocation (or a workspace handed in from outside) is not available.
// lmoe_route_noalloc serves them: its scratch (control words, logits and the
// routing before it is copied out) lives in a fixed array in device memory
// that is part of this library, so the caller passes only inputs and outputs.

#include <cstring>
#include <mutex>

#include "lmoe_internal.cuh"

namespace lmoe {

constexpr int kNoAllocMaxT = 64;                     // tokens per call
constexpr int kNoAllocMaxE = kMaxExpertsTopk;       // experts (1024)
constexpr int kNoAllocMaxK = kMaxTopK;              // experts per token (16)

struct NoAllocScratch {
    Ctrl ctrl;
    float logits[kNoAllocMaxT * kNoAllocMaxE];
    int32_t idx[kNoAllocMaxT * kNoAllocMaxK];
    float w[kNoAllocMaxT * kNoAllocMaxK];
};

// 274,432 bytes; every device that loads the library holds one copy until
// the process exits.  The name is a host-side stand-in: kernels receive the
// device address obtained below, never this symbol.
static __device__ __align__(256) unsigned char g_route_scratch[sizeof(NoAllocScratch)];

constexpr int kMaxDevices = 64;
static void* g_scratch_addr[kMaxDevices];
static std::once_flag g_scratch_once[kMaxDevices];
static cudaError_t g_scratch_err[kMaxDevices];

// Device address of this device's scratch, looked up once per device with
// that device current.
static cudaError_t scratch_for_current_device(NoAllocScratch** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_scratch_once[dev], [dev]() {
        void* ptr = nullptr;
        g_scratch_err[dev] = cudaGetSymbolAddress(&ptr, g_route_scratch);
        g_scratch_addr[dev] = g_scratch_err[dev] == cudaSuccess ? ptr : nullptr;
    });
    if (g_scratch_err[dev] != cudaSuccess) return g_scratch_err[dev];
    *out = static_cast<NoAllocScratch*>(g_scratch_addr[dev]);
    return cudaSuccess;
}

}  // namespace lmoe

using namespace lmoe;

extern "C" int lmoe_route_noalloc(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b,
                                  int T, int32_t* topk_idx, float* topk_w, void* stream) {
    if (cfg == nullptr) return LMOE_ERR_ARG;
    if (lmoe_cfg_check(cfg) != LMOE_OK) return lmoe_cfg_check(cfg);
    if (T < 0 || !x || !router_w || !topk_idx || !topk_w) return LMOE_ERR_ARG;
    auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
    if (!al(x, 16) || !al(router_w, 16) || !al(topk_idx, 4) || !al(topk_w, 4) || (router_b && !al(router_b, 4)))
        return LMOE_ERR_ARG;
    if (T > kNoAllocMaxT || cfg->n_experts > kNoAllocMaxE || cfg->top_k > kNoAllocMaxK) return LMOE_ERR_WORKSPACE;
    if (T == 0) return LMOE_OK;
    NoAllocScratch* sc = nullptr;
    if (scratch_for_current_device(&sc) != cudaSuccess) return LMOE_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the CTA tickets must start at zero; the status word is cleared too
    if (cudaMemsetAsync(&sc->ctrl, 0, sizeof(Ctrl), st) != cudaSuccess) return LMOE_ERR_CUDA;

    FwdParams p;
    memset(&p, 0, sizeof(p));
    p.H = cfg->hidden; p.L = cfg->latent; p.E = cfg->n_experts; p.K = cfg->top_k; p.G = cfg->n_groups;
    p.F = cfg->ffn; p.Fs = cfg->shared_ffn; p.du_fmt = cfg->du_fmt; p.router_bf16 = cfg->router_dtype == LMOE_BF16;
    p.T = T;
    p.x = static_cast<const uint16_t*>(x);
    p.router_w = router_w;
    p.router_b = router_b;
    p.out_idx = topk_idx;
    p.out_w = topk_w;
    p.ctrl = &sc->ctrl;
    p.r.logits = sc->logits;
    p.r.idx = sc->idx;
    p.r.w = sc->w;
    return run_gemv_path(p, st, true) == cudaSuccess ? LMOE_OK : LMOE_ERR_CUDA;
}
