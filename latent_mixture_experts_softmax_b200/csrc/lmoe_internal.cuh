// Internal interface between the C-ABI layer and the kernels.
#pragma once

#include "lmoe_common.cuh"

namespace lmoe {

constexpr int kMaxExpertsTopk = 1024;   // experts a router warp holds in registers (32 per lane)

// Streaming loads of weights that are read once: no L1 allocation.
__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ float4 ldg_stream(const float4* p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

// The CTA's threads split [ptr, ptr + bytes) into 64 KiB pieces and ask the
// TMA unit to bring each into L2 (a hint: nothing waits on it).
__device__ __forceinline__ void l2_prefetch_range(const void* ptr, size_t bytes) {
    constexpr size_t kPiece = 64 * 1024;
    const char* base = static_cast<const char*>(ptr);
    const size_t n = (bytes + kPiece - 1) / kPiece;
    for (size_t i = threadIdx.x; i < n; i += blockDim.x) {
        const size_t off = i * kPiece;
        const uint32_t len = (uint32_t)min(kPiece, bytes - off) & ~15u;
        if (len) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + off), "r"(len) : "memory");
    }
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

struct FwdParams {
    // shape
    int H, L, E, K, G, F, Fs, du_fmt, router_bf16;
    int efmt;   // expert records: LMOE_EXPERTS_NVFP4 or LMOE_EXPERTS_Q3K
    int act;    // expert inputs: LMOE_ACT_FP16 or LMOE_ACT_NVFP4 (W4A4)
    int T;
    // inputs
    const uint16_t* x;
    const void* router_w;
    const float* router_b;
    const uint8_t* group;
    const uint8_t* D;
    const uint8_t* U;
    const uint8_t* experts;
    const uint16_t* sg;
    const uint16_t* su;
    const uint16_t* sd;
    const uint16_t* residual;
    const uint16_t* gamma;   // RMSNorm of x before the block (stack), nullptr: none
    float eps;
    const int32_t* inject_idx;
    const float* inject_w;
    // outputs
    uint16_t* y;
    int32_t* out_idx;
    float* out_w;
    // workspace
    Ctrl* ctrl;
    Routing r;
    __half* x16;    // [T][H]       block input (normalised for the stack), fp16
    __half* h16;    // [T][G][L]    D_g x for the hit (token, group) pairs
    float* zsh;     // [T][Fs]      shared-expert hidden
    __half* zsh16;  // [T][Fs]      the same in fp16 (weight-streaming path)
    __half* o16w;   // [T*K][L]     routing-weighted expert outputs per slot (weight-streaming path)
    __half* z16;    // [T*K][F]     expert hidden per slot (slots grouped by expert)
    __half* s16;    // [T][G][L]    per-group weighted expert sums
    float* ypart;   // [G+1][T][H]  U_g parts and the shared part
    float* wpart;   // few-token path: partial 16x8 fragments of split reductions
    int* wtick;     // few-token path: parts finished per output tile
    size_t wtick_bytes;
    size_t du_bytes_D, du_bytes_U, rec_bytes;
    // launch shape of the router kernel
    int n_router_ctas, router_rows_per_warp;
    bool do_shared, do_buckets;
    bool shared_in_d;   // few tokens: the shared expert's gate/up run as items of the D kernel
    bool route_smem;    // few tokens: routing built in shared memory, all tables published
    bool prefetch_l2;   // stream the step's weights into L2 ahead of use (few tokens)
};

constexpr int kMaxStageEvents = 16;

cudaError_t run_gemv_path(const FwdParams& p, cudaStream_t st, bool route_only);
cudaError_t run_stream_path(const FwdParams& p, cudaStream_t st);
// workspace of the few-token path's split reductions, for up to T tokens
size_t stream_ws_part_bytes(int H, int L, int F, int Fs, int G, int E, int K, int T, int du_fmt);
size_t stream_ws_tick_bytes(int H, int L, int F, int Fs, int G, int E, int K, int T, int du_fmt);
// Few-token expert phases on the tensor cores (kind::mxf4nvf4): whether a
// step can take them, the workspace floats of their partial sums, launches.
bool nvf4_usable(const FwdParams& p);
size_t nvf4_part_floats();
cudaError_t run_nvf4_gateup(const FwdParams& p, cudaStream_t st);
cudaError_t run_nvf4_down(const FwdParams& p, cudaStream_t st);
void set_stage_events(void* const* events, int n);
void stage_mark(cudaStream_t st);
void stage_reset();
cudaError_t ensure_smem(const void* kernel, size_t smem);
cudaError_t run_debug_decode(int fmt, const void* blob, int R, int C, float ts, float* out, cudaStream_t st);
// D over a set of groups with fp16 or Q8_1 activations (the ablation)
size_t dproj_ablation_ws_bytes(int T, int H);
cudaError_t run_dproj_ablation(const uint16_t* x, const uint8_t* D, int T, int H, int L, int G, int fmt, int q81,
                               uint32_t gmask, size_t du_bytes, float* h, void* ws, cudaStream_t st);

}  // namespace lmoe
