// Shared device helpers of the latent-MoE kernels: storage-format decoders,
// workspace layout and small warp utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lmoe.h"

namespace lmoe {

constexpr int kWarp = 32;
constexpr int kMaxTopK = 16;
constexpr int kMaxExperts = 4096;
constexpr int kMaxGroups = 64;
constexpr int kChunk = 8;          // tokens held in registers per pass of the GEMV kernels
constexpr int kGemvWarps = 8;      // warps per GEMV CTA (split of the reduction dimension)

// ---------------------------------------------------------------------------
// scalar decoders
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Two bf16 packed in a 32-bit word -> (low, high) as floats.
__device__ __forceinline__ float2 bf16x2_to_f32x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ float fp16_bits_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Eight E2M1 codes (element 2i in the low nibble of byte i) -> four f16x2
// words holding elements (0,1), (2,3), (4,5), (6,7).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t h) { return __half22float2(*reinterpret_cast<const __half2*>(&h)); }

// Four E4M3 scales packed in a word -> floats (byte j -> out[j]).
__device__ __forceinline__ void e4m3x4_to_f32x4(uint32_t w, float (&s)[4]) {
    uint32_t lo, hi;
    asm("{\n\t.reg .b16 p0, p1;\n\t"
        "mov.b32 {p0, p1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, p0;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, p1;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
    float2 a = f16x2_to_f32x2(lo), b = f16x2_to_f32x2(hi);
    s[0] = a.x; s[1] = a.y; s[2] = b.x; s[3] = b.y;
}

// ---------------------------------------------------------------------------
// warp helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float silu(float a) { return a / (1.0f + __expf(-a)); }
// The same with the approximate division (relative error ~1e-6; the
// result is rounded to fp16 or bf16 right after).
__device__ __forceinline__ float silu_fast(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// Block-wide exclusive scan of one int per thread; returns the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* out, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nw ? scratch[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < nw) scratch[lane] = s;
    }
    __syncthreads();
    const int base = warp ? scratch[warp - 1] : 0;
    *out = base + x - v;
    const int total = scratch[nw - 1];
    __syncthreads();
    return total;
}


// ---------------------------------------------------------------------------
// status word and tickets (first 4 KiB of the workspace)
// ---------------------------------------------------------------------------

struct Ctrl {
    int status;                 // lmoe_status set by kernels
    int route_ticket;           // CTAs of the router that finished
    int pad[62];
    int tile_ticket[960];       // per output row tile of the U stage
};
static_assert(sizeof(Ctrl) <= 4096, "control block");

__device__ __forceinline__ void set_status(Ctrl* c, int s) { atomicCAS(&c->status, 0, s); }

// fp16 staging of activations: values outside the fp16 range (|v| > 65504,
// or NaN) would become inf; they are flagged in `bad`, and the caller
// reports LMOE_ERR_DEVICE_CHECK once.
__device__ __forceinline__ __half half_checked(float v, bool& bad) {
    bad |= !(fabsf(v) <= 65504.f);
    return __float2half_rn(v);
}
__device__ __forceinline__ __half2 half2_checked(float a, float b, bool& bad) {
    bad |= !(fabsf(a) <= 65504.f) | !(fabsf(b) <= 65504.f);
    return __floats2half2_rn(a, b);
}
__device__ __forceinline__ void report_range(Ctrl* c, bool bad) {
    if (bad) set_status(c, LMOE_ERR_DEVICE_CHECK);
}

// ---------------------------------------------------------------------------
// workspace carve-up (host and device agree through this struct)
// ---------------------------------------------------------------------------

struct Routing {
    int32_t* idx;        // [T][K]   routed experts (selection order)
    float* w;            // [T][K]   renormalised weights
    float* logits;       // [T][E]
    int32_t* n_unique;   // [1]      distinct experts hit
    int32_t* uexp;       // [T*K]    distinct experts, ascending
    int32_t* ucnt;       // [T*K]    (t, k) pairs per distinct expert
    int32_t* uoff;       // [T*K]    first slot of each distinct expert
    int32_t* ugrp;       // [T*K]    group of each distinct expert (few-token path)
    int32_t* slot_pair;  // [T*K]    slot -> pair t*K + k (slots grouped by expert)
    int32_t* pair_slot;  // [T*K]    pair -> slot
    int32_t* slot_tok;   // [T*K]    token of each slot (few-token path)
    float* slot_w;       // [T*K]    routing weight of each slot (few-token path)
    int32_t* pgrp;       // [T*K]    group of each pair (few-token path)
    int32_t* ghit;       // [G]      tokens hitting each group (any > 0 means hit)
    uint8_t* tghit;      // [T][G]   token t hits group g
};

}  // namespace lmoe
