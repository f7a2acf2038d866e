// Interface of the tensor-core (prefill) path.
#pragma once

#include <cstring>

#include "lmoe_internal.cuh"
#include "lmoe_sm100.cuh"

namespace lmoe {

enum GemmKind { G_ROUTER = 0, G_SHARED_GATEUP = 1, G_DPROJ = 2, G_GATEUP = 3, G_DOWN = 4, G_UPROJ = 5 };

constexpr int kNtDense = 256;    // tokens per tile of the dense GEMMs (router, shared, D, U)
constexpr int kNtExpert = 128;   // expert slots per tile of the expert GEMMs
constexpr int kMaxUParts = 11;   // pieces of a split U tile (K segments: groups, then shared hi / lo)
constexpr int kMaxUPieces = 160; // split U pieces per step (bounds the partial-sum workspace)

struct __align__(64) TmaMaps {
    CUtensorMap a;    // weight operand (bf16 kinds)
    CUtensorMap a2;   // second weight matrix (shared up)
    CUtensorMap b;    // activation operand
    CUtensorMap b2;   // second activation operand (shared-expert segment of U)
};

struct PrefillParams {
    int H, L, E, K, G, F, Fs, du_fmt, T;
    int efmt;            // expert records: LMOE_EXPERTS_NVFP4 or LMOE_EXPERTS_Q3K
    int act;             // expert inputs: LMOE_ACT_FP16 or LMOE_ACT_NVFP4 (W4A4)
    // inputs
    const uint16_t* x;
    const uint16_t* router_w_bf16;
    const float* router_b;
    const uint8_t* group;
    const uint8_t* D;
    const uint8_t* U;
    const uint8_t* experts;
    const uint16_t* sg;
    const uint16_t* su;
    const uint16_t* sd;
    const uint16_t* residual;
    const uint16_t* gamma;
    float eps;
    const int32_t* inject_idx;
    const float* inject_w;
    size_t du_bytes, rec_bytes;
    // outputs
    uint16_t* y;
    int32_t* out_idx;
    float* out_w;
    // workspace
    Ctrl* ctrl;
    float* logits;       // [T][E]
    int32_t* idx;        // [T][K]
    float* w;            // [T][K]
    uint32_t* tgmask;    // [T][G]  bit k: expert k of the token is in group g     (zeroed)
    int32_t* cnt;        // [E]                                                   (zeroed)
    int32_t* fill;       // [E]                                                   (zeroed)
    uint8_t* dhit;       // [ceil(T/kNtDense)][G] a token of the tile hits g      (zeroed)
    int32_t* n_etiles;   // [1]
    int32_t* n_unique;   // [1]
    int32_t* off;        // [E]
    int32_t* uexp;       // [min(E, T*K)]
    int32_t* ucnt;
    int32_t* uoff;
    int4* etile;         // expert token tiles {expert, first slot, slots (<= 128), distinct index}
    int32_t* slot_pair;  // [T*K]
    // U's last, partial wave of tiles runs split by K segments so that every
    // SM gets a share: tiles [u_whole, n) as u_parts pieces, piece p taking
    // segments [u_segb[p], u_segb[p + 1]); their fp32 partial sums go to
    // upart [piece][kNtDense tokens][128 rows] and k_u_reduce adds them up
    int u_whole, u_parts;
    int u_segb[kMaxUParts + 1];
    float* upart;
    float* wslot;        // [T*K] routing weight of each expert slot
    int32_t* pair_slot;  // [T*K]
    __half* xh;          // [T][H]   fp16 block input
    uint16_t* xr;        // [T][H]   bf16 normalised input (stack) or nullptr
    uint16_t* xr_lo;     // [T][H]   bf16 remainder of the normalised input
    __half* hperm;       // [T*K][L] D_g x per expert slot
    __half* zperm;       // [T*K][F]
    __half* operm;       // [T*K][L] weighted expert outputs
    __half* s;           // [T][G][L]
    uint16_t* zsh;       // [2][T][Fs] shared-expert hidden as bf16 high and low parts
    // W4A4: NVFP4 activations of hperm, then of zperm (one buffer serves both)
    uint8_t* aq;         // codes [K/32][T*K][16]
    uint32_t* asf;       // scale words [K/64][T*K]
    float* aG;           // [T*K]
};

cudaError_t run_prefill_route(PrefillParams p, cudaStream_t st);
cudaError_t run_act_quant(const __half* src, int n, int K, uint8_t* codes, uint32_t* sfw, float* G, cudaStream_t st);
cudaError_t run_w4a4_gateup(const PrefillParams& p, const uint8_t* aq, const uint32_t* asf, const float* aG, int n,
                            cudaStream_t st);
cudaError_t run_w4a4_down(const PrefillParams& p, const uint8_t* aq, const uint32_t* asf, const float* aG, int n,
                          cudaStream_t st);
cudaError_t run_prefill_path(PrefillParams p, cudaStream_t st, void* memset_base, size_t memset_bytes,
                             void (*mark)(cudaStream_t));

}  // namespace lmoe
