// Few-token path (T <= 8), weight-streaming kernels: one persistent CTA per
// SM streams 16-row weight tiles through a ring of shared-memory slots with
// the TMA engine (tensor-map tile loads of the stored formats, no
// conversion on the way) while eight compute warps dequantise each tile in
// registers and multiply it with the staged activations on the tensor pipe
// (mma.sync m16n8k16, fp16 operands, fp32 accumulation; the 8 MMA columns are
// the up to 8 tokens).  Several tiles per SM are in flight at once, so HBM
// streams without waiting on the arithmetic.
//
//   k_stream<DPROJ>   h16[t][g]   = D_g x_t            (hit groups)
//   k_stream<GATEUP>  z16[slot]   = silu(W_gate h) * (W_up h)
//   k_stream<DOWN>    o16w[slot]  = w_slot * W_down z
//   k_combine_small   s16[t][g]   = sum of o16w over the token's experts in g
//   k_stream<UPROJ>   y           = sum_g U_g s16[t][g] + S_down z_sh (+ residual)
//
// Method: teardown article "Edge0-145B: a Qwen MoE with its experts
// squeezed", section "A latent in front of the experts" (layer equation,
// per-group D/U); Edge0 145B / 120B model page, architecture tables.

#include <cstring>
#include <mutex>

#include "lmoe_internal.cuh"
#include "lmoe_route.cuh"
#include "lmoe_sm100.cuh"

namespace lmoe {

using namespace sm100;

enum StreamPhase { SP_DPROJ = 0, SP_GATEUP = 1, SP_DOWN = 2, SP_UPROJ = 3 };

constexpr int kSW = 16;                // compute warps per CTA
constexpr int kStreamThreads = 32 * (kSW + 2);   // + loader warp + reducer warp
constexpr int kMaxSlots = 16;          // weight slots in the ring

__host__ __device__ __forceinline__ int round128(int b) { return (b + 127) & ~127; }
constexpr int kActPad = 32;            // halves of padding per staged activation row
constexpr uint64_t kStreamWait = 4000000000ull;   // SM cycles per barrier wait

// Every weight map is 3-D over 16-bit units: (one K block's rows, contiguous;
// K blocks; matrices).  A box takes 16 consecutive rows of every K block of
// one matrix, so each TMA line is a 256-512 byte run, not one row.
struct __align__(64) StreamMaps {
    CUtensorMap wq;    // weight codes: D/U q (over groups) or expert gate/down q (over experts)
    CUtensorMap ws;    // weight scales: D/U d or expert gate/down s
    CUtensorMap wq2;   // expert up q
    CUtensorMap ws2;   // expert up s
    int q_row;         // 16-bit units per row of one K block in wq / wq2
    int s_row;         // 16-bit units per row of one K block in ws / ws2
};

struct Item {
    int kind;   // 0: weight tile of a group / expert, 1: shared-expert tile (UPROJ)
    int mat;    // group g or expert e
    int j;      // distinct-expert index (expert phases)
    int r0;     // first of the tile's 16 output rows
};

__device__ __forceinline__ void mma16816s(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hsub2u(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// 4 signed int8 -> two f16x2 of the exact integers; 4 nibbles -> (q - 8).
__device__ __forceinline__ void s8x4_h2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = hsub2u(__byte_perm(u, 0x64646464u, 0x4140), 0x64806480u);
    hi = hsub2u(__byte_perm(u, 0x64646464u, 0x4342), 0x64806480u);
}
__device__ __forceinline__ void u4x4_h2(uint32_t n, uint32_t& lo, uint32_t& hi) {
    lo = hsub2u(__byte_perm(n, 0x64646464u, 0x4140), 0x64086408u);
    hi = hsub2u(__byte_perm(n, 0x64646464u, 0x4342), 0x64086408u);
}

// Activation fragment of token g (zero when g >= nt): 8 halves at column k.
__device__ __forceinline__ uint4 act8(const __half* xs, int ld, int g, int nt, int k) {
    return g < nt ? *reinterpret_cast<const uint4*>(xs + (size_t)g * ld + k) : make_uint4(0, 0, 0, 0);
}
__device__ __forceinline__ uint2 act4(const __half* xs, int ld, int g, int nt, int k) {
    return g < nt ? *reinterpret_cast<const uint2*>(xs + (size_t)g * ld + k) : make_uint2(0, 0);
}

// One 16-row Q8_0 / Q4_0 tile in shared memory ([block][16 rows][32 | 16 B],
// scales [block][16 rows] fp16) times the staged activations, blocks [b0, b1).
template <int FMT>
__device__ __forceinline__ void tile_du(const uint8_t* q, const uint16_t* d, const __half* xs, int ld, int nt,
                                        int b0, int b1, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int b = b0; b < b1; ++b) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        if (FMT == LMOE_Q8_0) {
            const uint2 wg = *reinterpret_cast<const uint2*>(q + ((size_t)b * 16 + g) * 32 + 8 * t);
            const uint2 wh = *reinterpret_cast<const uint2*>(q + ((size_t)b * 16 + g + 8) * 32 + 8 * t);
            uint32_t ga0, ga1, ga2, ga3, ha0, ha1, ha2, ha3;
            s8x4_h2(wg.x, ga0, ga1);
            s8x4_h2(wg.y, ga2, ga3);
            s8x4_h2(wh.x, ha0, ha1);
            s8x4_h2(wh.y, ha2, ha3);
            const uint4 xv = act8(xs, ld, g, nt, 32 * b + 8 * t);
            mma16816s(c, ga0, ha0, ga1, ha1, xv.x, xv.y);
            mma16816s(c, ga2, ha2, ga3, ha3, xv.z, xv.w);
        } else {
            const uint32_t wg = *reinterpret_cast<const uint32_t*>(q + ((size_t)b * 16 + g) * 16 + 4 * t);
            const uint32_t wh = *reinterpret_cast<const uint32_t*>(q + ((size_t)b * 16 + g + 8) * 16 + 4 * t);
            uint32_t gl0, gl1, gh0, gh1, hl0, hl1, hh0, hh1;
            u4x4_h2(wg & 0x0F0F0F0Fu, gl0, gl1);
            u4x4_h2((wg >> 4) & 0x0F0F0F0Fu, gh0, gh1);
            u4x4_h2(wh & 0x0F0F0F0Fu, hl0, hl1);
            u4x4_h2((wh >> 4) & 0x0F0F0F0Fu, hh0, hh1);
            const uint2 xl = act4(xs, ld, g, nt, 32 * b + 4 * t);
            const uint2 xh = act4(xs, ld, g, nt, 32 * b + 16 + 4 * t);
            mma16816s(c, gl0, hl0, gl1, hl1, xl.x, xl.y);
            mma16816s(c, gh0, hh0, gh1, hh1, xh.x, xh.y);
        }
        const float dg = __half2float(__ushort_as_half(d[b * 16 + g]));
        const float dh = __half2float(__ushort_as_half(d[b * 16 + g + 8]));
        acc[0] = fmaf(dg, c[0], acc[0]);
        acc[1] = fmaf(dg, c[1], acc[1]);
        acc[2] = fmaf(dh, c[2], acc[2]);
        acc[3] = fmaf(dh, c[3], acc[3]);
    }
}

// One 16-row NVFP4 tile in shared memory (codes [chunk][16 rows][16 B],
// scales [chunk/2][16 rows][4 B]), chunks [c0, c1); the E4M3 scale is folded
// into the fp16 operand (exact), the tensor scale is left to the caller.
__device__ __forceinline__ void tile_nvfp4(const uint8_t* q, const uint8_t* s, const __half* xs, int ld, int nt,
                                           int c0, int c1, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int c = c0; c < c1; ++c) {
        const uint32_t wg = *reinterpret_cast<const uint32_t*>(q + ((size_t)c * 16 + g) * 16 + 4 * t);
        const uint32_t wh = *reinterpret_cast<const uint32_t*>(q + ((size_t)c * 16 + g + 8) * 16 + 4 * t);
        const uint32_t swg = *reinterpret_cast<const uint32_t*>(s + ((size_t)(c >> 1) * 16 + g) * 4);
        const uint32_t swh = *reinterpret_cast<const uint32_t*>(s + ((size_t)(c >> 1) * 16 + g + 8) * 4);
        const int sb = 2 * (c & 1) + (t >> 1);
        uint32_t scg, sch;
        {
            uint32_t hg, hh;
            asm("{\n\t.reg .b16 a, b;\n\tcvt.u16.u32 a, %2;\n\tcvt.u16.u32 b, %3;\n\t"
                "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
                : "=r"(hg), "=r"(hh)
                : "r"((swg >> (8 * sb)) & 0xFF), "r"((swh >> (8 * sb)) & 0xFF));
            scg = (hg & 0xFFFF) | (hg << 16);
            sch = (hh & 0xFFFF) | (hh << 16);
        }
        uint32_t a[4], b[4];
        e2m1x8_to_f16x8(wg, a);
        e2m1x8_to_f16x8(wh, b);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            a[j] = hmul2u(a[j], scg);
            b[j] = hmul2u(b[j], sch);
        }
        const uint4 xv = act8(xs, ld, g, nt, c * 32 + 8 * t);
        mma16816s(acc, a[0], b[0], a[1], b[1], xv.x, xv.y);
        mma16816s(acc, a[2], b[2], a[3], b[3], xv.z, xv.w);
    }
}

// 16 rows of bf16 weights ([16][K] row-major) against fp16 activations,
// 32-column blocks [b0, b1); bf16 -> fp16 in registers.
__device__ __forceinline__ void tile_bf16(const uint16_t* w, int K, const __half* xs, int ld, int nt, int b0, int b1,
                                          float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int b = b0; b < b1; ++b) {
        const uint4 wg = *reinterpret_cast<const uint4*>(w + (size_t)g * K + 32 * b + 8 * t);
        const uint4 wh = *reinterpret_cast<const uint4*>(w + (size_t)(g + 8) * K + 32 * b + 8 * t);
        auto cv = [](uint32_t v) {
            const float2 f = bf16x2_to_f32x2(v);
            __half2 h = __floats2half2_rn(f.x, f.y);
            return *reinterpret_cast<uint32_t*>(&h);
        };
        const uint4 xv = act8(xs, ld, g, nt, 32 * b + 8 * t);
        mma16816s(acc, cv(wg.x), cv(wh.x), cv(wg.y), cv(wh.y), xv.x, xv.y);
        mma16816s(acc, cv(wg.z), cv(wh.z), cv(wg.w), cv(wh.w), xv.z, xv.w);
    }
}

// ---------------------------------------------------------------------------
// work items
// ---------------------------------------------------------------------------


template <int PHASE>
__host__ __device__ __forceinline__ int stream_rows(int H, int L, int F) {
    return PHASE == SP_DPROJ ? L : PHASE == SP_GATEUP ? F : PHASE == SP_DOWN ? L : H;
}

// What the compute and reducer warps need to know about the item in a slot.
struct __align__(16) SlotMeta {
    float tail[4];   // expert record tail: tensor scales of gate, up, down
    Item item;
    int nt;          // activation rows (tokens or slots) of the item
    int off;         // first slot of the expert (expert phases)
};

template <int PHASE>
__device__ __forceinline__ int stream_items(const FwdParams& p, const StreamShared& sh) {
    const int tiles = stream_rows<PHASE>(p.H, p.L, p.F) / 16;
    if (PHASE == SP_DPROJ) return sh.n_hit * tiles;
    if (PHASE == SP_UPROJ) return (sh.n_hit + 1) * tiles;
    return sh.n_unique * tiles;
}

// Item i: D / experts run matrix-major (consecutive items share a
// matrix); U runs row-tile-major (consecutive items are the parts of one
// output tile: the hit groups ascending, then the shared expert).
template <int PHASE>
__device__ __forceinline__ Item stream_item(const StreamShared& sh, int tiles, int i) {
    Item it;
    it.kind = 0;
    it.j = 0;
    if (PHASE == SP_UPROJ) {
        const int parts = sh.n_hit + 1, part = i % parts;
        it.r0 = (i / parts) * 16;
        it.j = part;
        if (part < sh.n_hit) it.mat = sh.hg[part];
        else { it.kind = 1; it.mat = 0; }
        return it;
    }
    const int m = i / tiles;
    it.r0 = (i % tiles) * 16;
    if (PHASE == SP_DPROJ) {
        it.mat = sh.hg[m];
    } else {
        it.j = m;
        it.mat = sh.uexp[m];
    }
    return it;
}

// First item of CTA c when n items are split into contiguous chunks.
__device__ __forceinline__ int chunk_begin(int c, int n, int ctas) {
    return (int)(((long long)c * n) / ctas);
}

// Slot layout: weights (A, A2, S, S2) then the item's activations.
template <int PHASE, int FMT>
struct SlotPlan {
    __device__ static int a_bytes(const FwdParams& p) {
        if (PHASE == SP_DPROJ) return 16 * p.H * (FMT == LMOE_Q8_0 ? 32 : 16) / 32;
        if (PHASE == SP_UPROJ) return 16 * p.L * (FMT == LMOE_Q8_0 ? 32 : 16) / 32;
        if (PHASE == SP_GATEUP) return 16 * p.L / 2;
        return 16 * p.F / 2;
    }
    __device__ static int s_bytes(const FwdParams& p) {
        if (PHASE == SP_DPROJ) return 16 * (p.H / 32) * 2;
        if (PHASE == SP_UPROJ) return 16 * (p.L / 32) * 2;
        if (PHASE == SP_GATEUP) return 16 * (p.L / 64) * 4;
        return 16 * (p.F / 64) * 4;
    }
};

// Warp roles: kSW compute warps, one loader warp (one thread issues every
// copy), one reducer warp.  The compute warps split each item's reduction
// (K) evenly, hand their partial 16 x 8 fragments to the reducer through
// one of two shared buffers and go straight on to the next item; the
// reducer sums the partials and runs the epilogue.  No step of an item
// waits for another item's epilogue.
template <int PHASE, int FMT>
__global__ void __launch_bounds__(kStreamThreads, 1) k_stream(const __grid_constant__ StreamMaps maps, FwdParams p,
                                                              int n_slots, int slot_bytes) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
    __shared__ StreamShared sh;
    __shared__ SlotMeta meta[kMaxSlots];
    __shared__ SlotMeta red_meta[2];
    __shared__ __align__(8) uint64_t full[kMaxSlots];
    __shared__ __align__(8) uint64_t empty[kMaxSlots];
    __shared__ __align__(8) uint64_t red_full[2];
    __shared__ __align__(8) uint64_t red_empty[2];
    __shared__ __align__(8) uint64_t xbar;
    __shared__ int abort_flag;
    constexpr int NV = PHASE == SP_GATEUP ? 8 : 4;   // partial values per lane (gate [+ up])
    __shared__ float red[2][kSW][32][NV];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = p.T, H = p.H, L = p.L, F = p.F, Fs = p.Fs, G = p.G, K = p.K;
    // the CTA-level activation buffer (D: x for all tokens) precedes the slots
    const int xs_bytes = PHASE == SP_DPROJ ? round128(T * (H + kActPad) * 2) : 0;
    uint8_t* slots = smem + xs_bytes;

    // Routing, as the router kernel published it.  D runs right after the
    // router kernel and waits for it first.  The later kernels read the
    // routing before their own wait: their predecessor let them launch only
    // after its own wait, so the router kernel had completed by then.
    if (PHASE == SP_DPROJ) {
        grid_dep_wait();
        grid_dep_launch();
    }
    if (PHASE == SP_GATEUP || PHASE == SP_DOWN) {
        const int n = T * K;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            sh.uexp[i] = __ldcg(p.r.uexp + i);
            sh.ucnt[i] = __ldcg(p.r.ucnt + i);
            sh.uoff[i] = __ldcg(p.r.uoff + i);
            sh.ugrp[i] = __ldcg(p.r.ugrp + i);
            const int pr = __ldcg(p.r.slot_pair + i);
            sh.slot_tok[i] = pr / K;
            sh.slot_w[i] = __ldcg(p.r.w + pr);
        }
        if (threadIdx.x == 0) sh.n_unique = __ldcg(p.r.n_unique);
    } else {
        if (threadIdx.x < G) sh.hg[threadIdx.x] = __ldcg(p.r.ghit + threadIdx.x);
        __syncthreads();
        if (threadIdx.x == 0) {
            int n = 0;
            for (int g = 0; g < G; ++g)
                if (sh.hg[g] > 0) sh.hg[n++] = g;
            sh.n_hit = n;
        }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < n_slots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kSW);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&red_full[b], kSW);
            mbar_init(&red_empty[b], 1);
        }
        mbar_init(&xbar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int tiles = stream_rows<PHASE>(H, L, F) / 16;
    const int n_items = stream_items<PHASE>(p, sh);
    const int i0 = chunk_begin(blockIdx.x, n_items, gridDim.x);
    const int i1 = chunk_begin(blockIdx.x + 1, n_items, gridDim.x);
    using SP = SlotPlan<PHASE, FMT>;
    const int abytes = SP::a_bytes(p), sbytes = SP::s_bytes(p);
    // the item's activations follow its weights, 128-byte aligned (slots are);
    // in U a slot may instead hold 16 shared-expert rows (16 x Fs bf16)
    const int wbytes = (PHASE == SP_GATEUP ? 2 : 1) * (abytes + sbytes);
    const int act_off = ((PHASE == SP_UPROJ ? max(wbytes, 32 * Fs) : wbytes) + 127) & ~127;
    // reduction length and activation row stride (halves) inside a slot / the CTA buffer
    const int KR = PHASE == SP_DPROJ ? H : PHASE == SP_GATEUP ? L : PHASE == SP_DOWN ? F : L;
    const int ld = (PHASE == SP_DOWN) ? F : KR + kActPad;

    if (warp == kSW) {
        // ---------------------------------------------------------------- loader
        if (lane == 0) {
            uint32_t last_ph[kMaxSlots];
            for (int s = 0; s < kMaxSlots; ++s) last_ph[s] = 0xFFFFFFFFu;
            bool x_issued = false;
            if (PHASE == SP_DPROJ && i0 < i1) {
                mbar_arrive_expect_tx(&xbar, (uint32_t)T * H * 2);
                for (int t = 0; t < T; ++t)
                    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                                 ::"r"(smem_u32(smem + (size_t)t * (H + kActPad) * 2)), "l"(p.x16 + (size_t)t * H),
                                 "r"(H * 2), "r"(smem_u32(&xbar)) : "memory");
                x_issued = true;
            }
            // Copies of item i into slot s: the weights (which depend on the
            // routing only) and / or the activations (written by the
            // previous kernel).
            auto issue = [&](int i, int s, bool weights, bool acts) {
                const Item item = stream_item<PHASE>(sh, tiles, i);
                uint8_t* slot = slots + (size_t)s * slot_bytes;
                uint8_t* act = slot + act_off;
                SlotMeta& m = meta[s];
                auto bulk = [&](void* dst, const void* src, uint32_t nb) {
                    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                                 ::"r"(smem_u32(dst)), "l"(src), "r"(nb), "r"(smem_u32(&full[s])) : "memory");
                };
                auto tma3 = [&](void* dst, const CUtensorMap* mp, int c0, int c2) {
                    asm volatile(
                        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
                        "[%0], [%1, {%3, %4, %5}], [%2];"
                        ::"r"(smem_u32(dst)), "l"(mp), "r"(smem_u32(&full[s])), "r"(c0), "r"(0), "r"(c2)
                        : "memory");
                };
                int nact = T;
                if (PHASE == SP_GATEUP || PHASE == SP_DOWN) nact = sh.ucnt[item.j];
                if (weights) {
                    m.item = item;
                    m.nt = nact;
                    m.off = (PHASE == SP_GATEUP || PHASE == SP_DOWN) ? sh.uoff[item.j] : 0;
                    // one expect-tx for everything the slot will receive
                    uint32_t bytes;
                    if (PHASE == SP_UPROJ && item.kind == 1) bytes = 16 * Fs * 2 + T * Fs * 2;
                    else if (PHASE == SP_GATEUP) bytes = wbytes + 16 + nact * L * 2;
                    else if (PHASE == SP_DOWN) bytes = wbytes + 16 + nact * F * 2;
                    else if (PHASE == SP_UPROJ) bytes = wbytes + T * L * 2;
                    else bytes = wbytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    if (PHASE == SP_UPROJ && item.kind == 1) {
                        bulk(slot, p.sd + (size_t)item.r0 * Fs, 16 * Fs * 2);
                    } else {
                        const int cq = item.r0 * maps.q_row, cs = item.r0 * maps.s_row;
                        tma3(slot, &maps.wq, cq, item.mat);
                        tma3(slot + abytes, &maps.ws, cs, item.mat);
                        if (PHASE == SP_GATEUP || PHASE == SP_DOWN) {
                            const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
                            bulk(m.tail, p.experts + (size_t)item.mat * p.rec_bytes + 3 * nq + 3 * ns, 16);
                        }
                        if (PHASE == SP_GATEUP) {
                            tma3(slot + abytes + sbytes, &maps.wq2, cq, item.mat);
                            tma3(slot + 2 * abytes + sbytes, &maps.ws2, cs, item.mat);
                        }
                    }
                }
                if (acts) {
                    if (PHASE == SP_UPROJ && item.kind == 1) {
                        bulk(act, p.zsh16, T * Fs * 2);
                    } else if (PHASE == SP_GATEUP) {
                        const int off = sh.uoff[item.j], g = sh.ugrp[item.j];
                        for (int c = 0; c < nact; ++c)
                            bulk(act + (size_t)c * ld * 2, p.h16 + ((size_t)sh.slot_tok[off + c] * G + g) * L, L * 2);
                    } else if (PHASE == SP_DOWN) {
                        bulk(act, p.z16 + (size_t)sh.uoff[item.j] * F, nact * F * 2);
                    } else if (PHASE == SP_UPROJ) {
                        for (int t = 0; t < T; ++t)
                            bulk(act + (size_t)t * ld * 2, p.s16 + ((size_t)t * G + item.mat) * L, L * 2);
                    }
                }
            };
            // the first ring's worth of weights streams before the previous
            // kernel has finished
            const int n_pre = PHASE == SP_DPROJ ? 0 : min(n_slots, i1 - i0);
            for (int k = 0; k < n_pre; ++k) {
                issue(i0 + k, k, true, false);
                last_ph[k] = 0;
            }
            if (PHASE != SP_DPROJ) {
                grid_dep_wait();
                grid_dep_launch();
            }
            for (int k = 0; k < n_pre; ++k) issue(i0 + k, k, false, true);
            int it = n_pre;
            for (int i = i0 + n_pre; i < i1; ++i, ++it) {
                const int s = it % n_slots;
                const uint32_t ph = (it / n_slots) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, &abort_flag, kStreamWait)) break;
                issue(i, s, true, true);
                last_ph[s] = ph;
            }
            if (abort_flag) {
                // let every copy already issued land before the CTA can leave
                int dummy = 0;
                for (int s = 0; s < n_slots; ++s)
                    if (last_ph[s] != 0xFFFFFFFFu) mbar_wait(&full[s], last_ph[s], &dummy, kStreamWait);
                if (x_issued) mbar_wait(&xbar, 0, &dummy, kStreamWait);
            }
        }
        __syncwarp();
    } else if (warp < kSW) {
        // ---------------------------------------------------------------- compute warps
        if (PHASE != SP_DPROJ) {
            grid_dep_wait();
            grid_dep_launch();
        }
        if (PHASE == SP_DPROJ && i0 < i1 && !mbar_wait(&xbar, 0, &abort_flag, kStreamWait)) goto done;
        {
            int it = 0;
            for (int i = i0; i < i1; ++i, ++it) {
                const int s = it % n_slots;
                const uint32_t ph = (it / n_slots) & 1;
                if (!mbar_wait(&full[s], ph, &abort_flag, kStreamWait)) break;
                const SlotMeta m = meta[s];
                const uint8_t* slot = slots + (size_t)s * slot_bytes;
                const uint8_t* act = slot + act_off;
                const __half* xs = PHASE == SP_DPROJ ? reinterpret_cast<const __half*>(smem) : reinterpret_cast<const __half*>(act);
                const int nt = m.nt;
                float a[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
                if (PHASE == SP_DPROJ || (PHASE == SP_UPROJ && m.item.kind == 0)) {
                    const int nb = KR / 32, per = (nb + kSW - 1) / kSW;
                    tile_du<FMT>(slot, reinterpret_cast<const uint16_t*>(slot + abytes), xs, ld, nt, warp * per,
                                 min(nb, (warp + 1) * per), a);
                } else if (PHASE == SP_UPROJ) {
                    const int nb = Fs / 32, per = (nb + kSW - 1) / kSW;
                    tile_bf16(reinterpret_cast<const uint16_t*>(slot), Fs, xs, Fs, nt, warp * per,
                              min(nb, (warp + 1) * per), a);
                } else {
                    const int nc = KR / 32, per = (nc + kSW - 1) / kSW;
                    tile_nvfp4(slot, slot + abytes, xs, ld, nt, warp * per, min(nc, (warp + 1) * per), a);
                    if (PHASE == SP_GATEUP)
                        tile_nvfp4(slot + abytes + sbytes, slot + 2 * abytes + sbytes, xs, ld, nt, warp * per,
                                   min(nc, (warp + 1) * per), u);
                }
                // every read of the slot is complete (the values are in registers)
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                const int b = it & 1;
                if (!mbar_wait(&red_empty[b], ((it >> 1) & 1) ^ 1, &abort_flag, kStreamWait)) break;
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    red[b][warp][lane][i4] = a[i4];
                    if (NV == 8) red[b][warp][lane][(4 + i4) % NV] = u[i4];
                }
                if (warp == 0 && lane == 0) red_meta[b] = m;
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_full[b]);
            }
        }
    } else {
        // ---------------------------------------------------------------- reducer + epilogue
        if (PHASE != SP_DPROJ) {
            grid_dep_wait();
            grid_dep_launch();
        }
        const int gg = lane >> 2, tt = lane & 3;
        float yacc[4] = {0.f, 0.f, 0.f, 0.f};   // U: running sum over the parts of one output tile
        int seg_first = -1;                      // U: first part of the current run in this CTA
        int it = 0;
        for (int i = i0; i < i1; ++i, ++it) {
            const int b = it & 1;
            if (!mbar_wait(&red_full[b], (it >> 1) & 1, &abort_flag, kStreamWait)) break;
            float a[4], u[4];
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                float sa = 0.f, su = 0.f;
#pragma unroll
                for (int w = 0; w < kSW; ++w) {
                    sa += red[b][w][lane][i4];
                    if (NV == 8) su += red[b][w][lane][(4 + i4) % NV];
                }
                a[i4] = sa;
                u[i4] = su;
            }
            const SlotMeta m = red_meta[b];
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty[b]);
            const Item item = m.item;
            const int nt = m.nt;
            if (PHASE != SP_UPROJ) {
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const int col = 2 * tt + (i4 & 1), row = item.r0 + gg + 8 * (i4 >> 1);
                    if (col >= nt) continue;
                    if (PHASE == SP_DPROJ) {
                        p.h16[((size_t)col * G + item.mat) * L + row] = __float2half_rn(a[i4]);
                    } else if (PHASE == SP_GATEUP) {
                        p.z16[(size_t)(m.off + col) * F + row] =
                            __float2half_rn(silu(a[i4] * m.tail[0]) * (u[i4] * m.tail[1]));
                    } else {
                        p.o16w[(size_t)(m.off + col) * L + row] =
                            __float2half_rn(sh.slot_w[m.off + col] * m.tail[2] * a[i4]);
                    }
                }
                continue;
            }
            // U: accumulate the parts of this tile that run consecutively here
            const int parts = sh.n_hit + 1;
            if (seg_first < 0) seg_first = item.j;
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) yacc[i4] += a[i4];
            const bool tile_end = item.j == parts - 1;
            if (!tile_end && i + 1 < i1) continue;
            const int tile = item.r0 / 16;
            const bool whole = seg_first == 0 && tile_end;
            if (whole) {
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const int col = 2 * tt + (i4 & 1), row = item.r0 + gg + 8 * (i4 >> 1);
                    if (col >= T) continue;
                    float v = yacc[i4];
                    if (p.residual) v += bf16_bits_to_f32(p.residual[(size_t)col * H + row]);
                    p.y[(size_t)col * H + row] = f32_to_bf16_bits(v);
                }
            } else {
                // this CTA holds parts [seg_first, item.j] of the tile: park
                // the partial sum under its first part; the CTA completing
                // the tile's parts adds the partials in part order
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const int col = 2 * tt + (i4 & 1), row = item.r0 + gg + 8 * (i4 >> 1);
                    if (col < T) p.ypart[((size_t)seg_first * T + col) * H + row] = yacc[i4];
                }
                __threadfence();
                __syncwarp();
                int last = 0;
                if (lane == 0) {
                    const int n_mine = item.j - seg_first + 1;
                    last = atomicAdd(&p.ctrl->tile_ticket[tile], n_mine) + n_mine == parts;
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
                    const int base = tile * parts;
                    for (int e2 = lane; e2 < T * 16; e2 += 32) {
                        const int t = e2 >> 4, row = item.r0 + (e2 & 15);
                        float v = 0.f;
                        for (int q = 0; q < parts; ++q) {
                            // q starts a run iff it starts the tile or some CTA's chunk
                            const int gi = base + q;
                            const int c = (int)(((long long)gi * gridDim.x + n_items - 1) / n_items);
                            if (q == 0 || chunk_begin(c, n_items, gridDim.x) == gi)
                                v += __ldcg(p.ypart + ((size_t)q * T + t) * H + row);
                        }
                        if (p.residual) v += bf16_bits_to_f32(p.residual[(size_t)t * H + row]);
                        p.y[(size_t)t * H + row] = f32_to_bf16_bits(v);
                    }
                    if (lane == 0) p.ctrl->tile_ticket[tile] = 0;
                }
            }
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) yacc[i4] = 0.f;
            seg_first = -1;
        }
    }
done:
    __syncthreads();
    if (abort_flag && threadIdx.x == 0) set_status(p.ctrl, LMOE_ERR_TIMEOUT);
}

// s16[t][g] = sum over the token's experts of group g of o16w (zero if none)
__global__ void k_combine_small(FwdParams p) {
    const int t = blockIdx.y, g = blockIdx.x;
    const int L = p.L, K = p.K;
    __shared__ int slots[kMaxTopK];
    __shared__ int n;
    grid_dep_wait();
    grid_dep_launch();
    if (threadIdx.x == 0) {
        int c = 0;
        for (int k = 0; k < K; ++k) {
            const int e = __ldcg(p.r.idx + t * K + k);
            if (p.group[e] == g) slots[c++] = __ldcg(p.r.pair_slot + t * K + k);
        }
        n = c;
    }
    __syncthreads();
    for (int c8 = threadIdx.x; c8 < L / 8; c8 += blockDim.x) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int i = 0; i < n; ++i) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.o16w + (size_t)slots[i] * L) + c8);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[j]));
                acc[2 * j] += f.x;
                acc[2 * j + 1] += f.y;
            }
        }
        __half2 h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = __floats2half2_rn(acc[2 * j], acc[2 * j + 1]);
        reinterpret_cast<uint4*>(p.s16 + ((size_t)t * p.G + g) * L)[c8] = *reinterpret_cast<uint4*>(h);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeFn encode() {
    static EncodeFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(ptr);
    }
    return fn;
}

// 3-D tensor of 16-bit units: (row_u16 * rows: one K block, contiguous;
// blocks; matrices), strides in bytes; the box is (row_u16 * 16, blocks, 1).
static bool map3(CUtensorMap* m, const void* base, uint64_t row_u16, uint64_t rows, uint64_t blocks,
                 uint64_t mats, uint64_t s_blk, uint64_t s_mat) {
    EncodeFn fn = encode();
    if (!fn || row_u16 * 16 > 256 || blocks > 256) return false;
    cuuint64_t dims[3] = {row_u16 * rows, blocks, mats};
    cuuint64_t strides[2] = {s_blk, s_mat};
    cuuint32_t box[3] = {(cuuint32_t)(row_u16 * 16), (cuuint32_t)blocks, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int g_sms = 0;

// Launch with programmatic stream serialisation: the kernel may start while
// its predecessor in the stream is still running; it orders itself with
// grid_dep_wait.
template <typename Kern, typename... Args>
static cudaError_t launch_dependent(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <int PHASE, int FMT>
static cudaError_t launch_stream(const StreamMaps& maps, const FwdParams& p, cudaStream_t st, int slot_bytes,
                                 int xs_bytes) {
    // dynamic shared memory: what the device allows per block minus the kernel's static part
    static size_t budget = 0;   // per kernel instance
    if (!budget) {
        cudaFuncAttributes fa;
        int dev = 0, optin = 0;
        cudaError_t e0 = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(k_stream<PHASE, FMT>));
        if (e0 == cudaSuccess) e0 = cudaGetDevice(&dev);
        if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e0 != cudaSuccess) return e0;
        budget = (size_t)optin - fa.sharedSizeBytes - 1024;
    }
    const int n_slots = (int)std::min<size_t>(16, (budget - xs_bytes) / slot_bytes);
    if (n_slots < 2) return cudaErrorInvalidValue;
    const size_t smem = 128 + xs_bytes + (size_t)n_slots * slot_bytes;
    auto kern = k_stream<PHASE, FMT>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    if (!g_sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    stage_mark(st);
    return launch_dependent(kern, dim3(g_sms), dim3(kStreamThreads), smem, st, maps, p, n_slots, slot_bytes);
}



struct StreamMapSet {
    StreamMaps d, gu, dn, u;
};

// Encode the four phases' tensor maps of one layer's weights.
static bool encode_stream_maps(const FwdParams& p, StreamMapSet* out) {
    const int H = p.H, L = p.L, F = p.F, G = p.G, E = p.E;
    const size_t qb = p.du_fmt == LMOE_Q8_0 ? 32 : 16;
    const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
    const uint8_t* ex = p.experts;
    StreamMaps& md = out->d;
    StreamMaps& mgu = out->gu;
    StreamMaps& mdn = out->dn;
    StreamMaps& mu = out->u;
    std::memset(out, 0, sizeof(*out));
    bool ok = true;
    const int qr = (int)qb / 2;
    // D: q [H/32][L][qb] + d [H/32][L] fp16 per group
    ok &= map3(&md.wq, p.D, qr, L, H / 32, G, (uint64_t)L * qb, p.du_bytes_D);
    ok &= map3(&md.ws, p.D + (size_t)L * H / 32 * qb, 1, L, H / 32, G, (uint64_t)L * 2, p.du_bytes_D);
    md.q_row = qr; md.s_row = 1;
    // U: q [L/32][H][qb] + d [L/32][H]; the shared expert's down rows are plain copies
    ok &= map3(&mu.wq, p.U, qr, H, L / 32, G, (uint64_t)H * qb, p.du_bytes_U);
    ok &= map3(&mu.ws, p.U + (size_t)H * L / 32 * qb, 1, H, L / 32, G, (uint64_t)H * 2, p.du_bytes_U);
    mu.q_row = qr; mu.s_row = 1;
    // experts: gate/up q [L/32][F][16], s [L/64][F][4]; down q [F/32][L][16], s [F/64][L][4]
    ok &= map3(&mgu.wq, ex, 8, F, L / 32, E, (uint64_t)F * 16, p.rec_bytes);
    ok &= map3(&mgu.wq2, ex + nq, 8, F, L / 32, E, (uint64_t)F * 16, p.rec_bytes);
    ok &= map3(&mgu.ws, ex + 3 * nq, 2, F, L / 64, E, (uint64_t)F * 4, p.rec_bytes);
    ok &= map3(&mgu.ws2, ex + 3 * nq + ns, 2, F, L / 64, E, (uint64_t)F * 4, p.rec_bytes);
    mgu.q_row = 8; mgu.s_row = 2;
    ok &= map3(&mdn.wq, ex + 2 * nq, 8, L, F / 32, E, (uint64_t)L * 16, p.rec_bytes);
    ok &= map3(&mdn.ws, ex + 3 * nq + 2 * ns, 2, L, F / 64, E, (uint64_t)L * 4, p.rec_bytes);
    mdn.q_row = 8; mdn.s_row = 2;
    return ok;
}

// The maps depend only on the weight pointers and the shape, so each layer's
// set is encoded once and kept (a small round-robin cache; a stack of layers
// cycles through it).
static bool stream_maps_for(const FwdParams& p, StreamMapSet* out) {
    struct Key {
        const void *D, *U, *ex;
        int H, L, F, G, E, fmt;
        size_t bd, bu, br;
        bool operator==(const Key& o) const { return std::memcmp(this, &o, sizeof(Key)) == 0; }
    };
    constexpr int kCache = 64;
    static Key keys[kCache];
    static StreamMapSet sets[kCache];
    static int n = 0, next = 0;
    static std::mutex mu;
    Key k;
    std::memset(&k, 0, sizeof(k));
    k.D = p.D; k.U = p.U; k.ex = p.experts;
    k.H = p.H; k.L = p.L; k.F = p.F; k.G = p.G; k.E = p.E; k.fmt = p.du_fmt;
    k.bd = p.du_bytes_D; k.bu = p.du_bytes_U; k.br = p.rec_bytes;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (keys[i] == k) {
            *out = sets[i];
            return true;
        }
    if (!encode_stream_maps(p, out)) return false;
    keys[next] = k;
    sets[next] = *out;
    next = (next + 1) % kCache;
    if (n < kCache) ++n;
    return true;
}

// D, experts, combine, U for T <= 8 (the router kernel has run).
cudaError_t run_stream_path(const FwdParams& p, cudaStream_t st) {
    const int H = p.H, L = p.L, F = p.F, Fs = p.Fs, G = p.G;
    const size_t qb = p.du_fmt == LMOE_Q8_0 ? 32 : 16;
    StreamMapSet ms;
    if (!stream_maps_for(p, &ms)) return cudaErrorInvalidValue;
    const StreamMaps& md = ms.d;
    const StreamMaps& mgu = ms.gu;
    const StreamMaps& mdn = ms.dn;
    const StreamMaps& mu = ms.u;

    const int act_d = 0;
    const int slot_d = round128(16 * H * (int)qb / 32 + 16 * (H / 32) * 2);
    // activation rows per slot: at most T (an expert sees each token once)
    const int T = p.T;
    const int slot_gu = round128(round128(2 * (16 * L / 2 + 16 * (L / 64) * 4)) + T * (L + kActPad) * 2);
    const int slot_dn = round128(round128(16 * F / 2 + 16 * (F / 64) * 4) + T * F * 2);
    const int slot_u = round128(round128(std::max(16 * L * (int)qb / 32 + 16 * (L / 32) * 2, 32 * Fs)) +
                                T * std::max(L + kActPad, Fs) * 2);
    (void)act_d;
    cudaError_t e;
    const int xs_d = round128(T * (H + kActPad) * 2);
    e = p.du_fmt == LMOE_Q8_0 ? launch_stream<SP_DPROJ, LMOE_Q8_0>(md, p, st, slot_d, xs_d)
                              : launch_stream<SP_DPROJ, LMOE_Q4_0>(md, p, st, slot_d, xs_d);
    if (e != cudaSuccess) return e;
    e = launch_stream<SP_GATEUP, LMOE_Q8_0>(mgu, p, st, slot_gu, 0);
    if (e != cudaSuccess) return e;
    e = launch_stream<SP_DOWN, LMOE_Q8_0>(mdn, p, st, slot_dn, 0);
    if (e != cudaSuccess) return e;
    stage_mark(st);
    if ((e = launch_dependent(k_combine_small, dim3(G, p.T), dim3(128), 0, st, p)) != cudaSuccess) return e;
    e = p.du_fmt == LMOE_Q8_0 ? launch_stream<SP_UPROJ, LMOE_Q8_0>(mu, p, st, slot_u, 0)
                              : launch_stream<SP_UPROJ, LMOE_Q4_0>(mu, p, st, slot_u, 0);
    return e;
}

}  // namespace lmoe
