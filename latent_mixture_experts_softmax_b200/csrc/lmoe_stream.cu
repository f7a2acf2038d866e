// Few-token path (T <= 8), weight-streaming kernels.  One CTA per SM, 16
// warps.  A work item is one 16-row tile of one matrix over its reduction
// (K), in steps of a few stored K blocks.  Items are split into contiguous
// chunks per CTA, and a chunk's steps into equal contiguous ranges per warp;
// each warp streams its range's stored bytes (codes and scales exactly as
// they sit in HBM) through its own ring of shared-memory step buffers with
// per-thread asynchronous copies (cp.async, 16 bytes per thread; the
// bulk-copy engine's fixed cost per copy would cap the rate), dequantises in
// registers and multiplies on the tensor pipe (mma.sync m16n8k16, fp16
// operands, fp32 accumulation; the 8 MMA columns are the up to 8 tokens).
// The activations of a chunk are read once into a shared-memory cache.  An
// item cut by warp ranges is summed in shared memory, in K order; U's output
// tiles, whose items (hit groups and the shared expert) sit in different
// CTAs, meet in the workspace, and the warp that completes a tile (ticket)
// adds the parts in order and runs the epilogue.
//
//   k_wstream<DPROJ>   h16[t][g]   = D_g x_t            (every group)
//   k_wstream<GATEUP>  z16[slot]   = silu(W_gate h) * (W_up h)
//   k_wstream<DOWN>    o16w[slot]  = w_slot * W_down z
//   k_wstream<UPROJ>   y           = sum_g U_g s[g][t] + S_down z_sh (+ residual), where
//                      s[g][t] = sum of o16w over token t's experts in group g is formed
//                      while the CTA fills its activation cache
//
// Method: teardown article "Edge0-145B: a Qwen MoE with its experts
// squeezed", section "A latent in front of the experts" (layer equation,
// per-group D/U); Edge0 145B / 120B model page, architecture tables.

#include <algorithm>
#include <cstdlib>
#include <cstring>


#include "lmoe_internal.cuh"
#include "lmoe_q3k.cuh"
#include "lmoe_route.cuh"
#include "lmoe_sm100.cuh"

namespace lmoe {

using namespace sm100;

enum StreamPhase { SP_DPROJ = 0, SP_GATEUP = 1, SP_DOWN = 2, SP_UPROJ = 3 };

// The format parameter of the phase templates: the D/U format (LMOE_Q8_0 /
// LMOE_Q4_0) for D and U, the expert format for gate/up and down.
constexpr int kEfNvfp4 = LMOE_EXPERTS_NVFP4;
constexpr int kEfQ3k = LMOE_EXPERTS_Q3K;

constexpr int kWW = 16;                     // warps per CTA
constexpr int kWThreads = 32 * kWW;
constexpr int kPD = 3;                      // step buffers per warp (2 steps in flight)
constexpr int kStepBytes = 2304;            // largest step (see step_geom)
constexpr int kMaxChunkParts = 8;           // distinct matrices in one CTA's chunk
constexpr int kActPad = 32;                 // halves of padding per cached activation row

__host__ __device__ __forceinline__ int round128(int b) { return (b + 127) & ~127; }

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

// Four E4M3 scales (one stored word) -> two f16x2: bytes 0, 1 and bytes 2, 3.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// One 32-column NVFP4 chunk c of a 16-row tile: codes [chunk][16 rows][16 B];
// sg / sh are the lane's E4M3 scales of rows g and g + 8 as f16x2 (both
// halves equal), folded into the fp16 operand (exact); the tensor scale is
// left to the caller.
__device__ __forceinline__ void nvfp4_chunk_scaled(const uint8_t* q, const __half* xs, int ld, int nt, int c,
                                                   uint32_t sg, uint32_t sh, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t wg = *reinterpret_cast<const uint32_t*>(q + ((size_t)c * 16 + g) * 16 + 4 * t);
    const uint32_t wh = *reinterpret_cast<const uint32_t*>(q + ((size_t)c * 16 + g + 8) * 16 + 4 * t);
    uint32_t a[4], b[4];
    e2m1x8_to_f16x8(wg, a);
    e2m1x8_to_f16x8(wh, b);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        a[j] = hmul2u(a[j], sg);
        b[j] = hmul2u(b[j], sh);
    }
    const uint4 xv = act8(xs, ld, g, nt, c * 32 + 8 * t);
    mma16816s(acc, a[0], b[0], a[1], b[1], xv.x, xv.y);
    mma16816s(acc, a[2], b[2], a[3], b[3], xv.z, xv.w);
}

// One 16-row NVFP4 tile in shared memory (codes [chunk][16 rows][16 B],
// scales [chunk/2][16 rows][4 B]: byte j of a row's word scales its 16-column
// block j of the chunk pair), chunks [0, c1).  Chunks go in pairs (even,
// odd) that share one scale word per row, converted once; lane t's columns
// 8t..8t+7 of a chunk lie in the pair's block t/2 (even chunk) or 2 + t/2
// (odd chunk).  Even and odd chunks accumulate separately so that
// consecutive MMAs do not wait on each other; the two sums are added at the
// end.
__device__ __forceinline__ void tile_nvfp4(const uint8_t* q, const uint8_t* s, const __half* xs, int ld, int nt,
                                           int c1, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t sel = (t >> 1) ? 0x3232u : 0x1010u;   // duplicate the high / low half
    float acc2[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < c1; c += 2) {
        const uint32_t swg = *reinterpret_cast<const uint32_t*>(s + ((size_t)(c >> 1) * 16 + g) * 4);
        const uint32_t swh = *reinterpret_cast<const uint32_t*>(s + ((size_t)(c >> 1) * 16 + g + 8) * 4);
        uint32_t g01, g23, h01, h23;
        e4m3x4_to_f16x2x2(swg, g01, g23);
        e4m3x4_to_f16x2x2(swh, h01, h23);
        nvfp4_chunk_scaled(q, xs, ld, nt, c, __byte_perm(g01, 0u, sel), __byte_perm(h01, 0u, sel), acc);
        if (c + 1 < c1)
            nvfp4_chunk_scaled(q, xs, ld, nt, c + 1, __byte_perm(g23, 0u, sel), __byte_perm(h23, 0u, sel), acc2);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] += acc2[j];
}

// 16 rows of bf16 weights ([16][K] row-major) against fp16 activations,
// 32-column blocks [b0, b1); bf16 -> fp16 in registers (a weight outside the
// fp16 range is flagged in `bad`).
__device__ __forceinline__ void tile_bf16(const uint16_t* w, int K, const __half* xs, int ld, int nt, int b0, int b1,
                                          float (&acc)[4], bool& bad) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll 2
    for (int b = b0; b < b1; ++b) {
        const uint4 wg = *reinterpret_cast<const uint4*>(w + (size_t)g * K + 32 * b + 8 * t);
        const uint4 wh = *reinterpret_cast<const uint4*>(w + (size_t)(g + 8) * K + 32 * b + 8 * t);
        auto cv = [&bad](uint32_t v) {
            const float2 f = bf16x2_to_f32x2(v);
            __half2 h = half2_checked(f.x, f.y, bad);
            return *reinterpret_cast<uint32_t*>(&h);
        };
        const uint4 xv = act8(xs, ld, g, nt, 32 * b + 8 * t);
        mma16816s(acc, cv(wg.x), cv(wh.x), cv(wg.y), cv(wh.y), xv.x, xv.y);
        mma16816s(acc, cv(wg.z), cv(wh.z), cv(wg.w), cv(wh.w), xv.z, xv.w);
    }
}


// The IQ4_NL byte -> (level of the low nibble, level of the high nibble)
// table of the CTA (fp16 pairs), filled at kernel start.
__device__ __forceinline__ uint32_t* iq4nl_lut() {
    __shared__ uint32_t lut[256];
    return lut;
}

// One 128-column half of a 16-row Q3_K tile in shared memory (planes lo
// [16][32], hi [16][16], sc [16][6], d [16] fp16) times the activations at
// columns [0, 128) of xs.  Sub-block j is one k16 MMA: lane t takes the
// elements 16j + 4t .. 16j + 4t + 3 of rows g and g + 8, whose code bits sit
// in bits 2t.. of lo word j and bits 4(j & 1) + t of hi word j / 2; the
// operand is (q - 4) * (sc_j - 32), an integer of at most 128 (exact in
// fp16); the super-block scale d multiplies the step's sum.
__device__ __forceinline__ void tile_q3k_half(const uint8_t* m, const __half* xs, int ld, int nt, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint8_t* lo = m;
    const uint8_t* hi = m + 512;
    const uint8_t* sc = m + 768;
    const uint16_t* dd = reinterpret_cast<const uint16_t*>(m + 864);
    auto sc48 = [&](int row) {
        const uint16_t* p16 = reinterpret_cast<const uint16_t*>(sc + row * 6);
        return (uint64_t)p16[0] | ((uint64_t)p16[1] << 16) | ((uint64_t)p16[2] << 32);
    };
    const uint64_t sg = sc48(g), sh = sc48(g + 8);
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t lg = *reinterpret_cast<const uint32_t*>(lo + g * 32 + 4 * j);
        const uint32_t lh = *reinterpret_cast<const uint32_t*>(lo + (g + 8) * 32 + 4 * j);
        const uint32_t hg = *reinterpret_cast<const uint32_t*>(hi + g * 16 + 4 * (j >> 1));
        const uint32_t hh = *reinterpret_cast<const uint32_t*>(hi + (g + 8) * 16 + 4 * (j >> 1));
        const int hs = 4 * (j & 1) + t;
        const uint32_t qg = ((lg >> (2 * t)) & 0x03030303u) | (((hg >> hs) & 0x01010101u) << 2);
        const uint32_t qh = ((lh >> (2 * t)) & 0x03030303u) | (((hh >> hs) & 0x01010101u) << 2);
        const __half2 fg = __half2half2(__int2half_rn((int)((sg >> (6 * j)) & 63) - 32));
        const __half2 fh = __half2half2(__int2half_rn((int)((sh >> (6 * j)) & 63) - 32));
        auto op = [](uint32_t q, uint32_t sel, __half2 f) {
            uint32_t v = hsub2u(__byte_perm(q, 0x64646464u, sel), 0x64046404u);     // (q - 4) pairs
            return hmul2u(v, *reinterpret_cast<const uint32_t*>(&f));
        };
        const uint2 xv = g < nt ? *reinterpret_cast<const uint2*>(xs + (size_t)g * ld + 16 * j + 4 * t)
                                : make_uint2(0, 0);
        mma16816s(c, op(qg, 0x4140u, fg), op(qh, 0x4140u, fh), op(qg, 0x4342u, fg), op(qh, 0x4342u, fh), xv.x, xv.y);
    }
    const float dg = __half2float(__ushort_as_half(dd[g])), dh = __half2float(__ushort_as_half(dd[g + 8]));
    acc[0] = fmaf(dg, c[0], acc[0]);
    acc[1] = fmaf(dg, c[1], acc[1]);
    acc[2] = fmaf(dh, c[2], acc[2]);
    acc[3] = fmaf(dh, c[3], acc[3]);
}

// A 16-row IQ4_NL tile in shared memory (codes [block][16 rows][16 B], d
// [block][16 rows] fp16), blocks [0, b1): as Q4_0 with the level table in
// place of q - 8 (lane t: elements 4t..4t+3 from the low nibbles of its
// 4 bytes, 16 + 4t.. from the high ones).
__device__ __forceinline__ void tile_iq4nl(const uint8_t* q, const uint16_t* d, const __half* xs, int ld, int nt,
                                           int b1, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t* lut = iq4nl_lut();
#pragma unroll 2
    for (int b = 0; b < b1; ++b) {
        const uint32_t wg = *reinterpret_cast<const uint32_t*>(q + ((size_t)b * 16 + g) * 16 + 4 * t);
        const uint32_t wh = *reinterpret_cast<const uint32_t*>(q + ((size_t)b * 16 + g + 8) * 16 + 4 * t);
        const uint32_t g0 = lut[wg & 0xFF], g1 = lut[(wg >> 8) & 0xFF], g2 = lut[(wg >> 16) & 0xFF], g3 = lut[wg >> 24];
        const uint32_t h0 = lut[wh & 0xFF], h1 = lut[(wh >> 8) & 0xFF], h2 = lut[(wh >> 16) & 0xFF], h3 = lut[wh >> 24];
        const uint2 xl = act4(xs, ld, g, nt, 32 * b + 4 * t);
        const uint2 xh = act4(xs, ld, g, nt, 32 * b + 16 + 4 * t);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        mma16816s(c, __byte_perm(g0, g1, 0x5410), __byte_perm(h0, h1, 0x5410), __byte_perm(g2, g3, 0x5410),
                  __byte_perm(h2, h3, 0x5410), xl.x, xl.y);
        mma16816s(c, __byte_perm(g0, g1, 0x7632), __byte_perm(h0, h1, 0x7632), __byte_perm(g2, g3, 0x7632),
                  __byte_perm(h2, h3, 0x7632), xh.x, xh.y);
        const float dg = __half2float(__ushort_as_half(d[b * 16 + g]));
        const float dh = __half2float(__ushort_as_half(d[b * 16 + g + 8]));
        acc[0] = fmaf(dg, c[0], acc[0]);
        acc[1] = fmaf(dg, c[1], acc[1]);
        acc[2] = fmaf(dh, c[2], acc[2]);
        acc[3] = fmaf(dh, c[3], acc[3]);
    }
}

// ---------------------------------------------------------------------------
// items, steps and parts
// ---------------------------------------------------------------------------

// K blocks (32 elements) per step and the step's byte layout:
//   D / U groups Q8_0: 4 blocks  codes [4][16][32] + scales [4][16] fp16 = 2176 B
//   D / U groups Q4_0: 8 blocks  codes [8][16][16] + scales [8][16] fp16 = 2304 B
//   gate/up NVFP4:     4 chunks  gate codes [4][16][16], up codes, gate scales [2][16][4], up scales = 2304 B
//   down NVFP4:        8 chunks  codes [8][16][16] + scales [4][16][4] = 2304 B
//   U shared bf16:     2 blocks  [16 rows][64] bf16 = 2048 B
//   D shared gate/up:  1 block   gate [16 rows][32] bf16, then up = 2048 B
template <int PHASE, int FMT>
__host__ __device__ __forceinline__ int step_blocks(bool shared_part) {
    if (PHASE == SP_GATEUP) return 4;
    if (PHASE == SP_DOWN) return 8;
    if (PHASE == SP_UPROJ && shared_part) return 2;
    if (PHASE == SP_DPROJ && shared_part) return 1;
    return FMT == LMOE_Q8_0 ? 4 : 8;
}

template <int PHASE>
__host__ __device__ __forceinline__ int stream_rows(int H, int L, int F) {
    return PHASE == SP_DPROJ ? L : PHASE == SP_GATEUP ? F : PHASE == SP_DOWN ? L : H;
}

// One decoded work item.
struct WItem {
    int mat;       // group (D, U), expert (gate/up, down); -1: the shared expert (U)
    int j;         // distinct-expert index (gate/up, down) / part index (U)
    int r0;        // first output row
    int tile;      // output tile index
    int q;         // reduction part
    int kb0, kb1;  // K blocks of the part
};

struct WPlan {
    int ks;        // reduction parts per tile (1: a tile's K is cut only between warps)
    int tiles;     // output tiles per matrix
    int n_mats;    // matrices (D: every group; experts; U: hit groups + shared)
};

// Items run matrix-major (consecutive items share a matrix, so a CTA's chunk
// touches few of them and caches few activation rows), then reduction part,
// then tile.
template <int PHASE, int FMT>
__device__ __forceinline__ WItem decode_item(const FwdParams& p, const StreamShared& sh, const WPlan& pl, int i) {
    WItem it;
    if (PHASE == SP_DPROJ && i >= p.G * pl.tiles) {
        // the shared expert's gate and up rows (16 features over the whole
        // block input), after every group's D items; one 32-column block per step
        it.mat = -1;
        it.j = p.G;
        it.q = 0;
        it.tile = i - p.G * pl.tiles;
        it.r0 = it.tile * 16;
        it.kb0 = 0;
        it.kb1 = p.H / 32;
        return it;
    }
    const int per_mat = pl.tiles * pl.ks;
    const int m = i / per_mat, rem = i - m * per_mat;
    it.q = rem / pl.tiles;
    it.tile = rem - it.q * pl.tiles;
    it.r0 = it.tile * 16;
    it.j = m;
    bool shared_part = false;
    int nb;
    if (PHASE == SP_DPROJ) {
        it.mat = m;                       // every group, in order
        nb = p.H / 32;
    } else if (PHASE == SP_UPROJ) {
        shared_part = m == sh.n_hit;
        it.mat = shared_part ? -1 : sh.hg[m];
        nb = shared_part ? p.Fs / 32 : p.L / 32;
    } else {
        it.mat = sh.uexp[m];
        nb = (PHASE == SP_GATEUP ? p.L : p.F) / 32;
    }
    const int sb = step_blocks<PHASE, FMT>(shared_part);
    const int ns = (nb + sb - 1) / sb;
    it.kb0 = min(nb, (it.q * ns / pl.ks) * sb);
    it.kb1 = min(nb, ((it.q + 1) * ns / pl.ks) * sb);
    return it;
}

// c * n stays far below 2^31 (at most 148 CTAs x a few thousand items)
__device__ __forceinline__ int chunk_begin(int c, int n, int ctas) { return (c * n) / ctas; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Issue the copies of step `st` of item `it` into `buf` (every lane).
template <int PHASE, int FMT>
__device__ __forceinline__ void issue_step(const FwdParams& p, const WItem& it, int st, uint8_t* buf, int lane) {
    const int L = p.L, F = p.F, H = p.H, Fs = p.Fs;
    const bool shared_part = (PHASE == SP_UPROJ || PHASE == SP_DPROJ) && it.mat < 0;
    const int sb = step_blocks<PHASE, FMT>(shared_part);
    const int kb = it.kb0 + st * sb;
    const int nblk = min(sb, it.kb1 - kb);
    if (PHASE == SP_DPROJ && shared_part) {
        // gate then up rows r0 .. r0 + 15, columns 32 kb .. + 31 (64 bytes a row)
        for (int c = lane; c < 128; c += 32) {
            const int mm = c >> 6, row = (c >> 2) & 15, o = (c & 3) * 16;
            const uint16_t* src = (mm ? p.su : p.sg) + (size_t)(it.r0 + row) * H + (size_t)kb * 32;
            cp_async16(buf + (size_t)mm * 1024 + row * 64 + o, reinterpret_cast<const uint8_t*>(src) + o);
        }
    } else if (PHASE == SP_DPROJ || (PHASE == SP_UPROJ && !shared_part)) {
        const int qb = FMT == LMOE_Q8_0 ? 32 : 16;
        const int R = PHASE == SP_DPROJ ? L : H;
        const int C = PHASE == SP_DPROJ ? H : L;
        const uint8_t* mat = (PHASE == SP_DPROJ ? p.D + (size_t)it.mat * p.du_bytes_D : p.U + (size_t)it.mat * p.du_bytes_U);
        const uint8_t* dsc = mat + (size_t)R * C / 32 * qb;
        const int cpb = qb;                 // 16-byte chunks of codes per block (16 rows x qb bytes / 16)
        const int n_codes = nblk * cpb, n_sc = nblk * 2;
        for (int c = lane; c < n_codes + n_sc; c += 32) {
            if (c < n_codes) {
                const int b = c / cpb, o = (c - b * cpb) * 16;
                cp_async16(buf + (size_t)c * 16, mat + ((size_t)(kb + b) * R + it.r0) * qb + o);
            } else {
                const int c2 = c - n_codes, b = c2 >> 1;
                cp_async16(buf + (size_t)sb * 16 * qb + (size_t)c2 * 16, dsc + ((size_t)(kb + b) * R + it.r0) * 2 + (c2 & 1) * 16);
            }
        }
    } else if (PHASE == SP_UPROJ) {
        // shared expert down rows [H][Fs] bf16: 16 rows x 64 columns per 2 blocks
        const int n = 16 * nblk * 4;        // 16-byte chunks: 4 per row per block
        for (int c = lane; c < n; c += 32) {
            const int row = c / (nblk * 4), o = (c - row * nblk * 4) * 16;
            cp_async16(buf + (size_t)row * 128 + o, reinterpret_cast<const uint8_t*>(p.sd + (size_t)(it.r0 + row) * Fs) + (size_t)kb * 64 + o);
        }
    } else if (FMT == kEfQ3k) {
        const uint8_t* rec = p.experts + (size_t)it.mat * p.rec_bytes;
        const size_t gb = q3k_matrix_bytes(F, L);
        if (PHASE == SP_GATEUP) {
            // one 128-column half h for gate and up: planes lo 512 | hi 256 | sc 96 | d 32 bytes each
            const int h = kb / 4;
            const size_t nh = (size_t)L / 128;
            for (int mm = 0; mm < 2; ++mm) {
                const uint8_t* m = rec + mm * gb;
                uint8_t* bm = buf + mm * 896;
                for (int c = lane; c < 56; c += 32) {
                    const uint8_t* src;
                    uint8_t* dst;
                    if (c < 32) {
                        src = m + ((size_t)h * F + it.r0) * 32 + c * 16;
                        dst = bm + c * 16;
                    } else if (c < 48) {
                        src = m + nh * F * 32 + ((size_t)h * F + it.r0) * 16 + (c - 32) * 16;
                        dst = bm + 512 + (c - 32) * 16;
                    } else if (c < 54) {
                        src = m + nh * F * 48 + ((size_t)h * F + it.r0) * 6 + (c - 48) * 16;
                        dst = bm + 768 + (c - 48) * 16;
                    } else {
                        src = m + nh * F * 54 + ((size_t)(h / 2) * F + it.r0) * 2 + (c - 54) * 16;
                        dst = bm + 864 + (c - 54) * 16;
                    }
                    cp_async16(dst, src);
                }
            }
        } else {
            // IQ4_NL down [L][F]: as the Q4_0 steps (8 blocks of 16 rows x 16 B, then the fp16 d)
            const uint8_t* mat = rec + 2 * gb;
            const uint8_t* dsc = mat + (size_t)L * F / 2;
            const int n_codes = nblk * 16, n_sc = nblk * 2;
            for (int c = lane; c < n_codes + n_sc; c += 32) {
                if (c < n_codes) {
                    const int b = c / 16, o = (c - b * 16) * 16;
                    cp_async16(buf + (size_t)c * 16, mat + ((size_t)(kb + b) * L + it.r0) * 16 + o);
                } else {
                    const int c2 = c - n_codes, b = c2 >> 1;
                    cp_async16(buf + (size_t)sb * 256 + (size_t)c2 * 16, dsc + ((size_t)(kb + b) * L + it.r0) * 2 + (c2 & 1) * 16);
                }
            }
        }
    } else {
        const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
        const uint8_t* rec = p.experts + (size_t)it.mat * p.rec_bytes;
        const int R = PHASE == SP_GATEUP ? F : L;
        const uint8_t* q0 = rec + (PHASE == SP_GATEUP ? 0 : 2 * nq);
        const uint8_t* s0 = rec + 3 * nq + (PHASE == SP_GATEUP ? 0 : 2 * ns);
        const int nmat = PHASE == SP_GATEUP ? 2 : 1;      // gate and up
        const int n_codes = nblk * 16, n_sc = ((nblk + 1) / 2) * 4;
        const int qbytes = sb * 256, sbytes = (sb / 2) * 64;
        for (int mm = 0; mm < nmat; ++mm) {
            const uint8_t* qm = q0 + mm * nq;
            const uint8_t* sm = s0 + mm * ns;
            uint8_t* bq = buf + mm * qbytes;
            uint8_t* bs = buf + nmat * qbytes + mm * sbytes;
            for (int c = lane; c < n_codes + n_sc; c += 32) {
                if (c < n_codes) {
                    const int b = c >> 4, o = (c & 15) * 16;
                    cp_async16(bq + (size_t)c * 16, qm + ((size_t)(kb + b) * R + it.r0) * 16 + o);
                } else {
                    const int c2 = c - n_codes, b = c2 >> 2;
                    cp_async16(bs + (size_t)c2 * 16, sm + ((size_t)(kb / 2 + b) * R + it.r0) * 4 + (c2 & 3) * 16);
                }
            }
        }
    }
}

// Multiply step `st` (in `buf`) with the item's activations.
template <int PHASE, int FMT>
__device__ __forceinline__ void compute_step(const FwdParams& p, const WItem& it, int st, const uint8_t* buf,
                                             const __half* xs, int ld, int nt, float (&a)[4], float (&u)[4]) {
    const bool shared_part = (PHASE == SP_UPROJ || PHASE == SP_DPROJ) && it.mat < 0;
    const int sb = step_blocks<PHASE, FMT>(shared_part);
    const int kb = it.kb0 + st * sb;
    const int nblk = min(sb, it.kb1 - kb);
    const __half* x = xs + kb * 32;
    if (PHASE == SP_DPROJ && shared_part) {
        bool bad = false;
        tile_bf16(reinterpret_cast<const uint16_t*>(buf), 32, x, ld, nt, 0, 1, a, bad);
        tile_bf16(reinterpret_cast<const uint16_t*>(buf + 1024), 32, x, ld, nt, 0, 1, u, bad);
        report_range(p.ctrl, bad);
    } else if (PHASE == SP_DPROJ || (PHASE == SP_UPROJ && !shared_part)) {
        const int qb = FMT == LMOE_Q8_0 ? 32 : 16;
        tile_du<FMT>(buf, reinterpret_cast<const uint16_t*>(buf + sb * 16 * qb), x, ld, nt, 0, nblk, a);
    } else if (PHASE == SP_UPROJ) {
        bool bad = false;
        tile_bf16(reinterpret_cast<const uint16_t*>(buf), 64, x, ld, nt, 0, nblk, a, bad);
        report_range(p.ctrl, bad);
    } else if (PHASE == SP_GATEUP && FMT == kEfQ3k) {
        tile_q3k_half(buf, x, ld, nt, a);
        tile_q3k_half(buf + 896, x, ld, nt, u);
    } else if (PHASE == SP_GATEUP) {
        tile_nvfp4(buf, buf + 2 * 1024, x, ld, nt, nblk, a);
        tile_nvfp4(buf + 1024, buf + 2 * 1024 + 128, x, ld, nt, nblk, u);
    } else if (FMT == kEfQ3k) {
        tile_iq4nl(buf, reinterpret_cast<const uint16_t*>(buf + sb * 256), x, ld, nt, nblk, a);
    } else {
        tile_nvfp4(buf, buf + 2048, x, ld, nt, nblk, a);
    }
}

template <int PHASE>
__device__ __forceinline__ int n_steps(const WItem& it, int sb) { return (it.kb1 - it.kb0 + sb - 1) / sb; }

// Steps of a phase's items in item order: items [0, nA) take nsA steps
// each, the others nsB (U: the hit groups' matrices, then the shared
// expert's); first(i) is item i's first step.  A CTA's steps are cut into
// equal contiguous ranges, one per warp, so every warp streams the same
// number of steps whatever the number of items.
struct StepMap {
    int nA, nsA, nsB;
    __device__ __forceinline__ int first(int i) const { return i <= nA ? i * nsA : nA * nsA + (i - nA) * nsB; }
    __device__ __forceinline__ int item(int st) const {
        const int sA = nA * nsA;
        return st < sA ? st / nsA : nA + (st - sA) / nsB;
    }
};

// ---------------------------------------------------------------------------
// one phase: chunk, activation cache, per-warp pipeline
// ---------------------------------------------------------------------------

// The chunk of items of one CTA and the activation rows of its matrices.
struct ChunkInfo {
    int i0, i1;                  // items [i0, i1)
    int m0, nm, rows, skip;      // first matrix, matrices, cached rows, refused
    int row0[kMaxChunkParts];    // first cache row of each matrix
    int src[kMaxChunkParts * 8]; // source of each cache row (phase-specific code)
    alignas(16) float tail[kMaxChunkParts][4];  // experts: tensor scales of gate, up, down
};

// One warp's load cursor over its range of steps.
struct LoadCursor {
    int st, s1;        // next step to issue, end of the range
    int j, j0, j1;     // its item, the item's first step and end
    int n_issued;
    WItem it;
};

template <int PHASE>
__host__ __device__ __forceinline__ int cache_ld(int H, int L, int F, int Fs) {
    return PHASE == SP_DPROJ ? H + kActPad : PHASE == SP_GATEUP ? L + kActPad : PHASE == SP_DOWN ? F + kActPad
                                                                                               : (L > Fs ? L : Fs) + kActPad;
}

// Matrices of a phase: D every group (it runs before or beside the routing),
// U the hit groups and the shared expert, the experts' phases the distinct
// experts.
template <int PHASE>
__device__ __forceinline__ int phase_mats(const FwdParams& p, const StreamShared& sh) {
    return PHASE == SP_DPROJ ? p.G : PHASE == SP_UPROJ ? sh.n_hit + 1 : sh.n_unique;
}

// Warp 0 decides the CTA's chunk and its cache rows (visible to all after
// the __syncthreads in here); threads < 4 * nm then fetch the experts'
// tensor scales (visible after the caller's next __syncthreads).
template <int PHASE, int FMT>
__device__ void phase_setup(const FwdParams& p, const StreamShared& sh, const WPlan& plan, int cache_bytes,
                            ChunkInfo& ci) {
    const int T = p.T, G = p.G;
    const int ld = cache_ld<PHASE>(p.H, p.L, p.F, p.Fs);
    if (threadIdx.x < 32) {
        // warp 0: every lane computes the chunk; lane jj lays out the cache
        // rows of the chunk's matrix jj (at most T rows each)
        const int lane = threadIdx.x;
        const int n_items = phase_mats<PHASE>(p, sh) * plan.tiles * plan.ks +
                            (PHASE == SP_DPROJ && p.shared_in_d ? p.Fs / 16 : 0);
        const int per_mat = plan.tiles * plan.ks;
        const int i0 = chunk_begin(blockIdx.x, n_items, gridDim.x);
        const int i1 = chunk_begin(blockIdx.x + 1, n_items, gridDim.x);
        const int m0 = i0 / per_mat, m1 = i0 < i1 ? (i1 - 1) / per_mat : m0 - 1;
        const int nm = PHASE == SP_DPROJ ? 1 : m1 - m0 + 1;
        const int m = m0 + lane;
        const bool act = lane < nm && lane < kMaxChunkParts;
        const int nr = act ? ((PHASE == SP_GATEUP || PHASE == SP_DOWN) ? sh.ucnt[m] : T) : 0;
        int pre = nr;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, pre, o);
            if (lane >= o) pre += v;
        }
        const int rows = __shfl_sync(0xffffffffu, pre, 31);
        const bool fits = nm <= kMaxChunkParts && rows <= kMaxChunkParts * 8 && (size_t)rows * ld * 2 <= (size_t)cache_bytes;
        if (act && fits) {
            const int r0 = pre - nr;
            ci.row0[lane] = r0;
            for (int c = 0; c < nr; ++c) {
                int src;
                if (PHASE == SP_DPROJ) src = c;                                                     // x row
                else if (PHASE == SP_GATEUP) src = sh.slot_tok[sh.uoff[m] + c] * G + sh.ugrp[m];  // h16 row
                else if (PHASE == SP_DOWN) src = sh.uoff[m] + c;                                    // z16 row
                else src = m < sh.n_hit ? sh.hg[m] * T + c : -1 - c;                               // s[g][t] / shared hidden
                ci.src[r0 + c] = src;
            }
        }
        if (lane == 0) {
            if (!fits) set_status(p.ctrl, LMOE_ERR_UNSUPPORTED);
            ci.i0 = i0;
            ci.i1 = fits ? i1 : i0;
            ci.m0 = m0;
            ci.nm = fits ? nm : 0;
            ci.rows = fits ? rows : 0;
            ci.skip = !fits;
        }
    }
    __syncthreads();
    if ((PHASE == SP_GATEUP || PHASE == SP_DOWN) && threadIdx.x < 4 * ci.nm) {
        // the experts' tensor scales (gate, up, down; plain loads, read only
        // by the epilogues, after later barriers); the Q3_K build has none
        const int jj = threadIdx.x >> 2, k = threadIdx.x & 3;
        const size_t nq = (size_t)p.L * p.F / 2, ns = (size_t)p.L * p.F / 16;
        ci.tail[jj][k] = FMT == kEfQ3k ? 1.f
                       : __ldg(reinterpret_cast<const float*>(p.experts + (size_t)sh.uexp[ci.m0 + jj] * p.rec_bytes +
                                                              3 * nq + 3 * ns) + k);
    }
}

template <int PHASE, int FMT>
__device__ __forceinline__ StepMap step_map(const FwdParams& p, const StreamShared& sh, const WPlan& pl) {
    const int nb = (PHASE == SP_DPROJ ? p.H : PHASE == SP_DOWN ? p.F : p.L) / 32;
    const int sb = step_blocks<PHASE, FMT>(false);
    StepMap m;
    m.nsA = (nb + sb - 1) / sb;
    if (PHASE == SP_UPROJ) {
        m.nA = sh.n_hit * pl.tiles;
        const int sbs = step_blocks<PHASE, FMT>(true);
        m.nsB = (p.Fs / 32 + sbs - 1) / sbs;
    } else {
        m.nA = pl.n_mats * pl.tiles;
        // D's shared-expert items: one 32-column block per step
        m.nsB = PHASE == SP_DPROJ ? p.H / 32 : m.nsA;
    }
    return m;
}

// First step of warp w's range in the CTA's chunk.
__device__ __forceinline__ int range_start(const StepMap& m, const ChunkInfo& ci, int w) {
    const int b = m.first(ci.i0), S = m.first(ci.i1) - b;
    return b + (int)(((long long)w * S) / kWW);
}

// Issue the next step of the warp's range (an empty commit group past its end).
template <int PHASE, int FMT>
__device__ __forceinline__ void cursor_issue(const FwdParams& p, const StreamShared& sh, const WPlan& plan,
                                             const StepMap& m, uint8_t* ring, LoadCursor& c, int lane) {
    if (c.st < c.s1) issue_step<PHASE, FMT>(p, c.it, c.st - c.j0, ring + (size_t)(c.n_issued % kPD) * kStepBytes, lane);
    cp_async_commit();
    ++c.n_issued;
    if (c.st >= c.s1) return;
    if (++c.st == c.j1 && c.st < c.s1) {
        ++c.j;
        c.it = decode_item<PHASE, FMT>(p, sh, plan, c.j);
        c.j0 = c.j1;
        c.j1 = m.first(c.j + 1);
    }
}

// The warp's first kPD - 1 steps (weights only: they depend on the routing).
template <int PHASE, int FMT>
__device__ void phase_prime(const FwdParams& p, const StreamShared& sh, const WPlan& plan, const ChunkInfo& ci,
                            const StepMap& m, uint8_t* ring, LoadCursor& c) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    c.st = range_start(m, ci, warp);
    c.s1 = range_start(m, ci, warp + 1);
    c.n_issued = 0;
    if (c.st < c.s1) {
        c.j = m.item(c.st);
        c.it = decode_item<PHASE, FMT>(p, sh, plan, c.j);
        c.j0 = m.first(c.j);
        c.j1 = m.first(c.j + 1);
    }
#pragma unroll
    for (int k = 0; k < kPD - 1; ++k) cursor_issue<PHASE, FMT>(p, sh, plan, m, ring, c, lane);
}

// D's activations: the block input rows (bf16) as fp16, RMS-normalised
// (gamma[k] x[k] / sqrt(mean(x^2) + eps), the stack's pre-norm) when gamma
// is given.  D reads the input itself, so it depends on no earlier kernel
// of the step.
__device__ void fill_x(const FwdParams& p, __half* cache, int ld, float* rs) {
    const int T = p.T, H = p.H, nc = H / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto unpack = [](const uint4 v, float (&f)[8]) {
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 q = bf16x2_to_f32x2(w4[j]);
            f[2 * j] = q.x;
            f[2 * j + 1] = q.y;
        }
    };
    if (p.gamma != nullptr) {
        for (int t = warp; t < T; t += blockDim.x >> 5) {
            float ss = 0.f;
            for (int c = lane; c < nc; c += 32) {
                float f[8];
                unpack(__ldg(reinterpret_cast<const uint4*>(p.x + (size_t)t * H) + c), f);
#pragma unroll
                for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
            }
            ss = warp_sum(ss);
            if (lane == 0) rs[t] = rsqrtf(ss / (float)H + p.eps);
        }
        __syncthreads();
    }
    bool bad = false;
    for (int i = threadIdx.x; i < T * nc; i += blockDim.x) {
        const int t = i / nc, c = i - t * nc;
        float f[8];
        unpack(__ldg(reinterpret_cast<const uint4*>(p.x + (size_t)t * H) + c), f);
        if (p.gamma != nullptr) {
            float g[8];
            unpack(__ldg(reinterpret_cast<const uint4*>(p.gamma) + c), g);
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] *= rs[t] * g[j];
        }
        __half2 h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = half2_checked(f[2 * j], f[2 * j + 1], bad);
        *reinterpret_cast<uint4*>(cache + (size_t)t * ld + 8 * c) = *reinterpret_cast<uint4*>(h);
    }
    // only CTA 0 reports, so that a bad input costs one atomic, not one per CTA
    if (blockIdx.x == 0) report_range(p.ctrl, bad);
}

// The chunk's activations from global memory, by plain loads of every thread.
template <int PHASE>
__device__ void phase_fill(const FwdParams& p, const StreamShared& sh, const ChunkInfo& ci, __half* cache) {
    const int T = p.T, H = p.H, L = p.L, F = p.F, Fs = p.Fs, K = p.K;
    const int ld = cache_ld<PHASE>(H, L, F, Fs);
    if (PHASE == SP_DPROJ) {
        __shared__ float rs[8];
        if (ci.rows > 0) fill_x(p, cache, ld, rs);
        return;
    }
    const int KC = PHASE == SP_DPROJ ? H : PHASE == SP_GATEUP ? L : PHASE == SP_DOWN ? F : max(L, Fs);
    const int per = KC / 8;
    bool bad = false;
    for (int qv = threadIdx.x; qv < ci.rows * per; qv += blockDim.x) {
        const int r = qv / per, c = qv - r * per;
        const int src = ci.src[r];
        uint4 v;
        if (PHASE == SP_GATEUP) {
            v = __ldcg(reinterpret_cast<const uint4*>(p.h16 + (size_t)src * L) + c);
        } else if (PHASE == SP_DOWN) {
            v = __ldcg(reinterpret_cast<const uint4*>(p.z16 + (size_t)src * F) + c);
        } else if (src >= 0) {
            // U: s[g][t] = sum of the weighted expert outputs of token t's
            // experts in group g (fp32, in k order), rounded to fp16
            if (8 * c >= L) continue;
            const int g = src / T, t = src - g * T;
            float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int k = 0; k < K; ++k) {
                if (sh.pgrp[t * K + k] != g) continue;
                const uint4 o = __ldcg(reinterpret_cast<const uint4*>(p.o16w + (size_t)sh.pair_slot[t * K + k] * L) + c);
                const uint32_t w4[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[j]));
                    acc8[2 * j] += f.x;
                    acc8[2 * j + 1] += f.y;
                }
            }
            __half2 h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) h[j] = half2_checked(acc8[2 * j], acc8[2 * j + 1], bad);
            v = *reinterpret_cast<uint4*>(h);
        } else {
            if (8 * c >= Fs) continue;
            v = __ldcg(reinterpret_cast<const uint4*>(p.zsh16 + (size_t)(-1 - src) * Fs) + c);
        }
        *reinterpret_cast<uint4*>(cache + (size_t)r * ld + 8 * c) = v;
    }
    if (PHASE == SP_UPROJ) report_range(p.ctrl, bad);
}

// An item's 16x8 result is complete: its epilogue, or (U, whose output tile
// sums the hit groups' and the shared expert's items) its partial and, in
// the warp that completes the tile (ticket), the ordered sum and epilogue.
template <int PHASE, int FMT>
__device__ __forceinline__ void item_finish(const FwdParams& p, const StreamShared& sh, const WPlan& plan,
                                            const ChunkInfo& ci, const WItem& cit, float (&a)[4], float (&u)[4]) {
    const int lane = threadIdx.x & 31;
    const int T = p.T, H = p.H, L = p.L, F = p.F, G = p.G;
    const int jj = cit.j - ci.m0;
    const int nt = (PHASE == SP_GATEUP || PHASE == SP_DOWN) ? sh.ucnt[cit.j] : T;
    const int gg = lane >> 2, tt = lane & 3;
    const int nparts = PHASE == SP_UPROJ ? phase_mats<PHASE>(p, sh) * plan.ks : plan.ks;
    bool finish = nparts == 1;
    if (!finish) {
        // partial of part (j, q) of tile (mat, tile); U: all matrices are parts of one tile
        const int key = PHASE == SP_UPROJ ? cit.tile : cit.j * plan.tiles + cit.tile;
        const int part = PHASE == SP_UPROJ ? cit.j * plan.ks + cit.q : cit.q;
        float* dst = p.wpart + (((size_t)key * nparts + part) * 32 + lane) * 8;
        *reinterpret_cast<float4*>(dst) = make_float4(a[0], a[1], a[2], a[3]);
        if (PHASE == SP_GATEUP) *reinterpret_cast<float4*>(dst + 4) = make_float4(u[0], u[1], u[2], u[3]);
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(p.wtick + key, 1) == nparts - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
            __threadfence();
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, su[4] = {0.f, 0.f, 0.f, 0.f};
            for (int q = 0; q < nparts; ++q) {
                const float* sp = p.wpart + (((size_t)key * nparts + q) * 32 + lane) * 8;
                const float4 v = __ldcg(reinterpret_cast<const float4*>(sp));
                sa[0] += v.x; sa[1] += v.y; sa[2] += v.z; sa[3] += v.w;
                if (PHASE == SP_GATEUP) {
                    const float4 w4 = __ldcg(reinterpret_cast<const float4*>(sp + 4));
                    su[0] += w4.x; su[1] += w4.y; su[2] += w4.z; su[3] += w4.w;
                }
            }
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) { a[i4] = sa[i4]; u[i4] = su[i4]; }
            if (lane == 0) p.wtick[key] = 0;
            finish = true;
        }
    }
    if (finish) {
        const float* ts = (PHASE == SP_GATEUP || PHASE == SP_DOWN) ? ci.tail[jj] : nullptr;
        bool bad = false;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
            const int col = 2 * tt + (i4 & 1), row = cit.r0 + gg + 8 * (i4 >> 1);
            if (col >= nt) continue;
            if (PHASE == SP_DPROJ && cit.mat < 0) {
                p.zsh16[(size_t)col * p.Fs + row] = half_checked(silu(a[i4]) * u[i4], bad);
            } else if (PHASE == SP_DPROJ) {
                p.h16[((size_t)col * G + cit.mat) * L + row] = half_checked(a[i4], bad);
            } else if (PHASE == SP_GATEUP) {
                p.z16[(size_t)(sh.uoff[cit.j] + col) * F + row] = half_checked(silu(a[i4] * ts[0]) * (u[i4] * ts[1]), bad);
            } else if (PHASE == SP_DOWN) {
                const int slot = sh.uoff[cit.j] + col;
                p.o16w[(size_t)slot * L + row] = half_checked(sh.slot_w[slot] * ts[2] * a[i4], bad);
            } else {
                float v = a[i4];
                if (p.residual) v += bf16_bits_to_f32(p.residual[(size_t)col * H + row]);
                p.y[(size_t)col * H + row] = f32_to_bf16_bits(v);
            }
        }
        report_range(p.ctrl, bad);
    }
}

// The warp's range of steps: stream, multiply, finish.  An item whose steps
// all fall in the range is finished by the warp; an item cut by range
// boundaries leaves one 16x8 partial per warp in shared memory (in the
// warp's step ring, free once its range is done: slot 0 for the range's
// first item, slot 1 for its last), and after a barrier the warp where the
// item begins adds the partials in warp order (K order) and finishes it.
// Contains __syncthreads.
template <int PHASE, int FMT>
__device__ void phase_run(const FwdParams& p, const StreamShared& sh, const WPlan& plan, const ChunkInfo& ci,
                          const StepMap& m, uint8_t* ring_base, const __half* cache, LoadCursor& lc) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = p.T, H = p.H, L = p.L, F = p.F;
    const int ld = cache_ld<PHASE>(H, L, F, p.Fs);
    uint8_t* ring = ring_base + (size_t)warp * kPD * kStepBytes;
    const int s0 = range_start(m, ci, warp), s1 = range_start(m, ci, warp + 1);
    float a[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
    float ha[4] = {0.f, 0.f, 0.f, 0.f}, hu[4] = {0.f, 0.f, 0.f, 0.f};
    bool first_cut = false, last_cut = false;
    int n_done = 0;
    int st = s0;
    while (st < s1) {
        const int j = m.item(st);
        const WItem cit = decode_item<PHASE, FMT>(p, sh, plan, j);
        const int j0 = m.first(j), j1 = m.first(j + 1);
        const int e = min(s1, j1);
        const int jj = cit.j - ci.m0;
        const __half* xs = PHASE == SP_DPROJ ? cache : cache + (size_t)ci.row0[jj] * ld;
        const int nt = (PHASE == SP_GATEUP || PHASE == SP_DOWN) ? sh.ucnt[cit.j] : T;
        for (; st < e; ++st) {
            cursor_issue<PHASE, FMT>(p, sh, plan, m, ring, lc, lane);
            cp_async_wait<kPD - 1>();
            __syncwarp();
            compute_step<PHASE, FMT>(p, cit, st - j0, ring + (size_t)(n_done % kPD) * kStepBytes, xs, ld, nt, a, u);
            __syncwarp();
            ++n_done;
        }
        if (j0 >= s0 && j1 <= s1) {
            item_finish<PHASE, FMT>(p, sh, plan, ci, cit, a, u);
        } else if (j0 < s0) {
            first_cut = true;
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) { ha[i4] = a[i4]; hu[i4] = u[i4]; }
        } else {
            last_cut = true;
            break;
        }
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) { a[i4] = 0.f; u[i4] = 0.f; }
    }
    cp_async_wait<0>();
    __syncwarp();
    float* part = reinterpret_cast<float*>(ring);
    constexpr bool kTwoSums = PHASE == SP_GATEUP || PHASE == SP_DPROJ;   // gate and up (D: shared expert)
    if (first_cut) {
        *reinterpret_cast<float4*>(part + lane * 8) = make_float4(ha[0], ha[1], ha[2], ha[3]);
        if (kTwoSums) *reinterpret_cast<float4*>(part + lane * 8 + 4) = make_float4(hu[0], hu[1], hu[2], hu[3]);
    }
    if (last_cut) {
        *reinterpret_cast<float4*>(part + 256 + lane * 8) = make_float4(a[0], a[1], a[2], a[3]);
        if (kTwoSums) *reinterpret_cast<float4*>(part + 256 + lane * 8 + 4) = make_float4(u[0], u[1], u[2], u[3]);
    }
    __syncthreads();
    if (last_cut) {
        // the item begun here and continued by the next warps
        const int j = m.item(s1 - 1);
        const WItem cit = decode_item<PHASE, FMT>(p, sh, plan, j);
        const int j1 = m.first(j + 1);
        for (int w = warp + 1; w < kWW && range_start(m, ci, w) < j1; ++w) {
            if (range_start(m, ci, w + 1) == range_start(m, ci, w)) continue;   // empty range
            const float* q = reinterpret_cast<const float*>(ring_base + (size_t)w * kPD * kStepBytes) + lane * 8;
            const float4 v = *reinterpret_cast<const float4*>(q);
            a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
            if (kTwoSums) {
                const float4 w4 = *reinterpret_cast<const float4*>(q + 4);
                u[0] += w4.x; u[1] += w4.y; u[2] += w4.z; u[3] += w4.w;
            }
        }
        item_finish<PHASE, FMT>(p, sh, plan, ci, cit, a, u);
    }
}

// Routing tables of a later kernel, as the router kernel published them.
template <int PHASE>
__device__ void stage_published_routing(const FwdParams& p, StreamShared& sh) {
    const int T = p.T, G = p.G, K = p.K;
    if (PHASE == SP_GATEUP || PHASE == SP_DOWN) {
        const int n = T * K;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            sh.uexp[i] = __ldcg(p.r.uexp + i);
            sh.ucnt[i] = __ldcg(p.r.ucnt + i);
            sh.uoff[i] = __ldcg(p.r.uoff + i);
            sh.ugrp[i] = __ldcg(p.r.ugrp + i);
            sh.slot_tok[i] = __ldcg(p.r.slot_tok + i);
            sh.slot_w[i] = __ldcg(p.r.slot_w + i);
        }
        if (threadIdx.x == 0) sh.n_unique = __ldcg(p.r.n_unique);
    } else {
        if (threadIdx.x < G) sh.hg[threadIdx.x] = __ldcg(p.r.ghit + threadIdx.x);
        if (PHASE == SP_UPROJ) {
            for (int i = threadIdx.x; i < T * K; i += blockDim.x) {
                sh.pgrp[i] = __ldcg(p.r.pgrp + i);
                sh.pair_slot[i] = __ldcg(p.r.pair_slot + i);
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int n = 0;
            for (int g = 0; g < G; ++g)
                if (sh.hg[g] > 0) sh.hg[n++] = g;
            sh.n_hit = n;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// one kernel per phase (a router kernel ran before; routing published)
// ---------------------------------------------------------------------------

template <int PHASE, int FMT>
__global__ void __launch_bounds__(kWThreads, 1) k_wstream(FwdParams p, WPlan pl, int cache_bytes) {
    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the shared array, so that the compiler
    // still knows every access through it is a shared-memory access
    uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    __shared__ StreamShared sh;
    __shared__ ChunkInfo ci;
    const int warp = threadIdx.x >> 5;
    __half* cache = reinterpret_cast<__half*>(smem);
    uint8_t* ring = smem + cache_bytes + (size_t)warp * kPD * kStepBytes;

    if (PHASE == SP_DOWN && FMT == kEfQ3k) iq4nl_fill_lut(iq4nl_lut());   // ordered by the barriers below
    // D needs nothing from the router kernel and starts while it runs; it
    // waits for it only at its end, so that D's completion implies the
    // router kernel's.  The later kernels read the routing before their own
    // wait: their predecessor let them launch only after its own wait, so
    // the router kernel had completed by then.
    if (PHASE != SP_DPROJ) stage_published_routing<PHASE>(p, sh);
    WPlan plan = pl;
    plan.n_mats = phase_mats<PHASE>(p, sh);
    phase_setup<PHASE, FMT>(p, sh, plan, cache_bytes, ci);
    const StepMap m = step_map<PHASE, FMT>(p, sh, plan);
    LoadCursor lc;
    phase_prime<PHASE, FMT>(p, sh, plan, ci, m, ring, lc);
    if (PHASE != SP_DPROJ) {
        grid_dep_wait();
        grid_dep_launch();
    }
    phase_fill<PHASE>(p, sh, ci, cache);
    __syncthreads();
    phase_run<PHASE, FMT>(p, sh, plan, ci, m, smem + cache_bytes, cache, lc);
    if (PHASE == SP_DPROJ) {
        grid_dep_wait();
        grid_dep_launch();
    }
}

// ---------------------------------------------------------------------------
// launch helpers
// ---------------------------------------------------------------------------

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


// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Reduction parts per tile of each phase.  Measured on B200: splitting a
// tile's reduction over several warps (to have an item for every warp)
// costs more in partial round trips and tickets than the parallelism
// returns, so every tile is reduced by one warp (one part); U's tiles still
// meet through a ticket, because the hit groups and the shared expert are
// separate items of one output tile.
struct WPlans {
    WPlan d, gu, dn, u;
    size_t part_floats, ticks;
};

template <int PHASE, int FMT>
static WPlan plan_for(int H, int L, int F, int Fs, int G, int n_mats_max) {
    WPlan w;
    w.tiles = stream_rows<PHASE>(H, L, F) / 16;
    w.n_mats = n_mats_max;
    w.ks = 1;
    (void)Fs;
    (void)G;
    return w;
}

WPlans stream_plans(int H, int L, int F, int Fs, int G, int E, int K, int T, int du_fmt) {
    WPlans P;
    const int nu = std::min(T * K, E);
    if (du_fmt == LMOE_Q8_0) {
        P.d = plan_for<SP_DPROJ, LMOE_Q8_0>(H, L, F, Fs, G, G);
        P.u = plan_for<SP_UPROJ, LMOE_Q8_0>(H, L, F, Fs, G, G + 1);
    } else {
        P.d = plan_for<SP_DPROJ, LMOE_Q4_0>(H, L, F, Fs, G, G);
        P.u = plan_for<SP_UPROJ, LMOE_Q4_0>(H, L, F, Fs, G, G + 1);
    }
    P.gu = plan_for<SP_GATEUP, LMOE_Q8_0>(H, L, F, Fs, G, nu);
    P.dn = plan_for<SP_DOWN, LMOE_Q8_0>(H, L, F, Fs, G, nu);
    // partials (8 floats per lane, 32 lanes) and tickets, the largest phase
    auto parts = [](const WPlan& w) { return (size_t)w.n_mats * w.tiles * w.ks; };
    P.part_floats = std::max(256 * std::max({parts(P.d), parts(P.gu), parts(P.dn), parts(P.u)}), nvf4_part_floats());
    P.ticks = std::max({(size_t)P.d.n_mats * P.d.tiles, (size_t)P.gu.n_mats * P.gu.tiles, (size_t)P.dn.n_mats * P.dn.tiles,
                        (size_t)P.u.tiles});
    return P;
}

size_t stream_ws_part_bytes(int H, int L, int F, int Fs, int G, int E, int K, int T, int du_fmt) {
    return stream_plans(H, L, F, Fs, G, E, K, T, du_fmt).part_floats * sizeof(float);
}
size_t stream_ws_tick_bytes(int H, int L, int F, int Fs, int G, int E, int K, int T, int du_fmt) {
    return stream_plans(H, L, F, Fs, G, E, K, T, du_fmt).ticks * sizeof(int);
}

template <int PHASE, int FMT>
static cudaError_t launch_wstream(const FwdParams& p, const WPlan& plan, int cache_rows, cudaStream_t st) {
    const int ld = PHASE == SP_DPROJ ? p.H + kActPad
                 : PHASE == SP_GATEUP ? p.L + kActPad
                 : PHASE == SP_DOWN ? p.F + kActPad
                                    : std::max(p.L, p.Fs) + kActPad;
    const int cache_bytes = round128(cache_rows * ld * 2);
    const size_t smem = 128 + (size_t)cache_bytes + (size_t)kWW * kPD * kStepBytes;
    auto kern = k_wstream<PHASE, FMT>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    if (!g_sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    stage_mark(st);
    // D runs beside the router kernel's routing CTA, which keeps one SM
    const int grid = PHASE == SP_DPROJ ? std::max(1, g_sms - 1) : g_sms;
    return launch_dependent(kern, dim3(grid), dim3(kWThreads), smem, st, p, plan, cache_bytes);
}

// LMOE_FEW_TOKEN_EXPERTS selects the few-token NVFP4 expert phases:
// "tensor_cores" runs them on the tensor-core kernels (kind::mxf4nvf4, the
// weights as stored); anything else (the default) on the weight-streaming
// kernels (mma.sync, weights dequantised in registers), which measure
// faster on the Edge0 shapes.  Read at every call.
static bool tensor_core_experts() {
    const char* s = std::getenv("LMOE_FEW_TOKEN_EXPERTS");
    return s && std::strcmp(s, "tensor_cores") == 0;
}

// D, experts, combine, U for T <= 8 (the router kernel has run).
cudaError_t run_stream_path(const FwdParams& p, cudaStream_t st) {
    const int H = p.H, L = p.L, F = p.F, Fs = p.Fs, G = p.G, T = p.T;
    const WPlans P = stream_plans(H, L, F, Fs, G, p.E, p.K, T, p.du_fmt);
    if (!g_sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    // cache rows: the distinct matrices one CTA's contiguous chunk can span, T rows each
    auto chunk_rows = [&](const WPlan& w) {
        const int per_mat = w.tiles * w.ks;
        const int chunk = (w.n_mats * per_mat + g_sms - 1) / g_sms;
        const int mats = std::min(w.n_mats, (chunk + per_mat - 1) / per_mat + 1);
        return std::min(mats, kMaxChunkParts) * T;
    };
    cudaError_t e = p.du_fmt == LMOE_Q8_0 ? launch_wstream<SP_DPROJ, LMOE_Q8_0>(p, P.d, T, st)
                              : launch_wstream<SP_DPROJ, LMOE_Q4_0>(p, P.d, T, st);
    if (e != cudaSuccess) return e;
    if (p.act == LMOE_ACT_NVFP4 || (nvf4_usable(p) && tensor_core_experts())) {
        // NVFP4 experts on the tensor cores, weights as stored
        if ((e = run_nvf4_gateup(p, st)) != cudaSuccess) return e;
        if ((e = run_nvf4_down(p, st)) != cudaSuccess) return e;
    } else {
        e = p.efmt == kEfQ3k ? launch_wstream<SP_GATEUP, kEfQ3k>(p, P.gu, chunk_rows(P.gu), st)
                             : launch_wstream<SP_GATEUP, kEfNvfp4>(p, P.gu, chunk_rows(P.gu), st);
        if (e != cudaSuccess) return e;
        e = p.efmt == kEfQ3k ? launch_wstream<SP_DOWN, kEfQ3k>(p, P.dn, chunk_rows(P.dn), st)
                             : launch_wstream<SP_DOWN, kEfNvfp4>(p, P.dn, chunk_rows(P.dn), st);
        if (e != cudaSuccess) return e;
    }
    e = p.du_fmt == LMOE_Q8_0 ? launch_wstream<SP_UPROJ, LMOE_Q8_0>(p, P.u, chunk_rows(P.u), st)
                              : launch_wstream<SP_UPROJ, LMOE_Q4_0>(p, P.u, chunk_rows(P.u), st);
    return e;
}

}  // namespace lmoe

