// Few-token expert phases (gate/up and down, NVFP4 records, T <= 8) on the
// tensor cores, with the weights read exactly as they are stored.
//
// The teardown article's "What is 4-bit" section defines the expert format:
// E2M1 codes, one E4M3 scale per 16 elements, and an fp32 scale per matrix.
// That is the operand format of tcgen05.mma kind::mxf4nvf4.  So the weight
// tiles go from HBM to shared memory in their stored byte order (a
// [32-column chunk][row][16 B] block is the no-swizzle K-major canonical
// layout), and their scale words go to tensor memory.  No weight passes
// through a register.
//
// The other operand of kind::mxf4nvf4 is E2M1 too.  An fp16 activation row
// x (h for gate/up, z for down) therefore enters as J = 6 E2M1 rows that sum
// to it:
//   x ~= sum_j G_j * s_j[b] * q_j[k]      (k in 16-element block b)
// G_j = max|x| / (6 * 448) * 5^-j is one fp32 per row and term.  s_j[b] is the
// E4M3 scale of block b, rounded up from max|r_j| / (6 G_j).  q_j holds the
// E2M1 codes of r_j / (s_j G_j).  Here r_j is the residual that the earlier
// terms leave: r_0 = x, r_{j+1} = r_j - G_j s_j q_j, computed exactly from the
// decoded codes.
//   Each term removes at least 81% of the residual, because rounding to the
// E2M1 grid leaves at most 1/6 of the block maximum and the E4M3 rounding of
// the scale adds at most 1/8 of that.  So after six terms the error is below
// 5e-5 of the block maximum, under the rounding of x to fp16.  The 5^-j
// decay keeps every s_j at or below 448.
//   The terms of token i are the B columns i*J .. i*J + J - 1 of the MMA
// (N = 16, 32 or 48).  The epilogue sums them in fp32 with their G_j.
//
// One CTA per SM, 9 warps:
//   0-3  loaders: 16-byte cp.async copies of each K stage's codes and scale
//        words into a ring of shared-memory slots, three stages in flight;
//        then each warp copies the stage's scale words to its 32-lane TMEM
//        subpartition.  (TMA copies measured slower here: a fixed cost per
//        copy on each SM capped a ring of 16 KB and 2 KB boxes near 15 GB/s
//        per SM.)
//   4-7  the activation operand of each expert run (shared memory, scales
//        in tensor memory), built one piece ahead; the epilogue: tensor
//        memory -> fp32 per token -> SwiGLU (gate/up) or routing weight
//        (down) -> fp16
//   8    MMA issue (one thread), TMEM allocation
// Work: the items (distinct expert, 128-row tile) of the phase, each a run of
// 256-column K stages, laid end to end and cut into equal contiguous stage
// ranges, one per CTA.  An item cut by range boundaries leaves an fp32
// partial per piece in the workspace; the CTA that finishes last (ticket)
// adds them in CTA order and runs the epilogue.

#include <cstring>

#include "lmoe_internal.cuh"
#include "lmoe_sm100.cuh"

namespace lmoe {
namespace {

using namespace sm100;

enum NvPhase { NV_GATEUP = 0, NV_DOWN = 1 };

constexpr int kNvJExact = 6;             // E2M1 terms per activation row (fp16-level inputs)
constexpr int kNvJW4A4 = 1;              // one term: NVFP4 activations (W4A4)
constexpr int kNvThreads = 288;
constexpr int kNvMaxN = 48;              // B columns: 8 tokens x 6 terms
constexpr int kNvMaxCtas = 160;
constexpr int kNvMaxPairs = 8 * kMaxTopK;
constexpr int kNvMaxK = 2048;            // reduction length (scale columns of B in TMEM)
constexpr uint64_t kNvWaitLimit = 4000000000ull;   // SM cycles per barrier wait (about 2 s)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColD = 0;            // accumulators: 2 buffers x 2 matrices x 64 columns
constexpr uint32_t kColSFA = 256;        // weight scales: stage slot x matrix x 4 MMAs x 4 columns
constexpr uint32_t kColSFB = 384;        // activation scales: 4 columns per 64-column MMA step
constexpr int kStageK = 256;             // columns of one TMA stage (8 chunks of 32)
constexpr int kCodeBox = 128 * 128;      // bytes of one stage's codes of one matrix (8 chunks x 128 rows x 16 B)
constexpr int kScaleBox = 4 * 128 * 4;   // bytes of one stage's scale words of one matrix

template <int PHASE>
struct NvGeom {
    static constexpr int NM = PHASE == NV_GATEUP ? 2 : 1;        // weight matrices per item (gate, up)
    static constexpr int STAGES = PHASE == NV_GATEUP ? 4 : 8;    // TMA ring depth
};

struct __align__(64) NvArgs {
    FwdParams p;
    int ncap;        // B columns the shared memory holds (multiple of 16)
};

// ---------------------------------------------------------------------------
// PTX wrappers specific to this kernel
// ---------------------------------------------------------------------------

__device__ __forceinline__ void cp_async16_nv(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_nv() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_nv() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared-memory descriptor of a K-major operand in the no-swizzle canonical
// layout: 8-row x 16-byte core matrices, `lbo` bytes between the two core
// matrices of one 64-element (32-byte) MMA step along K, `sbo` bytes between
// 8-row groups.  Descriptor version 1, layout type 0.
__device__ __forceinline__ uint64_t sdesc_nosw(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFF) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (format code 1),
// both K-major, UE4M3 scales (scale format 0), M = 128, K = 64 per MMA, fp32
// accumulation; the scale words sit at byte 0 of their TMEM columns.
__host__ __device__ constexpr uint32_t idesc_mxf4nvf4(int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_mxf4nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns from registers: lane i of the
// warp writes TMEM lane (taddr.lane + i).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// E4M3 code of s rounded to nearest (saturating at 448), and its value.
__device__ __forceinline__ uint32_t e4m3_rn(float s) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.f), "f"(s));
    return h & 0xFFu;
}
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(c));
    return __half2float(__ushort_as_half((uint16_t)(r & 0xFFFFu)));
}
// The smallest E4M3 value not below s (0 < s; 448 at most).
__device__ __forceinline__ uint32_t e4m3_up(float s) {
    uint32_t c = e4m3_rn(s);
    if (e4m3_value(c) < s && c < 0x7Eu) ++c;
    return c;
}
// Two E2M1 codes (round to nearest, saturating at 6) in one byte: lo in the
// low nibble.
__device__ __forceinline__ uint32_t e2m1x2_rn(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------------------
// the work split (identical in every role)
// ---------------------------------------------------------------------------

struct NvWork {
    int tiles;   // 128-row tiles of one expert matrix
    int spi;     // K stages per item
    int S;       // stages of the phase
    int G;       // CTAs
    int s0, s1;  // this CTA's stages
    // fewer stages than CTAs: one stage each for the first S CTAs (no empty
    // range lies between two CTAs that share an item)
    __device__ __forceinline__ int start(int c) const {
        return S >= G ? (int)(((long long)c * S) / G) : (c < S ? c : S);
    }
    // the CTA whose range holds stage s
    __device__ __forceinline__ int cta_of(int s) const {
        if (S < G) return s;
        int c = (int)(((long long)s * G) / S);
        if (c > G - 1) c = G - 1;
        while (c + 1 < G && start(c + 1) <= s) ++c;
        while (c > 0 && start(c) > s) --c;
        return c;
    }
};

struct NvShared {
    int uexp[kNvMaxPairs];
    int ucnt[kNvMaxPairs];
    int uoff[kNvMaxPairs];
    int ugrp[kNvMaxPairs];
    int slot_tok[kNvMaxPairs];
    float slot_w[kNvMaxPairs];
    int n_unique;
    int last;                    // epilogue: this CTA finishes the item
    float red[4][8];             // per-warp row maxima of the activation build
};

// Piece of the CTA's stage range that begins at stage s: [s, e) within one item.
__device__ __forceinline__ int piece_end(const NvWork& w, int s) {
    const int item_end = (s / w.spi + 1) * w.spi;
    return item_end < w.s1 ? item_end : w.s1;
}
// Whether the piece starting at s begins a run of a new expert (a new B operand).
__device__ __forceinline__ bool starts_build(const NvWork& w, int s) {
    return s == w.s0 || (s / w.spi) / w.tiles != ((s - 1) / w.spi) / w.tiles;
}
// Whether stage s is the last of its expert run within the range.
__device__ __forceinline__ bool ends_build(const NvWork& w, int s) {
    return s + 1 == w.s1 || (s / w.spi) / w.tiles != ((s + 1) / w.spi) / w.tiles;
}

// ---------------------------------------------------------------------------
// activation operand of one expert (warps 0-3, 128 threads)
// ---------------------------------------------------------------------------

template <int PHASE>
__device__ __forceinline__ const __half* act_row(const FwdParams& p, const NvShared& sh, int j, int i) {
    if (PHASE == NV_GATEUP) {
        const int t = sh.slot_tok[sh.uoff[j] + i];
        return p.h16 + ((size_t)t * p.G + sh.ugrp[j]) * p.L;
    }
    return p.z16 + (size_t)(sh.uoff[j] + i) * p.F;
}

// Rows i*J + jj of the B operand (codes in [K/32][npad][16 B], scale bytes
// [npad][K/16]) and their fp32 term scales; then the scale words to TMEM
// columns kColSFB + 4k + n/32, lane n%32 of every subpartition.
template <int PHASE, int J>
__device__ void build_b(const FwdParams& p, NvShared& sh, int j, int K, uint8_t* sB, uint8_t* sfbb, float* cs,
                        uint32_t tmem_base, bool& bad) {
    const int tid = threadIdx.x - 128, warp = tid >> 5, lane = tid & 31;   // warps 4-7: subpartitions 0-3
    const int ne = sh.ucnt[j], N = ne * J, npad = (N + 15) & ~15;
    const int nb = K / 16;
    // 1. row maxima
    for (int i = 0; i < ne; ++i) {
        const uint4* row = reinterpret_cast<const uint4*>(act_row<PHASE>(p, sh, j, i));
        float m = 0.f;
        for (int c = tid; c < K / 8; c += 128) {
            const uint4 v = __ldcg(row + c);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[u]));
                m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) sh.red[warp][i] = m;
    }
    named_bar_sync(2, 128);
    if (tid < N) {
        const int i = tid / J, jj = tid - i * J;
        const float amax = fmaxf(fmaxf(sh.red[0][i], sh.red[1][i]), fmaxf(sh.red[2][i], sh.red[3][i]));
        float g = amax > 0.f ? amax * (1.f / (6.f * 448.f)) : 1.f;
        for (int u = 0; u < jj; ++u) g *= 0.2f;
        cs[tid] = g;
    }
    named_bar_sync(2, 128);
    // 2. the terms, one 16-element block per thread
    for (int t = tid; t < ne * nb; t += 128) {
        const int i = t / nb, b = t - i * nb;
        const uint4* src = reinterpret_cast<const uint4*>(act_row<PHASE>(p, sh, j, i) + 16 * b);
        const uint4 v0 = __ldcg(src), v1 = __ldcg(src + 1);
        float r[16];
        {
            const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w8[u]));
                r[2 * u] = f.x;
                r[2 * u + 1] = f.y;
            }
        }
#pragma unroll 1
        for (int jj = 0; jj < J; ++jj) {
            const int n = i * J + jj;
            const float g = cs[n];
            float amax = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(r[e]));
            uint32_t sc = 0, lo = 0, hi = 0;
            if (amax > 0.f) {
                sc = e4m3_up(amax / (6.f * g));
                const float sd = e4m3_value(sc) * g;
                const float inv = 1.f / sd;
#pragma unroll
                for (int e = 0; e < 4; ++e) lo |= e2m1x2_rn(r[2 * e] * inv, r[2 * e + 1] * inv) << (8 * e);
#pragma unroll
                for (int e = 0; e < 4; ++e) hi |= e2m1x2_rn(r[8 + 2 * e] * inv, r[8 + 2 * e + 1] * inv) << (8 * e);
                uint32_t dl[4], dh[4];
                e2m1x8_to_f16x8(lo, dl);
                e2m1x8_to_f16x8(hi, dh);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&dl[e]));
                    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&dh[e]));
                    r[2 * e] = fmaf(-a.x, sd, r[2 * e]);
                    r[2 * e + 1] = fmaf(-a.y, sd, r[2 * e + 1]);
                    r[8 + 2 * e] = fmaf(-c.x, sd, r[8 + 2 * e]);
                    r[8 + 2 * e + 1] = fmaf(-c.y, sd, r[8 + 2 * e + 1]);
                }
            }
            *reinterpret_cast<uint2*>(sB + ((size_t)(b >> 1) * npad + n) * 16 + (b & 1) * 8) = make_uint2(lo, hi);
            sfbb[n * nb + b] = (uint8_t)sc;
        }
        (void)bad;
    }
    // padding columns: zero codes and scales
    for (int t = tid; t < (npad - N) * nb; t += 128) {
        const int n = N + t / nb, b = t % nb;
        *reinterpret_cast<uint2*>(sB + ((size_t)(b >> 1) * npad + n) * 16 + (b & 1) * 8) = make_uint2(0u, 0u);
        sfbb[n * nb + b] = 0;
    }
    fence_proxy_async_smem();
    named_bar_sync(2, 128);
    // 3. scale words to TMEM (each warp: its subpartition, the same words);
    // the tcgen05 loads and stores are warp-collective (.sync.aligned), so
    // every lane reaches each of them together
    const int nk = K / 64;
    for (int k0 = 0; k0 < nk; k0 += 4) {
        uint32_t v[16];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int n = lane + 32 * bb, k = k0 + kk;
                v[kk * 4 + bb] = (k < nk && n < npad) ? *reinterpret_cast<const uint32_t*>(sfbb + n * nb + 4 * k) : 0u;
            }
        }
        __syncwarp();
        tmem_st_32x32b_x16(tmem_base + ((uint32_t)(32 * warp) << 16) + kColSFB + 4 * k0, v);
    }
    __syncwarp();
    tmem_st_wait();
    tc_fence_before();
    named_bar_sync(2, 128);
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

template <int PHASE, int J>
__global__ void __launch_bounds__(kNvThreads, 1) k_nvf4(const __grid_constant__ NvArgs a) {
    using Geo = NvGeom<PHASE>;
    constexpr int NM = Geo::NM, STAGES = Geo::STAGES;
    constexpr int LA = STAGES - 2;   // stages in flight ahead; one more slot gives the MMA a stage of slack
    const FwdParams& p = a.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int K = PHASE == NV_GATEUP ? p.L : p.F;   // reduction
    const int R = PHASE == NV_GATEUP ? p.F : p.L;   // rows of one matrix
    const int ncap = a.ncap;
    uint8_t* sA = smem;                                              // [slot][m] codes
    uint8_t* sS = sA + STAGES * NM * kCodeBox;                       // [slot][m] scale words
    uint8_t* sB = sS + STAGES * NM * kScaleBox;                      // activation codes
    uint8_t* sfbb = sB + (size_t)ncap * (K / 2);                     // activation scale bytes
    float* cs = reinterpret_cast<float*>(sfbb + (size_t)ncap * (K / 16));   // [2][ncap] term scales
    uint64_t* bars = reinterpret_cast<uint64_t*>(cs + 2 * ncap);
    uint64_t* full = bars;               // [STAGES] stage landed, weight scales in TMEM (4 loader warps)
    uint64_t* empty = full + STAGES;     // [STAGES] the stage's MMAs completed (commit)
    uint64_t* b_full = empty + STAGES;   // activation operand built (1)
    uint64_t* b_empty = b_full + 1;      // the expert run's MMAs completed (commit)
    uint64_t* tfull = b_empty + 1;       // [2] piece accumulated (commit)
    uint64_t* tempty = tfull + 2;        // [2] accumulator read (4 epilogue warps)
    uint64_t* final_bar = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    __shared__ NvShared sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // routing tables (published by the router kernel, which completed before
    // this grid could launch)
    {
        const int n = p.T * p.K;
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            sh.uexp[i] = __ldcg(p.r.uexp + i);
            sh.ucnt[i] = __ldcg(p.r.ucnt + i);
            sh.uoff[i] = __ldcg(p.r.uoff + i);
            sh.ugrp[i] = __ldcg(p.r.ugrp + i);
            sh.slot_tok[i] = __ldcg(p.r.slot_tok + i);
            sh.slot_w[i] = __ldcg(p.r.slot_w + i);
        }
        if (threadIdx.x == 0) sh.n_unique = __ldcg(p.r.n_unique);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(b_full, 1);
        mbar_init(b_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 4);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 8) {
        __syncwarp();
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    NvWork w;
    w.tiles = R / 128;
    w.spi = (K + kStageK - 1) / kStageK;
    w.S = sh.n_unique * w.tiles * w.spi;
    w.G = gridDim.x;
    w.s0 = w.start(blockIdx.x);
    w.s1 = w.start(blockIdx.x + 1);
    const size_t nq = (size_t)p.L * p.F / 2, ns = (size_t)p.L * p.F / 16;

    if (warp < 4) {
        // -------------------------------------------------------- loaders
        // Stage i of the range goes to ring slot i % STAGES by 16-byte
        // cp.async copies: thread t copies row t of each 32-column chunk of
        // the stage (the 128 threads cover a chunk's 2 KB contiguously) and
        // two 16-byte pieces of scale words.  LA stages stay in flight; when
        // stage i - LA has landed, each warp copies its scale words to its
        // TMEM subpartition and the four warps arrive on full.
        const int lt = threadIdx.x;
        const int n = w.s1 - w.s0;
        bool dead = false;
        for (int i = 0; i < n + LA; ++i) {
            if (i < n) {
                const int slot = i % STAGES;
                if (!dead) dead = !mbar_wait(&empty[slot], ((i / STAGES) & 1) ^ 1, abort_flag, kNvWaitLimit);
                if (!dead) {
                    const int s = w.s0 + i;
                    const int item = s / w.spi, q = s - item * w.spi;
                    const int jd = item / w.tiles, tile = item - jd * w.tiles;
                    const uint8_t* rec = p.experts + (size_t)sh.uexp[jd] * p.rec_bytes;
                    const int nch = min(8, K / 32 - q * 8), ncp = min(4, K / 64 - q * 4);
#pragma unroll
                    for (int m = 0; m < NM; ++m) {
                        const uint8_t* qm = rec + (PHASE == NV_GATEUP ? m : 2) * nq;
                        uint8_t* dq = sA + (slot * NM + m) * kCodeBox;
                        for (int c = 0; c < nch; ++c)
                            cp_async16_nv(dq + c * 2048 + lt * 16, qm + ((size_t)(q * 8 + c) * R + tile * 128 + lt) * 16);
                        const uint8_t* sm = rec + 3 * nq + (PHASE == NV_GATEUP ? m : 2) * ns;
                        uint8_t* ds = sS + (slot * NM + m) * kScaleBox;
                        for (int x = lt; x < ncp * 32; x += 128) {
                            const int cp = x >> 5, r4 = x & 31;
                            cp_async16_nv(ds + cp * 512 + r4 * 16, sm + ((size_t)(q * 4 + cp) * R + tile * 128 + 4 * r4) * 4);
                        }
                    }
                }
            }
            cp_async_commit_nv();
            if (i >= LA) {
                const int j = i - LA, slot = j % STAGES;
                cp_async_wait_nv<LA>();
                fence_proxy_async_smem();
                dead = __any_sync(0xffffffffu, dead);
                named_bar_sync(1, 128);
                if (!dead) {
                    const uint32_t* src = reinterpret_cast<const uint32_t*>(sS);
#pragma unroll
                    for (int m = 0; m < NM; ++m) {
                        uint32_t v[16];
#pragma unroll
                        for (int k = 0; k < 4; ++k)
#pragma unroll
                            for (int bb = 0; bb < 4; ++bb)
                                v[k * 4 + bb] = src[(slot * NM + m) * 512 + k * 128 + lane + 32 * bb];
                        __syncwarp();
                        tmem_st_32x32b_x16(tmem_base + ((uint32_t)(32 * warp) << 16) + kColSFA + (uint32_t)((slot * NM + m) * 16), v);
                    }
                    __syncwarp();
                    tmem_st_wait();
                    tc_fence_before();
                }
                __syncwarp();
                if (lane == 0 && !dead) mbar_arrive(&full[slot]);
            }
            if (i == LA - 1) {
                // the first stages are in flight: follow the predecessor grid
                grid_dep_wait();
                grid_dep_launch();
            }
        }
        cp_async_wait_nv<0>();
    } else if (warp == 8) {
        // -------------------------------------------------------- MMA issue
        grid_dep_wait();
        grid_dep_launch();
        if (lane == 0) {
            uint32_t it = 0, pc = 0, bidx = 0;
            bool dead = false, issued = false;
            for (int s = w.s0; s < w.s1 && !dead;) {
                const int e_end = piece_end(w, s);
                const int d = pc & 1;
                if (!mbar_wait(&tempty[d], ((pc >> 1) & 1) ^ 1, abort_flag, kNvWaitLimit)) { dead = true; break; }
                tc_fence_after();
                const int jd = (s / w.spi) / w.tiles;
                const int npad = (sh.ucnt[jd] * J + 15) & ~15;
                const uint32_t idesc = idesc_mxf4nvf4(npad);
                const uint32_t d_tmem = tmem_base + kColD + d * 128;
                for (int st = s; st < e_end; ++st) {
                    if (starts_build(w, st)) {
                        if (!mbar_wait(b_full, bidx & 1, abort_flag, kNvWaitLimit)) { dead = true; break; }
                        ++bidx;
                    }
                    const int slot = it % STAGES;
                    if (!mbar_wait(&full[slot], (it / STAGES) & 1, abort_flag, kNvWaitLimit)) { dead = true; break; }
                    tc_fence_after();
                    const int q = st % w.spi;
                    const int kk = min(4, (K - q * kStageK) / 64);
                    for (int k = 0; k < kk; ++k) {
                        const int kg = q * 4 + k;
                        const uint64_t bdesc = sdesc_nosw(smem_u32(sB) + (uint32_t)(kg * 32 * npad), (uint32_t)npad * 16, 128);
#pragma unroll
                        for (int m = 0; m < NM; ++m) {
                            const uint64_t adesc =
                                sdesc_nosw(smem_u32(sA + (slot * NM + m) * kCodeBox) + (uint32_t)(k * 4096), 2048, 128);
                            umma_mxf4nvf4(d_tmem + m * 64, adesc, bdesc, idesc,
                                          tmem_base + kColSFA + (uint32_t)((slot * NM + m) * 16 + 4 * k),
                                          tmem_base + kColSFB + (uint32_t)(4 * kg), (st > s || k > 0) ? 1u : 0u);
                        }
                    }
                    issued = true;
                    umma_commit(&empty[slot]);
                    if (ends_build(w, st)) umma_commit(b_empty);
                    ++it;
                }
                if (dead) break;
                umma_commit(&tfull[d]);
                ++pc;
                s = e_end;
            }
            if (issued) {
                umma_commit(final_bar);
                volatile int dummy = 0;
                mbar_wait(final_bar, 0, &dummy, kNvWaitLimit);
            }
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------- activations and epilogue (warps 4-7)
        // Each expert run's activation operand is built one piece ahead: as
        // soon as the MMAs of the previous expert are done (b_empty), before
        // that expert's last epilogue, so the tensor core resumes at once.
        grid_dep_wait();
        grid_dep_launch();
        const int et = threadIdx.x - 128;           // row within the tile (TMEM lane)
        const int sub = warp & 3;
        uint32_t pc = 0, nbuilt = 0;
        int cur_b = -1;
        bool dead = false, bad = false;
        float* wpart = p.wpart;
        auto build = [&](int s_first) {
            const int jd = (s_first / w.spi) / w.tiles;
            if (nbuilt >= 1 && !dead) dead = !mbar_wait(b_empty, (nbuilt - 1) & 1, abort_flag, kNvWaitLimit);
            dead = __any_sync(0xffffffffu, dead);
            tc_fence_after();
            if (!dead) build_b<PHASE, J>(p, sh, jd, K, sB, sfbb, cs + (nbuilt & 1) * ncap, tmem_base, bad);
            else {
                named_bar_sync(2, 128);
                named_bar_sync(2, 128);
                named_bar_sync(2, 128);
                named_bar_sync(2, 128);
            }
            if (et == 0 && !dead) mbar_arrive(b_full);
            ++nbuilt;
        };
        for (int s = w.s0; s < w.s1;) {
            const int e_end = piece_end(w, s);
            if (s == w.s0) build(s);
            if (starts_build(w, s)) ++cur_b;
            // the next expert run's operand, ahead of this piece's epilogue
            if (e_end < w.s1 && starts_build(w, e_end)) build(e_end);
            const float* csb = cs + (cur_b & 1) * ncap;
            const int item = s / w.spi;
            const int jd = item / w.tiles, tile = item - jd * w.tiles;
            const int ne = sh.ucnt[jd], N = ne * J, npad = (N + 15) & ~15;
            const int d = pc & 1;
            const int row = tile * 128 + et;
            // the expert's tensor scales
            const float* tsp = reinterpret_cast<const float*>(p.experts + (size_t)sh.uexp[jd] * p.rec_bytes + 3 * nq + 3 * ns);
            const float ts0 = __ldg(tsp + (PHASE == NV_GATEUP ? 0 : 2)), ts1 = __ldg(tsp + 1);
            float P[NM][8];
#pragma unroll
            for (int m = 0; m < NM; ++m)
#pragma unroll
                for (int i = 0; i < 8; ++i) P[m][i] = 0.f;
            if (!dead) dead = !mbar_wait(&tfull[d], (pc >> 1) & 1, abort_flag, kNvWaitLimit);
            dead = __any_sync(0xffffffffu, dead);
            if (!dead) {
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(32 * sub) << 16) + kColD + d * 128;
#pragma unroll
                for (int m = 0; m < NM; ++m) {
#pragma unroll
                    for (int c0 = 0; c0 < kNvMaxN; c0 += 16) {
                        if (c0 < npad) {
                            uint32_t v[16];
                            __syncwarp();
                            tmem_ld_32x32b_x16(taddr + m * 64 + c0, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int u = 0; u < 16; ++u) {
                                const int n = c0 + u;
                                if (n < N) P[m][n / J] = fmaf(csb[n], __uint_as_float(v[u]), P[m][n / J]);
                            }
                        }
                    }
                }
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(&tempty[d]);
            const int a0 = item * w.spi, a1 = a0 + w.spi;
            const bool whole = a0 >= w.s0 && a1 <= w.s1;
            bool finish = whole;
            if (!whole) {
                const int slot = a0 < w.s0 ? 0 : 1;
                float* dst = wpart + (size_t)((blockIdx.x * 2 + slot) * NM) * 1024;
#pragma unroll
                for (int m = 0; m < NM; ++m)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (i < ne) dst[m * 1024 + i * 128 + et] = P[m][i];
                __threadfence();
                named_bar_sync(2, 128);
                const int c_first = w.cta_of(a0), c_last = w.cta_of(a1 - 1);
                if (et == 0) sh.last = atomicAdd(p.wtick + item, 1) == c_last - c_first;
                named_bar_sync(2, 128);
                finish = sh.last != 0;
                if (finish) {
                    __threadfence();
#pragma unroll
                    for (int m = 0; m < NM; ++m)
#pragma unroll
                        for (int i = 0; i < 8; ++i) P[m][i] = 0.f;
                    for (int c = c_first; c <= c_last; ++c) {
                        const int sl = a0 < w.start(c) ? 0 : 1;
                        const float* src = wpart + (size_t)((c * 2 + sl) * NM) * 1024;
#pragma unroll
                        for (int m = 0; m < NM; ++m)
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                if (i < ne) P[m][i] += __ldcg(src + m * 1024 + i * 128 + et);
                    }
                    if (et == 0) p.wtick[item] = 0;
                }
                named_bar_sync(2, 128);
            }
            if (finish && !dead) {
                const int u0 = sh.uoff[jd];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i >= ne) break;
                    if (PHASE == NV_GATEUP) {
                        const float g = P[0][i] * ts0, u = P[NM - 1][i] * ts1;
                        p.z16[(size_t)(u0 + i) * p.F + row] = half_checked(silu(g) * u, bad);
                    } else {
                        const float o = sh.slot_w[u0 + i] * ts0 * P[0][i];
                        p.o16w[(size_t)(u0 + i) * p.L + row] = half_checked(o, bad);
                    }
                }
            }
            ++pc;
            s = e_end;
        }
        report_range(p.ctrl, bad);
    }

    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) set_status(p.ctrl, LMOE_ERR_TIMEOUT);
    if (warp == 8) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int PHASE>
size_t nv_smem_bytes(const FwdParams& p, int ncap) {
    using Geo = NvGeom<PHASE>;
    const int K = PHASE == NV_GATEUP ? p.L : p.F;
    return 1024 + (size_t)Geo::STAGES * Geo::NM * (kCodeBox + kScaleBox) + (size_t)ncap * (K / 2) +
           (size_t)ncap * (K / 16) + 2 * ncap * sizeof(float) + (2 * Geo::STAGES + 7) * 8 + 16;
}

int nv_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    }
    return n;
}

template <int PHASE, int J>
cudaError_t launch_nvf4(const FwdParams& p, cudaStream_t st) {
    NvArgs a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.ncap = (p.T * J + 15) & ~15;
    const size_t smem = nv_smem_bytes<PHASE>(p, a.ncap);
    auto kern = k_nvf4<PHASE, J>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(nv_sms(), kNvMaxCtas);
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kNvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    stage_mark(st);
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

// Whether the tensor-core expert phases take this step: NVFP4 records, at
// most 8 tokens, 128-row tiles and 64-column MMA steps that divide the
// matrices, TMA-aligned records, and room in shared memory.
bool nvf4_usable(const FwdParams& p) {
    if (p.efmt != LMOE_EXPERTS_NVFP4 || p.T < 1 || p.T > 8) return false;
    if (p.F % 128 || p.L % 128 || p.F % 64 || p.L % 64) return false;
    if (p.L > kNvMaxK || p.F > kNvMaxK) return false;
    if (p.rec_bytes % 16 || (reinterpret_cast<uintptr_t>(p.experts) & 15)) return false;
    if (nv_sms() > kNvMaxCtas) return false;
    const int ncap = (p.T * (p.act == LMOE_ACT_NVFP4 ? kNvJW4A4 : kNvJExact) + 15) & ~15;
    return nv_smem_bytes<NV_GATEUP>(p, ncap) <= 227 * 1024 && nv_smem_bytes<NV_DOWN>(p, ncap) <= 227 * 1024;
}

// Workspace floats the phases' partial sums need (2 pieces per CTA).
size_t nvf4_part_floats() { return (size_t)kNvMaxCtas * 2 * 2 * 1024; }

// W4A4 (p.act == LMOE_ACT_NVFP4): one E2M1 term per activation row, the
// NVFP4 activation rule of include/lmoe.h; otherwise six terms (fp16-level).
cudaError_t run_nvf4_gateup(const FwdParams& p, cudaStream_t st) {
    return p.act == LMOE_ACT_NVFP4 ? launch_nvf4<NV_GATEUP, kNvJW4A4>(p, st) : launch_nvf4<NV_GATEUP, kNvJExact>(p, st);
}
cudaError_t run_nvf4_down(const FwdParams& p, cudaStream_t st) {
    return p.act == LMOE_ACT_NVFP4 ? launch_nvf4<NV_DOWN, kNvJW4A4>(p, st) : launch_nvf4<NV_DOWN, kNvJExact>(p, st);
}

}  // namespace lmoe
