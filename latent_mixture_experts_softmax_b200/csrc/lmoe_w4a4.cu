// W4A4 expert GEMMs of the many-token (prefill) path: NVFP4 weights times
// NVFP4 activations on the tensor cores (tcgen05.mma kind::mxf4nvf4).
//
// The teardown article's "What is 4-bit" section defines NVFP4: E2M1 codes
// with one E4M3 scale per 16 elements and an fp32 scale per matrix.  In the
// W4A4 mode (lmoe_cfg.act_fmt) the experts' inputs take the same form: each
// activation row (h for gate/up, z for down, both staged in fp16 by the
// kernel before) gets one fp32 scale G = max|v| / (6 * 448), per 16 elements
// the smallest E4M3 scale s >= max|v_block| / (6 G), and E2M1 codes nearest
// (ties to even, saturating) to v / (s G).  k_act_quant writes them; the GEMM
// multiplies codes and scales as stored and applies G (per column) and the
// weight matrix's fp32 scale in its epilogue.
//
// Layouts written by k_act_quant for n rows of K columns:
//   codes [K/32][n][16 B]  (a 32-column chunk of consecutive rows is
//                           contiguous: the no-swizzle K-major operand layout)
//   scale words [K/64][n]  (byte j of row r's word: block 4k + j)
//   G [n]
//
// The GEMM (one CTA per SM, persistent over its items): an item is one
// expert token tile (at most 128 slots, from the tile list the bucketing
// kernels built) times one 128-row tile of the weight operand, over the whole
// K in 256-column stages.  For gate/up the 128 rows are 64 output rows of
// both matrices, interleaved by TMEM subpartition: lanes 0-15 of
// subpartition b hold gate rows m0 + 16b .. m0 + 16b + 15 and lanes 16-31 the
// up rows of the same outputs, so the SwiGLU pairs meet by a warp shuffle.
// Warps:
//   0-3  loaders: per stage, thread r copies operand row r (its codes and
//        E4M3 scale words) and activation slot r with cp.async into a ring of
//        STAGES shared-memory slots, STAGES - 2 stages ahead of the MMA (one
//        slot of slack); once a stage has landed, each warp copies its
//        weight and activation scale words to its 32-lane TMEM subpartition
//        (scale columns 4k + b: rows / slots b*32 .. b*32+31)
//   4-11 epilogue: accumulators (TMEM, two buffers) -> * G * ts -> SwiGLU
//        (gate/up) or routing weight (down) -> fp16 zperm / operm; warps w
//        and w + 4 read TMEM subpartition w & 3, alternate 16-column chunks
//   12   MMA issue (one thread), TMEM allocation

#include <cstring>

#include "lmoe_prefill.cuh"

namespace lmoe {
namespace {

using namespace sm100;

constexpr int kW4Threads = 416;   // 4 loader warps, 8 epilogue warps, 1 MMA warp
constexpr int kW4MmaWarp = 12;
constexpr uint64_t kW4WaitLimit = 4000000000ull;   // SM cycles per barrier wait (about 2 s)
constexpr uint32_t kW4TmemCols = 512;
constexpr int kW4CodeBox = 128 * 128;    // bytes: 8 chunks x 128 rows x 16 B
constexpr int kW4ScaleBox = 4 * 128 * 4; // bytes: 4 64-column groups x 128 rows x 4 B

// 256-column stages of 36 KB (weight codes and scale words of 128 rows,
// activation codes and scale words of up to 128 slots); six fill 216 KB.
constexpr int kW4Stages = 6;
constexpr int kW4Ahead = kW4Stages - 2;
constexpr int kW4StageBytes = 2 * (kW4CodeBox + kW4ScaleBox);
constexpr uint32_t kW4ColSfa = 256, kW4ColSfb = 256 + 16 * kW4Stages;
static_assert(kW4ColSfb + 16 * kW4Stages <= kW4TmemCols, "TMEM columns");

struct __align__(64) W4Args {
    PrefillParams p;
    const uint8_t* aq;     // activation codes [K/32][n][16]
    const uint32_t* asf;   // activation scale words [K/64][n]
    const float* aG;       // [n]
    int n;                 // activation rows (T * K slots)
};

__device__ __forceinline__ void cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint64_t sdesc_plain(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return ((uint64_t)((saddr & 0x3FFFF) >> 4)) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}

__host__ __device__ constexpr uint32_t idesc_fp4(int N) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ void tst_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tst_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tld_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ uint32_t e4m3_code_rn(float s) {
    uint16_t h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.f), "f"(s));
    return h & 0xFFu;
}
__device__ __forceinline__ float e4m3_val(uint32_t c) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(c));
    return __half2float(__ushort_as_half((uint16_t)(r & 0xFFFFu)));
}
__device__ __forceinline__ uint32_t e2m1_pair(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One warp per activation row: the NVFP4 activation rule (module comment).
__global__ void __launch_bounds__(256) k_act_quant(const __half* src, int n, int K, uint8_t* codes, uint32_t* sfw,
                                                   float* G) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + warp;
    if (row >= n) return;
    const __half* r = src + (size_t)row * K;
    float amax = 0.f;
    for (int c = lane; c < K / 8; c += 32) {
        const uint4 v = __ldcg(reinterpret_cast<const uint4*>(r) + c);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w4[u]));
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float g = amax > 0.f ? amax * (1.f / (6.f * 448.f)) : 1.f;
    if (lane == 0) G[row] = g;
    uint8_t* sb = reinterpret_cast<uint8_t*>(sfw);
    for (int b = lane; b < K / 16; b += 32) {
        const uint4 v0 = __ldcg(reinterpret_cast<const uint4*>(r + 16 * b));
        const uint4 v1 = __ldcg(reinterpret_cast<const uint4*>(r + 16 * b) + 1);
        const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        float x[16];
        float bmax = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w8[u]));
            x[2 * u] = f.x;
            x[2 * u + 1] = f.y;
            bmax = fmaxf(bmax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
        uint32_t sc = 0, lo = 0, hi = 0;
        if (bmax > 0.f) {
            const float s = bmax / (6.f * g);
            sc = e4m3_code_rn(s);
            if (e4m3_val(sc) < s && sc < 0x7Eu) ++sc;
            const float inv = 1.f / (e4m3_val(sc) * g);
#pragma unroll
            for (int e = 0; e < 4; ++e) lo |= e2m1_pair(x[2 * e] * inv, x[2 * e + 1] * inv) << (8 * e);
#pragma unroll
            for (int e = 0; e < 4; ++e) hi |= e2m1_pair(x[8 + 2 * e] * inv, x[8 + 2 * e + 1] * inv) << (8 * e);
        }
        *reinterpret_cast<uint2*>(codes + ((size_t)(b >> 1) * n + row) * 16 + (b & 1) * 8) = make_uint2(lo, hi);
        sb[((size_t)(b >> 2) * n + row) * 4 + (b & 3)] = (uint8_t)sc;
    }
}

template <int KIND>
__global__ void __launch_bounds__(kW4Threads, 1) k_w4a4(const __grid_constant__ W4Args a) {
    constexpr int STAGES = kW4Stages, LA = kW4Ahead;
    const PrefillParams& p = a.p;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int K = KIND == G_GATEUP ? p.L : p.F;
    const int R = KIND == G_GATEUP ? p.F : p.L;
    const int mt = KIND == G_GATEUP ? R / 64 : R / 128;
    // slot s: weight codes [8][128][16] | weight scale words [4][128] |
    //         activation codes [8][128][16] | activation scale words [4][128]
    uint8_t* ring = smem;
    float* meta = reinterpret_cast<float*>(ring + STAGES * kW4StageBytes);   // [2 buffers][G | weight][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(meta + 512);
    uint64_t* full = bars;               // [STAGES] (4 loader warps)
    uint64_t* empty = full + STAGES;     // [STAGES] (commit)
    uint64_t* tfull = empty + STAGES;    // [2] item accumulated (commit)
    uint64_t* tempty = tfull + 2;        // [2] accumulator read (4 epilogue warps)
    uint64_t* final_bar = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kW4MmaWarp) {
        __syncwarp();
        tmem_alloc(tmem_slot, kW4TmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the tile list and counts are complete: this grid follows the bucketing
    // and quantisation kernels in the stream
    const int n_items = __ldcg(p.n_etiles) * mt;
    const int spi = (K + 255) / 256;
    const size_t nq = (size_t)p.L * p.F / 2, ns = (size_t)p.L * p.F / 16;
    // item i: the expert tile {expert, first slot, slots} (fetched one item
    // ahead by every role) and the row tile
    auto tile_of = [&](int i) -> int4 {
        return i < n_items ? __ldcg(p.etile + i / mt) : make_int4(0, 0, 0, 0);
    };
    auto m0_of = [&](int i) { return (i % mt) * (KIND == G_GATEUP ? 64 : 128); };

    if (warp < 4) {
        // -------------------------------------------------------- loaders
        const int r = threadIdx.x;    // operand row and activation slot of this thread
        bool dead = false;
        int n_st = 0;
        for (int i = blockIdx.x; i < n_items; i += gridDim.x) n_st += spi;
        int it_item = blockIdx.x, q = 0;
        const uint8_t* wq = nullptr;   // this row's codes, chunk 0
        const uint8_t* wsc = nullptr;  // this row's scale words, group 0
        const uint8_t* aq = nullptr;   // this slot's codes, chunk 0 (nullptr: past the tile)
        const uint32_t* as = nullptr;
        int4 nxt = tile_of(it_item);
        auto start_item = [&]() {
            const int4 d = nxt;
            nxt = tile_of(it_item + gridDim.x);
            const int mat = d.x, b0 = d.y, nrow = d.z, m0 = m0_of(it_item);
            const uint8_t* rec = p.experts + (size_t)mat * p.rec_bytes;
            int m = 2, row = m0 + r;
            if (KIND == G_GATEUP) {
                m = (r & 31) >> 4;                                   // 0 gate, 1 up
                row = m0 + 16 * (r >> 5) + (r & 15);
            }
            wq = rec + m * nq + (size_t)row * 16;
            wsc = rec + 3 * nq + m * ns + (size_t)row * 4;
            aq = r < nrow ? a.aq + (size_t)(b0 + r) * 16 : nullptr;
            as = r < nrow ? a.asf + b0 + r : nullptr;
        };
        if (it_item < n_items) start_item();
        const size_t wstep = (size_t)R * 16, sstep = (size_t)R * 4, astep = (size_t)a.n * 16;
        for (int i = 0; i < n_st + LA; ++i) {
            if (i < n_st) {
                const int slot = i % STAGES;
                if (!dead) dead = !mbar_wait(&empty[slot], ((i / STAGES) & 1) ^ 1, abort_flag, kW4WaitLimit);
                if (!dead) {
                    uint8_t* sl = ring + slot * kW4StageBytes;
                    const int nch = min(8, K / 32 - q * 8), ngr = min(4, K / 64 - q * 4);
                    const uint8_t* wqq = wq + (size_t)(q * 8) * wstep;
                    const uint8_t* wss = wsc + (size_t)(q * 4) * sstep;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        if (c < nch) cp16(sl + c * 2048 + r * 16, wqq + c * wstep);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        if (g < ngr) cp4(sl + kW4CodeBox + g * 512 + r * 4, wss + g * sstep);
                    if (aq) {
                        const uint8_t* aqq = aq + (size_t)(q * 8) * astep;
                        const uint32_t* ass = as + (size_t)(q * 4) * a.n;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (c < nch) cp16(sl + kW4CodeBox + kW4ScaleBox + c * 2048 + r * 16, aqq + c * astep);
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            if (g < ngr) cp4(sl + 2 * kW4CodeBox + kW4ScaleBox + g * 512 + r * 4, ass + (size_t)g * a.n);
                    }
                }
                if (++q == spi) {
                    q = 0;
                    it_item += gridDim.x;
                    if (it_item < n_items) start_item();
                }
            }
            cp_commit();
            if (i >= LA) {
                const int slot = (i - LA) % STAGES;
                cp_wait<LA>();
                fence_proxy_async_smem();
                dead = __any_sync(0xffffffffu, dead);
                named_bar_sync(1, 128);
                if (!dead) {
                    // scale words: lane a of warp w holds rows / slots a + 32b in columns 4k + b
                    const uint32_t* sw = reinterpret_cast<const uint32_t*>(ring + slot * kW4StageBytes + kW4CodeBox);
                    const uint32_t* sa =
                        reinterpret_cast<const uint32_t*>(ring + slot * kW4StageBytes + 2 * kW4CodeBox + kW4ScaleBox);
                    uint32_t v[16], u[16];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
#pragma unroll
                        for (int bb = 0; bb < 4; ++bb) {
                            v[k * 4 + bb] = sw[k * 128 + lane + 32 * bb];
                            u[k * 4 + bb] = sa[k * 128 + lane + 32 * bb];
                        }
                    const uint32_t lanes = (uint32_t)(32 * warp) << 16;
                    __syncwarp();
                    tst_x16(tmem_base + lanes + kW4ColSfa + (uint32_t)(slot * 16), v);
                    tst_x16(tmem_base + lanes + kW4ColSfb + (uint32_t)(slot * 16), u);
                    __syncwarp();
                    tst_wait();
                    tc_fence_before();
                }
                __syncwarp();
                if (lane == 0 && !dead) mbar_arrive(&full[slot]);
            }
        }
        cp_wait<0>();
    } else if (warp == kW4MmaWarp) {
        // -------------------------------------------------------- MMA issue
        if (lane == 0) {
            uint32_t it = 0, pc = 0;
            bool dead = false, issued = false;
            int4 nxt = tile_of(blockIdx.x);
            for (int i = blockIdx.x; i < n_items && !dead; i += gridDim.x, ++pc) {
                const int nrow = nxt.z;
                nxt = tile_of(i + gridDim.x);
                const uint32_t idesc = idesc_fp4((nrow + 15) & ~15);
                const uint32_t acc = pc & 1;
                if (!mbar_wait(&tempty[acc], ((pc >> 1) & 1) ^ 1, abort_flag, kW4WaitLimit)) { dead = true; break; }
                tc_fence_after();
                for (int q = 0; q < spi; ++q, ++it) {
                    const int slot = it % STAGES;
                    if (!mbar_wait(&full[slot], (it / STAGES) & 1, abort_flag, kW4WaitLimit)) { dead = true; break; }
                    tc_fence_after();
                    const uint32_t sl = smem_u32(ring + slot * kW4StageBytes);
                    const int kk = min(4, (K - q * 256) / 64);
                    for (int k = 0; k < kk; ++k) {
                        const uint64_t adesc = sdesc_plain(sl + (uint32_t)(k * 4096), 2048, 128);
                        const uint64_t bdesc = sdesc_plain(sl + kW4CodeBox + kW4ScaleBox + (uint32_t)(k * 4096), 2048, 128);
                        umma_fp4(tmem_base + acc * 128, adesc, bdesc, idesc, tmem_base + kW4ColSfa + (uint32_t)(slot * 16 + 4 * k),
                                 tmem_base + kW4ColSfb + (uint32_t)(slot * 16 + 4 * k), (q > 0 || k > 0) ? 1u : 0u);
                    }
                    issued = true;
                    umma_commit(&empty[slot]);
                }
                if (dead) break;
                umma_commit(&tfull[acc]);
            }
            if (issued) {
                // every MMA done before TMEM is freed, even after an abort
                umma_commit(final_bar);
                volatile int no_abort = 0;
                mbar_wait(final_bar, 0, &no_abort, kW4WaitLimit);
            }
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------- epilogue (warps 4-11)
        // Warps w and w + 4 share TMEM subpartition w & 3 and take alternate
        // 16-column chunks of the accumulator.
        const int et = threadIdx.x - 128;
        const int sub = warp & 3, half = (warp - 4) >> 2;
        uint32_t pc = 0;
        bool dead = false, bad = false;
        // the next item's tile, per-slot scales (G; the routing weight for
        // down) and tensor scales are fetched while this item drains
        int4 cur = tile_of(blockIdx.x), nxt = tile_of(blockIdx.x + gridDim.x);
        float nG = 0.f, nW = 0.f, nts0 = 0.f, nts1 = 0.f;
        auto fetch = [&](const int4& d, float& g, float& w, float& t0, float& t1) {
            if (et < d.z) {
                g = __ldcg(a.aG + d.y + et);
                if (KIND == G_DOWN) w = __ldcg(p.wslot + d.y + et);
            }
            const float* tsp = reinterpret_cast<const float*>(p.experts + (size_t)d.x * p.rec_bytes + 3 * nq + 3 * ns);
            t0 = __ldg(tsp + (KIND == G_GATEUP ? 0 : 2));
            t1 = __ldg(tsp + 1);
        };
        if (blockIdx.x < n_items) fetch(cur, nG, nW, nts0, nts1);
        for (int i = blockIdx.x; i < n_items; i += gridDim.x, ++pc) {
            const int mat = cur.x, b0 = cur.y, nrow = cur.z, m0 = m0_of(i);
            (void)mat;
            const uint32_t acc = pc & 1;
            // per slot of the item, the factor of each accumulator column:
            // G * gate (up) tensor scale, or G * down tensor scale * routing weight
            float* mA = meta + acc * 256;
            float* mB = mA + 128;
            if (et < nrow) {
                mA[et] = KIND == G_DOWN ? nG * nts0 * nW : nG * nts0;
                if (KIND == G_GATEUP) mB[et] = nG * nts1;
            }
            const bool more = i + gridDim.x < n_items;
            if (more) fetch(nxt, nG, nW, nts0, nts1);
            named_bar_sync(2, 256);
            if (!dead) dead = !mbar_wait(&tfull[acc], (pc >> 1) & 1, abort_flag, kW4WaitLimit);
            dead = __any_sync(0xffffffffu, dead);
            if (!dead) {
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(32 * sub) << 16) + acc * 128;
                const bool hi = lane >= 16;
                const int row = KIND == G_GATEUP ? m0 + 16 * sub + (lane & 15) : m0 + 32 * sub + lane;
                for (int c0 = 16 * half; c0 < nrow; c0 += 32) {
                    uint32_t v[16];
                    __syncwarp();
                    tld_x16(taddr + c0, v);
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    if (KIND == G_GATEUP) {
                        // lanes < 16: gate of columns c0..c0+7, partner's up; lanes >= 16:
                        // partner's gate of columns c0+8..c0+15, own up
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const float mine = __uint_as_float(hi ? v[u + 8] : v[u]);
                            const float other = __shfl_xor_sync(0xffffffffu, __uint_as_float(hi ? v[u] : v[u + 8]), 16);
                            const int s = c0 + u + (hi ? 8 : 0);
                            if (s < nrow) {
                                const float gv = (hi ? other : mine) * mA[s], uv = (hi ? mine : other) * mB[s];
                                p.zperm[(size_t)(b0 + s) * p.F + row] = half_checked(silu(gv) * uv, bad);
                            }
                        }
                    } else {
#pragma unroll
                        for (int u = 0; u < 16; ++u) {
                            const int s = c0 + u;
                            if (s < nrow) p.operm[(size_t)(b0 + s) * p.L + row] = half_checked(__uint_as_float(v[u]) * mA[s], bad);
                        }
                    }
                }
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(&tempty[acc]);
            cur = nxt;
            nxt = tile_of(i + 2 * gridDim.x);
        }
        report_range(p.ctrl, bad);
    }

    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) set_status(p.ctrl, LMOE_ERR_TIMEOUT);
    if (warp == kW4MmaWarp) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc(tmem_base, kW4TmemCols);
    }
}

int w4_sms() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    }
    return n;
}

constexpr size_t kW4Smem = 1024 + (size_t)kW4Stages * kW4StageBytes + 512 * 4 + (2 * kW4Stages + 5) * 8 + 16;

template <int KIND>
cudaError_t launch_w4a4(const PrefillParams& p, const uint8_t* aq, const uint32_t* asf, const float* aG, int n,
                        cudaStream_t st) {
    W4Args a;
    std::memset(&a, 0, sizeof(a));
    a.p = p;
    a.aq = aq;
    a.asf = asf;
    a.aG = aG;
    a.n = n;
    const size_t smem = kW4Smem;
    auto kern = k_w4a4<KIND>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(w4_sms());
    cfg.blockDim = dim3(kW4Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    // a plain launch: the kernel reads the activation codes the kernel
    // before it writes (its grid-dependency waits are then no-ops)
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

// Quantise n fp16 rows of K columns to NVFP4 activations (layouts in the
// module comment).
cudaError_t run_act_quant(const __half* src, int n, int K, uint8_t* codes, uint32_t* sfw, float* G, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    k_act_quant<<<(n + 7) / 8, 256, 0, st>>>(src, n, K, codes, sfw, G);
    return cudaGetLastError();
}

cudaError_t run_w4a4_gateup(const PrefillParams& p, const uint8_t* aq, const uint32_t* asf, const float* aG, int n,
                            cudaStream_t st) {
    return launch_w4a4<G_GATEUP>(p, aq, asf, aG, n, st);
}

cudaError_t run_w4a4_down(const PrefillParams& p, const uint8_t* aq, const uint32_t* asf, const float* aG, int n,
                          cudaStream_t st) {
    return launch_w4a4<G_DOWN>(p, aq, asf, aG, n, st);
}

}  // namespace lmoe
