// Latent-MoE block for many tokens (prefill): the dense contractions run on
// the 5th-generation tensor cores (tcgen05.mma, fp32 accumulators in TMEM)
// in one warp-specialised, persistent GEMM kernel template:
//
//   warps 0-3   epilogue: TMEM -> registers -> fused epilogue -> global
//   warps 4-11  converters: the weight operand is read from its storage
//               format (Q8_0, Q4_0, NVFP4, Q3_K / IQ4_NL), dequantised in
//               registers and written to shared memory in the UMMA K-major
//               128-byte-swizzled layout
//   warp 12     TMEM allocation and the single-thread UMMA issue
//   warp 13     TMA of the activation operand (and of bf16 weights)
//
// Operands are swapped with respect to the usual "tokens x weights" view:
// the weight rows are the MMA's M = 128 side and the tokens (or expert
// slots) are its N side, so one dequantised weight tile feeds up to 256
// tokens; the NVFP4 expert GEMMs take two 128-row weight tiles per item
// against each activation stage.  Every accumulator is fp32 in TMEM,
// double-buffered so the epilogue of one tile overlaps the main loop of the
// next.
//
// GEMMs of the block (teardown article "Edge0-145B: a Qwen MoE with its
// experts squeezed", section "A latent in front of the experts"; Edge0
// 145B / 120B model page, architecture tables):
//   ROUTER        logits[t][e]   = W_r[e] . x_t + b_e          (bf16 x bf16)
//   SHARED_GATEUP z_sh[t][f]     = silu(S_gate x_t) * (S_up x_t)  (bf16)
//   DPROJ         h[slot][l]     = (D_g x_t)[l] for every slot (t, k) with
//                                  group(e_k) = g               (fp16)
//   GATEUP        z[slot][f]     = silu(W_gate h) * (W_up h)    (fp16)
//   DOWN          o[slot][l]     = w_slot * (W_down z)[l]       (fp16)
//   UPROJ         y[t]           = sum_g U_g s[t][g] + S_down z_sh[t]
//                                  (+ residual)                 (fp16)
// with s[t][g] = sum of o over the token's experts of group g (combine
// kernel).  The routing, bucketing and combine steps are plain CUDA kernels
// in this file.

#include "lmoe_prefill.cuh"
#include "lmoe_q3k.cuh"

namespace lmoe {

using namespace sm100;

constexpr uint64_t kWaitLimit = 4000000000ull;   // SM cycles per barrier wait (about 2 s)

// ---------------------------------------------------------------------------
// tiles
// ---------------------------------------------------------------------------

struct TileRef {
    int valid;
    int mat;      // group (DPROJ) or expert (GATEUP / DOWN)
    int m0;       // first A row of the tile (feature)
    int b0;       // first B row (token or slot)
    int n;        // valid B rows
    int nq;       // token tile index (UPROJ / DPROJ hit flags)
    int na;       // 128-row A tiles of the item (2 in the two-tile expert GEMMs, else 1)
    int piece;    // U: -1 for a whole tile, else the piece of a split tile (its segment range)
    int part;     // U: the piece's segment range
};

// MA = 2 (expert GEMMs only): an item covers two 128-row A tiles that share
// each B stage, two MMAs per K step into two accumulators.  Gate/up: tile a
// holds gate and up rows m0 + 64a .. m0 + 64a + 63; down: rows m0 + 128a ..
// m0 + 128a + 127.  The last item of a matrix may have one.
template <int KIND, int NT, int MA = 1>
struct Sched {
    static_assert(MA == 1 || KIND == G_GATEUP || KIND == G_DOWN, "two A tiles: expert GEMMs only");
    __device__ static int m_tiles(const PrefillParams& p) {
        switch (KIND) {
            case G_ROUTER: return p.E / 128;
            case G_SHARED_GATEUP: return p.Fs / 64;
            case G_DPROJ: return p.G * (p.L / 128);
            case G_GATEUP: return (p.F / 64 + MA - 1) / MA;
            case G_DOWN: return (p.L / 128 + MA - 1) / MA;
            default: return p.H / 128;
        }
    }
    __device__ static int num_tiles(const PrefillParams& p) {
        if (KIND == G_GATEUP || KIND == G_DOWN) return m_tiles(p) * __ldcg(p.n_etiles);
        const int n = m_tiles(p) * ((p.T + NT - 1) / NT);
        if (KIND == G_UPROJ && p.u_parts > 1) return p.u_whole + (n - p.u_whole) * p.u_parts;
        return n;
    }
    __device__ static TileRef get(const PrefillParams& p, int i) {   // i: the work item
        TileRef t;
        const int mt = m_tiles(p);
        t.valid = 1;
        t.mat = 0;
        t.na = 1;
        t.piece = -1;
        t.part = -1;
        if (KIND == G_UPROJ && p.u_parts > 1 && i >= p.u_whole) {
            // a piece of a tile of the last wave
            t.piece = i - p.u_whole;
            t.part = t.piece % p.u_parts;
            i = p.u_whole + t.piece / p.u_parts;
        }
        if (KIND == G_GATEUP || KIND == G_DOWN) {
            // consecutive tiles share the expert's token rows
            const int et = i / mt, m = i % mt;
            const int4 d = __ldcg(p.etile + et);
            const int rows = KIND == G_GATEUP ? 64 : 128;           // output rows per A tile
            t.mat = d.x;
            t.m0 = m * rows * MA;
            t.b0 = d.y;
            t.n = min(NT, d.z);
            t.nq = 0;
            t.na = min(MA, ((KIND == G_GATEUP ? p.F : p.L) - t.m0) / rows);
        } else {
            // consecutive tiles share the weight tile (token tiles fastest),
            // except U: there the token tile's B operand (the group sums s
            // of every hit group, 28 KB a token at the Edge0 shapes) is what
            // outgrows L2 when all of it is in flight, so consecutive tiles
            // share the token tile and its B stages (weight tiles fastest)
            const int ntt = (p.T + NT - 1) / NT;
            const int m = KIND == G_UPROJ ? i % mt : i / ntt, q = KIND == G_UPROJ ? i / mt : i % ntt;
            t.nq = q;
            t.b0 = q * NT;
            t.n = min(NT, p.T - t.b0);
            if (KIND == G_DPROJ) {
                const int mpg = p.L / 128;
                t.mat = m / mpg;
                t.m0 = (m % mpg) * 128;
                t.valid = p.dhit[q * p.G + t.mat] != 0;
            } else if (KIND == G_SHARED_GATEUP) {
                t.m0 = m * 64;
            } else {
                t.m0 = m * 128;
            }
        }
        return t;
    }
    // UPROJ: one segment per group, then the shared expert's down projection.
    // ROUTER / SHARED_GATEUP on a normalised input: the input is split into
    // bf16 high and low parts, one segment each, so the products stay exact.
    // UPROJ segments G and G + 1: the shared expert's down projection on the
    // bf16 high and low parts of its hidden activations.
    __device__ static int num_segs(const PrefillParams& p) {
        if (KIND == G_UPROJ) return p.G + 2;
        if (KIND == G_ROUTER || KIND == G_SHARED_GATEUP) return p.xr ? 2 : 1;
        return 1;
    }
    __device__ static bool seg_active(const PrefillParams& p, const TileRef& t, int seg) {
        if (KIND != G_UPROJ) return true;
        if (t.part >= 0 && (seg < p.u_segb[t.part] || seg >= p.u_segb[t.part + 1])) return false;
        return seg >= p.G || p.dhit[t.nq * p.G + seg] != 0;
    }
    __device__ static int seg_k(const PrefillParams& p, int seg) {
        switch (KIND) {
            case G_ROUTER:
            case G_SHARED_GATEUP:
            case G_DPROJ: return p.H;
            case G_GATEUP: return p.L;
            case G_DOWN: return p.F;
            default: return seg >= p.G ? p.Fs : p.L;
        }
    }
    // A of this segment comes through TMA (plain bf16 weights: router, shared
    // expert) rather than from the dequantising producers; those segments run
    // bf16 x bf16.
    __device__ static bool tma_a(const PrefillParams& p, int seg) {
        if (KIND == G_ROUTER || KIND == G_SHARED_GATEUP) return true;
        return KIND == G_UPROJ && seg >= p.G;
    }
    static constexpr bool kAnyTmaA = KIND == G_ROUTER || KIND == G_SHARED_GATEUP || KIND == G_UPROJ;
};

// Walks the (tile, segment, 64-wide K stage) sequence of one CTA.  The
// active segments of a tile are read once, when the tile is entered.
template <int KIND, int NT, int MA = 1>
struct Cursor {
    using S = Sched<KIND, NT, MA>;
    int tile, seg, ks, nk, ntiles;
    uint64_t segmask;
    bool done;
    TileRef t;
    __device__ void begin(const PrefillParams& p) {
        ntiles = S::num_tiles(p);
        tile = (int)blockIdx.x - (int)gridDim.x;
        done = false;
        next_tile(p);
    }
    __device__ void next_tile(const PrefillParams& p) {
        while (true) {
            tile += gridDim.x;
            if (tile >= ntiles) { done = true; return; }
            t = S::get(p, tile);
            if (!t.valid) continue;
            segmask = 0;
            for (int sg = 0; sg < S::num_segs(p); ++sg)
                if (S::seg_active(p, t, sg)) segmask |= 1ull << sg;
            seg = -1;
            if (next_seg(p)) return;
        }
    }
    // advance to the next active segment of the current tile; false if none
    __device__ bool next_seg(const PrefillParams& p) {
        const uint64_t higher = seg < 0 ? segmask : (segmask & ~((2ull << seg) - 1));
        if (!higher) return false;
        seg = __ffsll((long long)higher) - 1;
        ks = 0;
        nk = S::seg_k(p, seg) / 64;
        return true;
    }
    __device__ void next_stage(const PrefillParams& p) {
        if (++ks < nk) return;
        if (next_seg(p)) return;
        next_tile(p);
    }
    __device__ bool last_stage_of_tile(const PrefillParams& p) const {
        if (ks + 1 < nk) return false;
        return (segmask & ~((2ull << seg) - 1)) == 0;
    }
};

// ---------------------------------------------------------------------------
// weight operand: raw loads and dequantisation to fp16 (one row, 64 columns)
// ---------------------------------------------------------------------------

// Raw weight bytes of one A stage (128 rows x 64 columns) as they are stored,
// copied into a shared-memory slot by the TMA engine (1-D bulk copies):
//   [part 0 | part 1 | scales]
// part j = 32-column block (Q8_0 / Q4_0) or chunk (NVFP4) j of the stage,
// 128 rows x (32 | 16) bytes, row r at r * bytes; scales: Q8_0 / Q4_0 two
// fp16 arrays of 128 (block 0, block 1), NVFP4 one word per row.  For the
// gate/up tiles rows 0-63 are gate rows and 64-127 the matching up rows.
template <int KIND>
__host__ __device__ constexpr int raw_part_bytes(int du_fmt) {
    return KIND == G_DPROJ || KIND == G_UPROJ ? 128 * (du_fmt == LMOE_Q8_0 ? 32 : 16) : 128 * 16;
}
template <int KIND>
__host__ __device__ constexpr int raw_slot_bytes(int du_fmt) {
    return (KIND == G_ROUTER || KIND == G_SHARED_GATEUP) ? 0 : 2 * raw_part_bytes<KIND>(du_fmt) + 512;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void cp_async16_sh(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4_sh(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_grp() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_grp() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// 4 bytes holding values v+bias (0..255) -> two half2 of (1024 + byte)
__device__ __forceinline__ void bytes_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    lo = __byte_perm(w, 0x64646464u, 0x4140);
    hi = __byte_perm(w, 0x64646464u, 0x4342);
}

// The stored bytes one converter thread dequantises for one stage: half h
// (columns 32h .. 32h+31 of the 64-column stage) of row r of the tile.
struct RawHalf {
    uint4 a, b;      // codes (Q8_0: 32 bytes; Q4_0, NVFP4: 16 bytes in a)
    uint32_t s;      // scale: fp16 bits (Q8_0, Q4_0) or the row's four E4M3 bytes of the 64 columns (NVFP4)
};

// Fetch RawHalf of (row r, half h) of the cursor's stage with plain loads
// (read-only path; the bulk-copy engine's fixed cost per copy would cap a
// per-stage stream of small copies).
template <int KIND, int NT, class Cur>
__device__ __forceinline__ void fetch_raw(const PrefillParams& p, const Cur& c, int r, int h, RawHalf& o) {
    const int k0 = c.ks * 64;
    if (KIND == G_DPROJ || (KIND == G_UPROJ && c.seg < p.G)) {
        const int R = KIND == G_DPROJ ? p.L : p.H;
        const int C = KIND == G_DPROJ ? p.H : p.L;
        const uint8_t* mat = (KIND == G_DPROJ ? p.D : p.U) + (size_t)(KIND == G_DPROJ ? c.t.mat : c.seg) * p.du_bytes;
        const size_t rowb = p.du_fmt == LMOE_Q8_0 ? 32 : 16;
        const size_t e = (size_t)(k0 / 32 + h) * R + c.t.m0 + r;
        const uint4* q = reinterpret_cast<const uint4*>(mat + e * rowb);
        o.a = __ldg(q);
        if (p.du_fmt == LMOE_Q8_0) o.b = __ldg(q + 1);
        o.s = __ldg(reinterpret_cast<const uint16_t*>(mat + (size_t)R * C / 32 * rowb) + e);
    } else if ((KIND == G_GATEUP || KIND == G_DOWN) && p.efmt == LMOE_EXPERTS_Q3K) {
        const uint8_t* rec = p.experts + (size_t)c.t.mat * p.rec_bytes;
        const size_t gb = q3k_matrix_bytes(p.F, p.L);
        if (KIND == G_GATEUP) {
            // 32 columns e0 .. e0 + 31 of one 128-column half h of a Q3_K row:
            // lo words e0/16, e0/16 + 1; hi word e0/32; the half's 6 scale
            // bytes; the super-block d
            const int row = c.t.m0 + (r & 63), R = p.F;
            const uint8_t* m = rec + (r >> 6) * gb;
            const int col = k0 + 32 * h, hf = col / 128, e0 = col % 128;
            const size_t nh = (size_t)p.L / 128;
            const uint2 lo = __ldg(reinterpret_cast<const uint2*>(m + ((size_t)hf * R + row) * 32 + 4 * (e0 / 16)));
            const uint32_t hi = __ldg(reinterpret_cast<const uint32_t*>(m + nh * R * 32 + ((size_t)hf * R + row) * 16 + 4 * (e0 / 32)));
            const uint16_t* scp = reinterpret_cast<const uint16_t*>(m + nh * R * 48 + ((size_t)hf * R + row) * 6);
            const uint16_t d = __ldg(reinterpret_cast<const uint16_t*>(m + nh * R * 54) + (size_t)(col / 256) * R + row);
            o.a = make_uint4(lo.x, lo.y, hi, d);
            o.b = make_uint4(__ldg(scp), __ldg(scp + 1), __ldg(scp + 2), (uint32_t)(e0 / 16));
        } else {
            // IQ4_NL down [L][F]: 32-column block k0 / 32 + h of row m0 + r
            const uint8_t* m = rec + 2 * gb;
            const size_t e = (size_t)(k0 / 32 + h) * p.L + c.t.m0 + r;
            o.a = __ldg(reinterpret_cast<const uint4*>(m + e * 16));
            o.s = __ldg(reinterpret_cast<const uint16_t*>(m + (size_t)p.L * p.F / 2) + e);
        }
    } else if (KIND == G_GATEUP || KIND == G_DOWN) {
        const size_t nq = (size_t)p.L * p.F / 2, ns = (size_t)p.L * p.F / 16;
        const uint8_t* rec = p.experts + (size_t)c.t.mat * p.rec_bytes;
        const int R = KIND == G_GATEUP ? p.F : p.L;
        const int row = KIND == G_GATEUP ? c.t.m0 + (r & 63) : c.t.m0 + r;
        const int m = KIND == G_GATEUP ? (r >> 6) : 2;                  // gate, up, down
        o.a = __ldg(reinterpret_cast<const uint4*>(rec + (size_t)m * nq + ((size_t)(k0 / 32 + h) * R + row) * 16));
        o.s = __ldg(reinterpret_cast<const uint32_t*>(rec + 3 * nq + (size_t)m * ns + ((size_t)(k0 / 64) * R + row) * 4));
    }
}

// Two-tile expert items: the NVFP4 bytes of row rr of A tile a (both
// 32-column halves of the stage), copied into this thread's ring slot: code
// chunks at slot[0, 16) and [16, 32), the row's 4-byte scale word at
// slot[32, 36).
template <int KIND>
__device__ __forceinline__ void fetch_row_async(const PrefillParams& p, const TileRef& t, int ks, int a, int rr,
                                                uint8_t* slot) {
    const int k0 = ks * 64;
    const size_t nq = (size_t)p.L * p.F / 2, ns = (size_t)p.L * p.F / 16;
    const uint8_t* rec = p.experts + (size_t)t.mat * p.rec_bytes;
    const int R = KIND == G_GATEUP ? p.F : p.L;
    const int row = KIND == G_GATEUP ? t.m0 + 64 * a + (rr & 63) : t.m0 + 128 * a + rr;
    const int m = KIND == G_GATEUP ? (rr >> 6) : 2;                  // gate, up, down
    const uint8_t* q = rec + (size_t)m * nq + ((size_t)(k0 / 32) * R + row) * 16;
    cp_async16_sh(slot, q);
    cp_async16_sh(slot + 16, q + (size_t)R * 16);
    cp_async4_sh(slot + 32, rec + 3 * nq + (size_t)m * ns + ((size_t)(k0 / 64) * R + row) * 4);
}

// RawHalf of (row r, half h) -> 16 half2 of the row's 32 columns.
template <int KIND>
__device__ __forceinline__ void dequant_half(const PrefillParams& p, const RawHalf& raw, int h, uint32_t (&o)[16]) {
    if (KIND == G_DPROJ || KIND == G_UPROJ) {
        const __half2 d = __half2half2(__ushort_as_half((uint16_t)raw.s));
        if (p.du_fmt == LMOE_Q8_0) {
            const uint4 a = raw.a;
            const uint4 b = raw.b;
            const uint32_t w8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            const __half2 off = __float2half2_rn(1152.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t lo, hi;
                bytes_to_h2x2(w8[i] ^ 0x80808080u, lo, hi);
                o[2 * i] = h2_bits(__hmul2(__hsub2(bits_h2(lo), off), d));
                o[2 * i + 1] = h2_bits(__hmul2(__hsub2(bits_h2(hi), off), d));
            }
        } else {
            const uint4 a = raw.a;
            const uint32_t w4[4] = {a.x, a.y, a.z, a.w};
            const __half2 off = __float2half2_rn(1032.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t lo, hi;
                bytes_to_h2x2(w4[i] & 0x0F0F0F0Fu, lo, hi);
                o[2 * i] = h2_bits(__hmul2(__hsub2(bits_h2(lo), off), d));
                o[2 * i + 1] = h2_bits(__hmul2(__hsub2(bits_h2(hi), off), d));
                bytes_to_h2x2((w4[i] >> 4) & 0x0F0F0F0Fu, lo, hi);
                o[8 + 2 * i] = h2_bits(__hmul2(__hsub2(bits_h2(lo), off), d));
                o[8 + 2 * i + 1] = h2_bits(__hmul2(__hsub2(bits_h2(hi), off), d));
            }
        }
    } else if (p.efmt == LMOE_EXPERTS_Q3K && KIND == G_GATEUP) {
        // w = d * (sc_j - 32) * (q - 4): exact in fp32, one rounding to fp16
        const float d = __half2float(__ushort_as_half((uint16_t)raw.a.w));
        const uint64_t sc = (uint64_t)raw.b.x | ((uint64_t)raw.b.y << 16) | ((uint64_t)raw.b.z << 32);
        const int j0 = (int)raw.b.w;
        const uint32_t lo2[2] = {raw.a.x, raw.a.y};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = 2 * k + u, b = i % 4, ii = (i % 16) / 4;
                const int q = ((lo2[i / 16] >> (8 * b + 2 * ii)) & 3) | (((raw.a.z >> (8 * b + i / 4)) & 1) << 2);
                const int f = (int)((sc >> (6 * (j0 + i / 16))) & 63) - 32;
                v[u] = d * (float)(f * (q - 4));
            }
            o[k] = h2_bits(__floats2half2_rn(v[0], v[1]));
        }
    } else if (p.efmt == LMOE_EXPERTS_Q3K) {
        // IQ4_NL: w = d * level[q], one rounding to fp16
        const float d = __half2float(__ushort_as_half((uint16_t)raw.s));
        const uint32_t w4[4] = {raw.a.x, raw.a.y, raw.a.z, raw.a.w};
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            float v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = 2 * k + u, byte = (w4[(i % 16) / 4] >> (8 * (i % 4))) & 0xFF;
                v[u] = d * (float)iq4nl_level(i < 16 ? (byte & 15) : (byte >> 4));
            }
            o[k] = h2_bits(__floats2half2_rn(v[0], v[1]));
        }
    } else {
        const uint4 a = raw.a;
        const uint32_t sw = raw.s;
        const uint32_t s16 = (sw >> (16 * h)) & 0xFFFF;          // scales of columns 32h..+15 and +16..+31
        uint32_t sc;
        asm("{\n\t.reg .b16 a;\n\tcvt.u16.u32 a, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\t}" : "=r"(sc) : "r"(s16));
        const __half2 s_lo = __low2half2(bits_h2(sc)), s_hi = __high2half2(bits_h2(sc));
        const uint32_t w4[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t hv[4];
            e2m1x8_to_f16x8(w4[i], hv);
            const __half2 sc2 = i < 2 ? s_lo : s_hi;
#pragma unroll
            for (int j = 0; j < 4; ++j) o[4 * i + j] = h2_bits(__hmul2(bits_h2(hv[j]), sc2));
        }
    }
}

// Half h of row r of a 128-byte-swizzled K-major tile (16-byte chunks 4h..4h+3).
__device__ __forceinline__ void store_half_swizzled(uint8_t* tile, int r, int h, const uint32_t (&o)[16]) {
    uint8_t* row = tile + r * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int cc = 4 * h + c;
        *reinterpret_cast<uint4*>(row + ((cc ^ (r & 7)) << 4)) = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
    }
}

// ---------------------------------------------------------------------------
// epilogue
// ---------------------------------------------------------------------------

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// Per epilogue warp, a 32-column x 32-row fp16 transpose buffer: row-major
// outputs ([column][row], rows contiguous in memory) leave a warp as 16-byte
// stores of 8 rows of one column instead of 2-byte stores of one row.
constexpr int kTrPitch = 40;   // halves per buffered column (80 bytes: 16-byte aligned, spreads banks)

template <int KIND, int NT>
__device__ __forceinline__ void epilogue_chunk(const PrefillParams& p, const TileRef& t, int warp, int lane, int c0,
                                               const uint32_t (&r)[32], float* xchg, const float* tscale,
                                               uint16_t* trw) {
    const int row = 32 * warp + lane;      // accumulator row (TMEM lane)
    const int ncol = min(32, t.n - c0);
    if (KIND == G_ROUTER) {
        const int e = t.m0 + row;
        const float b = p.router_b ? __ldg(p.router_b + e) : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < ncol) p.logits[(size_t)(t.b0 + c0 + j) * p.E + e] = u2f(r[j]) + b;
    } else if (KIND == G_DPROJ) {
        // metadata staged by the epilogue warps: group masks and slots of the tile's tokens
        const uint32_t* mmask = reinterpret_cast<const uint32_t*>(xchg);
        const int* mslot = reinterpret_cast<const int*>(mmask + NT);
        bool bad = false;
        // lane = row: the chunk's fp16 values into the transpose buffer; then
        // lane (column j, rows 8q .. 8q+7) writes them to every slot of the
        // token whose expert is in this group
#pragma unroll
        for (int j = 0; j < 32; ++j)
            trw[j * kTrPitch + lane] = j < ncol ? __half_as_ushort(half_checked(u2f(r[j]), bad)) : (uint16_t)0;
        __syncwarp();
        const int lbase = t.m0 + 32 * warp;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = lane + 32 * i, j = idx >> 2, q = idx & 3;
            if (j < ncol) {
                const uint4 v = *reinterpret_cast<const uint4*>(trw + j * kTrPitch + 8 * q);
                uint32_t mask = mmask[c0 + j];
                while (mask) {
                    const int k = __ffs(mask) - 1;
                    mask &= mask - 1;
                    *reinterpret_cast<uint4*>(p.hperm + (size_t)mslot[(c0 + j) * p.K + k] * p.L + lbase + 8 * q) = v;
                }
            }
        }
        __syncwarp();
        report_range(p.ctrl, bad);
    } else if (KIND == G_GATEUP || KIND == G_SHARED_GATEUP) {
        // rows 0-63: gate, rows 64-127: up.  Warps 0-1 finish columns 0-15
        // of the chunk, warps 2-3 columns 16-31; each hands the other pair
        // the half it does not finish.
        float* xg = xchg;              // gate, columns 16-31: [16][64]
        float* xu = xchg + 16 * 64;    // up, columns 0-15:    [16][64]
        const int r64 = row & 63;
        if (warp < 2) {
#pragma unroll
            for (int j = 0; j < 16; ++j) xg[j * 64 + r64] = u2f(r[16 + j]);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) xu[j * 64 + r64] = u2f(r[j]);
        }
        named_bar_sync(1, 128);
        const float tg = tscale[0], tu = tscale[1];
        const int f = t.m0 + r64;
        const int jb = warp < 2 ? 0 : 16;
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (jb + j < ncol) {
                const float a = (warp < 2 ? u2f(r[j]) : xg[j * 64 + r64]) * tg;
                const float u = (warp < 2 ? xu[j * 64 + r64] : u2f(r[16 + j])) * tu;
                const float z = silu_fast(a) * u;
                const int col = t.b0 + c0 + jb + j;
                if (KIND == G_GATEUP) {
                    p.zperm[(size_t)col * p.F + f] = half_checked(z, bad);
                } else {
                    const uint16_t hi = f32_to_bf16_bits(z);
                    p.zsh[(size_t)col * p.Fs + f] = hi;
                    p.zsh[((size_t)p.T + col) * p.Fs + f] = f32_to_bf16_bits(z - bf16_bits_to_f32(hi));
                }
            }
        }
        report_range(p.ctrl, bad);
        named_bar_sync(1, 128);
    } else if (KIND == G_DOWN) {
        // routing weights of the tile's slots staged in xchg by the epilogue warps
        const float td = tscale[2];
        bool bad = false;
        // lane = row into the transpose buffer, then 8 rows of one slot per 16-byte store
#pragma unroll
        for (int j = 0; j < 32; ++j)
            trw[j * kTrPitch + lane] =
                j < ncol ? __half_as_ushort(half_checked(u2f(r[j]) * td * xchg[c0 + j], bad)) : (uint16_t)0;
        __syncwarp();
        const int lbase = t.m0 + 32 * warp;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int idx = lane + 32 * i, j = idx >> 2, q = idx & 3;
            if (j < ncol)
                *reinterpret_cast<uint4*>(p.operm + (size_t)(t.b0 + c0 + j) * p.L + lbase + 8 * q) =
                    *reinterpret_cast<const uint4*>(trw + j * kTrPitch + 8 * q);
        }
        __syncwarp();
        report_range(p.ctrl, bad);
    } else if (t.piece >= 0) {
        // UPROJ, a piece of a split tile: its fp32 partial sum, [piece][token][row]
        float* dst = p.upart + ((size_t)t.piece * kNtDense + c0) * 128 + row;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < ncol) dst[(size_t)j * 128] = u2f(r[j]);
    } else {  // UPROJ
        const int hrow = t.m0 + row;
        float res[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            res[j] = (p.residual && j < ncol) ? bf16_bits_to_f32(__ldg(p.residual + (size_t)(t.b0 + c0 + j) * p.H + hrow)) : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (j < ncol) p.y[(size_t)(t.b0 + c0 + j) * p.H + hrow] = f32_to_bf16_bits(u2f(r[j]) + res[j]);
    }
}

// ---------------------------------------------------------------------------
// the GEMM kernel
// ---------------------------------------------------------------------------

template <int NT, int STAGES, int RS, int MA = 1, bool TR = true>
struct SmemPlan {
    static constexpr int kA = MA * 128 * 128;            // bytes per A stage (MA x 128 rows x 64 x 16-bit)
    static constexpr int kB = NT * 128;                  // bytes per B stage
    // a stage of the converters' ring of stored expert bytes: 32 bytes for
    // each of the 256 converter threads (16 code bytes, the 4-byte scale word)
    // a stage of the two-tile expert GEMMs' ring: 48 bytes for each of the
    // 256 converter threads (a whole row's 32 code bytes and its scale word)
    static constexpr int kRaw = 256 * 48;
    // gate/up exchange (32 x 64 fp32) or a tile's routing metadata (NT x (1 + 16) words)
    static constexpr int kXchg = (32 * 64 * 4 > NT * 4 * 17) ? 32 * 64 * 4 : NT * 4 * 17;
    static constexpr int kTr = TR ? 4 * 32 * kTrPitch * 2 : 0;   // the epilogue warps' transpose buffers (D, down)
    static constexpr int kBars = (2 * STAGES + 5) * 8;
    static constexpr int kTotal = 1024 /*alignment slack*/ + STAGES * (kA + kB) + RS * kRaw + kXchg + kTr + kBars + 16;
};

constexpr int kConvWarps = 8;      // dequantising warps (half a weight row per thread)
constexpr int kRawAhead = 4;       // stages whose stored weight bytes a converter thread holds
constexpr int kGemmThreads = 448;  // 4 epilogue, 8 converter, 1 MMA, 1 loader warps

template <int KIND, int NT, int STAGES, int RS, int MA = 1>
__global__ void __launch_bounds__(kGemmThreads, 1) k_umma_gemm(const __grid_constant__ TmaMaps maps, const PrefillParams p) {
    using S = Sched<KIND, NT, MA>;
    using Plan = SmemPlan<NT, STAGES, RS, MA, KIND == G_DPROJ || KIND == G_DOWN>;
    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic on the shared array, so that the compiler
    // still knows every access through it is a shared-memory access
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * Plan::kA;
    uint8_t* sRaw = sB + STAGES * Plan::kB;
    float* xchg = reinterpret_cast<float*>(sRaw + RS * Plan::kRaw);
    uint16_t* trbuf = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(xchg) + Plan::kXchg);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(trbuf) + Plan::kTr);
    // full[s]: the converter warps' arrivals and the loader's expect-tx
    // arrival with its copies' bytes (one barrier, so the MMA issuer waits
    // once per stage)
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* final_bar = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t kTmemCols = 2 * NT * MA;
    __shared__ float tscale[4];   // the current tile's tensor scales (epilogue)

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], kConvWarps + 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 12) {
        __syncwarp();
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncwarp();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 13) {
        // ------------------------------------------------------------ loader (one thread)
        if (lane == 0) {
            tma_prefetch_desc(&maps.b);
            Cursor<KIND, NT, MA> cb;           // activation / plain-weight stages
            cb.begin(p);
            uint32_t it_b = 0;
            uint32_t last_b[STAGES];
            for (int i = 0; i < STAGES; ++i) last_b[i] = 0xFFFFFFFFu;
            while (!cb.done) {
                const int s = it_b % STAGES;
                const uint32_t ph = (it_b / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimit)) break;
                const bool ta = S::tma_a(p, cb.seg);
                const int k0 = cb.ks * 64;
                mbar_arrive_expect_tx(&full[s], Plan::kB + (ta ? Plan::kA : 0));
                uint8_t* dB = sB + s * Plan::kB;
                if (KIND == G_UPROJ && cb.seg < p.G) tma_load_3d(dB, &maps.b, &full[s], k0, cb.seg, cb.t.b0);
                else if (KIND == G_UPROJ) tma_load_3d(dB, &maps.b2, &full[s], k0, cb.t.b0, cb.seg - p.G);
                else if (cb.seg > 0) tma_load_2d(dB, &maps.b2, &full[s], k0, cb.t.b0);
                else tma_load_2d(dB, &maps.b, &full[s], k0, cb.t.b0);
                if (ta) {
                    if (KIND == G_SHARED_GATEUP) {
                        tma_load_2d(sA + s * Plan::kA, &maps.a, &full[s], k0, cb.t.m0);
                        tma_load_2d(sA + s * Plan::kA + 64 * 128, &maps.a2, &full[s], k0, cb.t.m0);
                    } else {
                        tma_load_2d(sA + s * Plan::kA, &maps.a, &full[s], k0, cb.t.m0);
                    }
                }
                last_b[s] = ph;
                cb.next_stage(p);
                ++it_b;
            }
            if (*abort_flag) {
                // let every copy already issued land before the CTA can leave;
                // the phase also needs the converters' arrivals, which may
                // never come after an abort, so this wait is short (about
                // 0.1 s: the copies themselves take microseconds)
                volatile int dummy = 0;
                for (int i = 0; i < STAGES; ++i)
                    if (last_b[i] != 0xFFFFFFFFu) mbar_wait(&full[i], last_b[i], &dummy, kWaitLimit / 16);
            }
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 12) {
        // ------------------------------------------------------------ converters
        // Each thread owns half a weight row of every stage (a whole row of
        // one of the two A tiles in the two-tile expert GEMMs).  The stored
        // NVFP4 expert bytes come through a ring of RS stages in shared
        // memory filled by the thread's own cp.async copies (deep enough to
        // keep the loads in flight); the other formats are fetched with
        // plain loads kRawAhead - 1 stages ahead of use (a shared-memory
        // ring for Q8_0 D and U, which leaves room for only three operand
        // stages, measured slower).
        const int r = (threadIdx.x - 128) & 127;   // A row
        const int hh = (threadIdx.x - 128) >> 7;   // half of the 64 columns
        Cursor<KIND, NT, MA> cur, cf;
        cur.begin(p);
        cf = cur;
        if (MA == 2) {
            // two-tile items: thread c converts the whole 64-column row
            // c & 127 of A tile c >> 7, through its own ring of RS slots
            constexpr int kRS = RS > 0 ? RS : 1;
            const int c2 = threadIdx.x - 128, a2 = c2 >> 7, rr = c2 & 127;
            uint8_t* ring = sRaw + (size_t)c2 * 48;                          // + stage * Plan::kRaw
#pragma unroll 1
            for (int k = 0; k < kRS - 1; ++k) {
                if (!cf.done) {
                    if (a2 < cf.t.na) fetch_row_async<KIND>(p, cf.t, cf.ks, a2, rr, ring + (size_t)k * Plan::kRaw);
                    cf.next_stage(p);
                }
                cp_async_commit_grp();
            }
            uint32_t it = 0;
            while (!cur.done) {
                if (!cf.done) {
                    if (a2 < cf.t.na)
                        fetch_row_async<KIND>(p, cf.t, cf.ks, a2, rr, ring + (size_t)((it + kRS - 1) % kRS) * Plan::kRaw);
                    cf.next_stage(p);
                }
                cp_async_commit_grp();
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimit)) break;
                cp_async_wait_grp<kRS - 1>();
                if (a2 < cur.t.na) {
                    const uint8_t* slot = ring + (size_t)(it % kRS) * Plan::kRaw;
                    uint8_t* tile = sA + s * Plan::kA + a2 * (128 * 128);
                    RawHalf raw;
                    raw.s = *reinterpret_cast<const uint32_t*>(slot + 32);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        raw.a = *reinterpret_cast<const uint4*>(slot + 16 * h);
                        uint32_t o[16];
                        dequant_half<KIND>(p, raw, h, o);
                        store_half_swizzled(tile, rr, h, o);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[s]);
                cur.next_stage(p);
                ++it;
            }
            cp_async_wait_grp<0>();
        } else {
        RawHalf raw[kRawAhead];
#pragma unroll
        for (int k = 0; k < kRawAhead - 1; ++k) {
            if (!cf.done) {
                if (!S::tma_a(p, cf.seg)) fetch_raw<KIND, NT>(p, cf, r, hh, raw[k]);
                cf.next_stage(p);
            }
        }
        uint32_t it = 0;
        while (!cur.done) {
            if (!cf.done) {
                if (!S::tma_a(p, cf.seg)) fetch_raw<KIND, NT>(p, cf, r, hh, raw[kRawAhead - 1]);
                cf.next_stage(p);
            }
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            const bool ta = S::tma_a(p, cur.seg);
            if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimit)) break;
            if (!ta) {
                uint32_t o[16];
                dequant_half<KIND>(p, raw[0], hh, o);
                store_half_swizzled(sA + s * Plan::kA, r, hh, o);
                fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
#pragma unroll
            for (int k = 0; k + 1 < kRawAhead; ++k) raw[k] = raw[k + 1];
            cur.next_stage(p);
            ++it;
        }
        }
    } else if (warp == 12) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            Cursor<KIND, NT, MA> cur;
            cur.begin(p);
            uint32_t it = 0, tcount = 0;
            bool issued = false;
            while (!cur.done) {
                const int acc = tcount & 1;
                const uint32_t aph = (tcount >> 1) & 1;
                if (!mbar_wait(&tempty[acc], aph ^ 1, abort_flag, kWaitLimit)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * NT * MA;
                const int n_mma = (KIND == G_GATEUP || KIND == G_DOWN) ? ((cur.t.n + 15) & ~15) : NT;
                const int na = cur.t.na;
                bool first = true;
                bool ok = true;
                while (true) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    const bool ta = S::tma_a(p, cur.seg);
                    const uint32_t idesc = idesc_f16(128, n_mma, ta ? 1 : 0);
                    if (!mbar_wait(&full[s], ph, abort_flag, kWaitLimit)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t b_desc = sdesc_k128(smem_u32(sB + s * Plan::kB));
#pragma unroll
                    for (int a = 0; a < MA; ++a) {
                        if (a >= na) break;
                        // A tile a of the stage; both tiles share the B stage
                        const uint64_t a_desc = sdesc_k128(smem_u32(sA + s * Plan::kA + a * (128 * 128)));
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            umma_f16(d_tmem + a * NT, a_desc + 2 * j, b_desc + 2 * j, idesc, (first && j == 0) ? 0u : 1u);
                    }
                    first = false;
                    issued = true;
                    umma_commit(&empty[s]);
                    ++it;
                    const bool last = cur.last_stage_of_tile(p);
                    cur.next_stage(p);
                    if (last) break;
                }
                if (!ok) break;
                umma_commit(&tfull[acc]);
                ++tcount;
            }
            if (issued) {
                // all tensor-core work of this CTA done before TMEM is released
                umma_commit(final_bar);
                volatile int dummy = 0;
                mbar_wait(final_bar, 0, &dummy, kWaitLimit);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Every epilogue warp walks every tile and reaches every named
        // barrier; after a timeout (dead) the work is skipped.  The TMEM
        // loads are warp-collective, so the wait's outcome is made
        // warp-uniform and the warp converges before each load.
        Cursor<KIND, NT, MA> cur;
        cur.begin(p);
        uint32_t tcount = 0;
        bool dead = false;
        while (!cur.done) {
            const int acc = tcount & 1;
            const uint32_t ph = (tcount >> 1) & 1;
            // the tile's routing metadata goes to shared memory while the
            // accumulator is still being computed
            if (KIND == G_DPROJ) {
                uint32_t* mmask = reinterpret_cast<uint32_t*>(xchg);
                int* mslot = reinterpret_cast<int*>(mmask + NT);
                // batches of independent loads, then the shared-memory stores
                const int nn = cur.t.n * p.K;
                const int* src = p.pair_slot + (size_t)cur.t.b0 * p.K;
                for (int i0 = threadIdx.x; i0 < nn; i0 += 128 * 8) {
                    int v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) v[u] = i0 + 128 * u < nn ? __ldg(src + i0 + 128 * u) : 0;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        if (i0 + 128 * u < nn) mslot[i0 + 128 * u] = v[u];
                }
                for (int i0 = threadIdx.x; i0 < cur.t.n; i0 += 128 * 2) {
                    uint32_t v[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        v[u] = i0 + 128 * u < cur.t.n ? __ldg(p.tgmask + (size_t)(cur.t.b0 + i0 + 128 * u) * p.G + cur.t.mat) : 0u;
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        if (i0 + 128 * u < cur.t.n) mmask[i0 + 128 * u] = v[u];
                }
            } else if (KIND == G_DOWN) {
                for (int i = threadIdx.x; i < cur.t.n; i += 128) xchg[i] = __ldcg(p.wslot + cur.t.b0 + i);
            }
            if ((KIND == G_GATEUP || KIND == G_DOWN) && threadIdx.x < 3) {
                // the expert's tensor scales (gate, up, down) from its record
                // tail; the Q3_K build has none
                const size_t nq = (size_t)p.L * p.F / 2, ns = (size_t)p.L * p.F / 16;
                tscale[threadIdx.x] = p.efmt == LMOE_EXPERTS_Q3K ? 1.f :
                    __ldg(reinterpret_cast<const float*>(p.experts + (size_t)cur.t.mat * p.rec_bytes + 3 * nq + 3 * ns) + threadIdx.x);
            } else if (KIND == G_SHARED_GATEUP && threadIdx.x < 3) {
                tscale[threadIdx.x] = 1.f;
            }
            named_bar_sync(1, 128);
            if (!dead) dead = !mbar_wait(&tfull[acc], ph, abort_flag, kWaitLimit);
            dead = __any_sync(0xffffffffu, dead);
            if (!dead) {
                tc_fence_after();
                for (int a = 0; a < cur.t.na; ++a) {
                    // accumulator a of the item: A tile a's output rows
                    TileRef ta = cur.t;
                    ta.m0 += a * (KIND == G_GATEUP ? 64 : 128);
                    const uint32_t taddr = tmem_base + ((uint32_t)(32 * warp) << 16) + acc * NT * MA + a * NT;
                    for (int c0 = 0; c0 < cur.t.n; c0 += 32) {
                        uint32_t rr[32];
                        __syncwarp();
                        tmem_ld_32x32b_x32(taddr + c0, rr);
                        tmem_ld_wait();
                        epilogue_chunk<KIND, NT>(p, ta, warp, lane, c0, rr, xchg, tscale, trbuf + warp * 32 * kTrPitch);
                    }
                }
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(&tempty[acc]);
            named_bar_sync(1, 128);
            ++tcount;
            cur.next_tile(p);
        }
    }

    tc_fence_before();
    __syncwarp();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) set_status(p.ctrl, LMOE_ERR_TIMEOUT);
    if (warp == 12) {
        tc_fence_after();
        __syncwarp();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// routing and bucketing for many tokens
// ---------------------------------------------------------------------------

// fp16 copy of the block input (RMS-normalised first when gamma is given);
// values outside the fp16 range are reported as an invalid input.
__global__ void k_x_to_fp16(const PrefillParams p) {
    const int t = blockIdx.x;
    const uint16_t* row = p.x + (size_t)t * p.H;
    float scale = 1.f;
    if (p.gamma) {
        __shared__ float red[32];
        float ss = 0.f;
        for (int k = threadIdx.x; k < p.H; k += blockDim.x) {
            const float v = bf16_bits_to_f32(row[k]);
            ss += v * v;
        }
        ss = warp_sum(ss);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        if (threadIdx.x < 32) {
            float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
            v = warp_sum(v);
            if (threadIdx.x == 0) red[0] = rsqrtf(v / (float)p.H + p.eps);
        }
        __syncthreads();
        scale = red[0];
    }
    bool bad = false;
    for (int k = threadIdx.x; k < p.H; k += blockDim.x) {
        float v = bf16_bits_to_f32(row[k]);
        if (p.gamma) v *= scale * bf16_bits_to_f32(p.gamma[k]);
        bad |= !(fabsf(v) <= 65504.f);
        p.xh[(size_t)t * p.H + k] = __float2half_rn(v);
        if (p.xr) {
            const uint16_t hi = f32_to_bf16_bits(v);
            p.xr[(size_t)t * p.H + k] = hi;
            p.xr_lo[(size_t)t * p.H + k] = f32_to_bf16_bits(v - bf16_bits_to_f32(hi));
        }
    }
    if (bad) set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK);
}

// softmax top-k per token from the logits (warp per token)
__global__ void k_topk(const PrefillParams p) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= p.T) return;
    const int t = warp, E = p.E, K = p.K;
    if (p.inject_idx) {
        if (lane < K) {
            p.idx[(size_t)t * K + lane] = p.inject_idx[(size_t)t * K + lane];
            p.w[(size_t)t * K + lane] = p.inject_w[(size_t)t * K + lane];
        }
    } else {
        float v[kMaxExpertsTopk / 32];
        uint32_t taken = 0;
#pragma unroll
        for (int j = 0; j < kMaxExpertsTopk / 32; ++j) {
            const int e = lane + 32 * j;
            v[j] = e < E ? __ldcg(p.logits + (size_t)t * E + e) : -INFINITY;
        }
        float lmax = 0.f, denom = 0.f, my_l = 0.f;
        int my_e = 0;
        for (int k = 0; k < K; ++k) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < kMaxExpertsTopk / 32; ++j) {
                const int e = lane + 32 * j;
                if (e < E && !(taken >> j & 1u) && (v[j] > bv || (v[j] == bv && e < bi))) { bv = v[j]; bi = e; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            if ((bi & 31) == lane && bi < E) taken |= 1u << (bi >> 5);
            if (k == 0) lmax = bv;
            if (k == lane) { my_l = bv; my_e = bi; }
            denom += expf(bv - lmax);
        }
        if (lane < K) {
            p.idx[(size_t)t * K + lane] = my_e;
            p.w[(size_t)t * K + lane] = expf(my_l - lmax) / denom;
        }
    }
    if (lane < K) {
        if (p.out_idx) p.out_idx[(size_t)t * K + lane] = p.idx[(size_t)t * K + lane];
        if (p.out_w) p.out_w[(size_t)t * K + lane] = p.w[(size_t)t * K + lane];
    }
}

// counts per expert, group masks per token, hit flags per token tile
__global__ void k_bucket_count(const PrefillParams p) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= p.T * p.K) return;
    const int t = i / p.K, k = i - t * p.K;
    int e = p.idx[i];
    if (e < 0 || e >= p.E) { set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK); e = 0; p.idx[i] = 0; }
    int g = p.group[e];
    if (g >= p.G) { set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK); g = 0; }
    atomicAdd(p.cnt + e, 1);
    atomicOr(p.tgmask + (size_t)t * p.G + g, 1u << k);
    p.dhit[(t / kNtDense) * p.G + g] = 1;
}

// offsets, distinct experts and the expert token tiles (one CTA)
__global__ void k_bucket_scan(const PrefillParams p) {
    __shared__ int scratch[32];
    const int E = p.E;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e_lo = threadIdx.x * per, e_hi = min(E, e_lo + per);
    int c = 0, f = 0, nt = 0;
    for (int e = e_lo; e < e_hi; ++e) {
        const int ce = p.cnt[e];
        c += ce;
        f += ce > 0;
        nt += (ce + kNtExpert - 1) / kNtExpert;
    }
    int off0, u0, t0;
    block_exclusive_scan(c, &off0, scratch);
    const int n_unique = block_exclusive_scan(f, &u0, scratch);
    const int n_tiles = block_exclusive_scan(nt, &t0, scratch);
    for (int e = e_lo, o = off0, u = u0, tt = t0; e < e_hi; ++e) {
        const int ce = p.cnt[e];
        p.off[e] = o;
        if (ce > 0) {
            p.uexp[u] = e;
            p.ucnt[u] = ce;
            p.uoff[u] = o;
            for (int n0 = 0; n0 < ce; n0 += kNtExpert) p.etile[tt++] = make_int4(e, o + n0, min(kNtExpert, ce - n0), u);
            ++u;
        }
        o += ce;
    }
    if (threadIdx.x == 0) {
        *p.n_unique = n_unique;
        *p.n_etiles = n_tiles;
    }
}

__global__ void k_bucket_scatter(const PrefillParams p) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= p.T * p.K) return;
    const int e = p.idx[i];
    const int slot = p.off[e] + atomicAdd(p.fill + e, 1);
    p.slot_pair[slot] = i;
    p.pair_slot[i] = slot;
    p.wslot[slot] = p.w[i];
}

// U's split tiles: y = bf16(sum of the pieces' partial sums, in piece order,
// + residual).  A piece none of whose segments is active (no token of the
// tile hits its groups) was skipped by the GEMM and adds nothing.  One CTA
// per (split tile, token), a thread per row.
__global__ void k_u_reduce(const PrefillParams p) {
    const int tt = blockIdx.x, c = blockIdx.y, r = threadIdx.x;
    const int mt = p.H / 128;
    const int ti = p.u_whole + tt;                    // token-tile-major, as the GEMM's items
    const int m = ti % mt, q = ti / mt;
    const int tok = q * kNtDense + c;
    if (tok >= p.T) return;
    float acc = 0.f;
    for (int part = 0; part < p.u_parts; ++part) {
        bool active = false;
        for (int seg = p.u_segb[part]; seg < p.u_segb[part + 1]; ++seg)
            active |= seg >= p.G || p.dhit[q * p.G + seg] != 0;
        if (active) acc += __ldcg(p.upart + ((size_t)(tt * p.u_parts + part) * kNtDense + c) * 128 + r);
    }
    const int h = m * 128 + r;
    if (p.residual) acc += bf16_bits_to_f32(__ldg(p.residual + (size_t)tok * p.H + h));
    p.y[(size_t)tok * p.H + h] = f32_to_bf16_bits(acc);
}

// s[t][g] = sum over the token's experts of group g of o (already weighted);
// zero for groups the token does not hit.  One CTA per token, 16 bytes per thread.
__global__ void k_combine(const PrefillParams p) {
    const int t = blockIdx.x;
    const int nchunk = p.L / 8;
    bool bad = false;
    for (int g = 0; g < p.G; ++g) {
        const uint32_t mask = __ldg(p.tgmask + (size_t)t * p.G + g);
        for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            uint32_t m = mask;
            while (m) {
                const int k = __ffs(m) - 1;
                m &= m - 1;
                const int slot = __ldg(p.pair_slot + (size_t)t * p.K + k);
                const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.operm + (size_t)slot * p.L) + c);
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __half22float2(bits_h2(w4[j]));
                    acc[2 * j] += f.x;
                    acc[2 * j + 1] += f.y;
                }
            }
            uint4 out;
            out.x = h2_bits(half2_checked(acc[0], acc[1], bad));
            out.y = h2_bits(half2_checked(acc[2], acc[3], bad));
            out.z = h2_bits(half2_checked(acc[4], acc[5], bad));
            out.w = h2_bits(half2_checked(acc[6], acc[7], bad));
            reinterpret_cast<uint4*>(p.s + ((size_t)t * p.G + g) * p.L)[c] = out;
        }
    }
    report_range(p.ctrl, bad);
}

// ---------------------------------------------------------------------------
// host side: tensor maps and the launch sequence
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D map over a row-major [rows][cols] 16-bit matrix, box = 64 columns x box_rows.
static bool make_map_2d(CUtensorMap* m, const void* base, bool bf16, uint64_t rows, uint64_t cols, uint64_t row_stride_elems,
                        uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_stride_elems * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over s [T][G][L] fp16, box = 64 x 1 x box_rows.
static bool make_map_s(CUtensorMap* m, const void* base, uint64_t T, uint64_t G, uint64_t L, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {L, G, T};
    cuuint64_t strides[2] = {L * 2, G * L * 2};
    cuuint32_t box[3] = {64, 1, box_rows};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the shared hidden [2][T][Fs] bf16 (high, low), box = 64 x box_rows x 1.
static bool make_map_zsh(CUtensorMap* m, const void* base, uint64_t T, uint64_t Fs, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {Fs, T, 2};
    cuuint64_t strides[2] = {Fs * 2, T * Fs * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int g_num_sms = 0;

template <int KIND, int NT, int STAGES, int RS, int MA = 1>
static cudaError_t launch_gemm(const TmaMaps& maps, const PrefillParams& p, cudaStream_t st, int max_tiles) {
    const size_t smem = SmemPlan<NT, STAGES, RS, MA, KIND == G_DPROJ || KIND == G_DOWN>::kTotal;
    auto kern = k_umma_gemm<KIND, NT, STAGES, RS, MA>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int grid = max(1, min(g_num_sms, max_tiles));
    kern<<<grid, kGemmThreads, smem, st>>>(maps, p);
    return cudaGetLastError();
}

// U's split plan: the tiles of the last wave (n_u mod sms of them, if the
// wave is partial) become u_parts pieces each, contiguous segment ranges of
// about equal stage counts (a group segment is L / 64 stages, each shared
// segment Fs / 64); at most kMaxUParts pieces a tile and kMaxUPieces in all.
static void u_split_plan(PrefillParams& p, int n_u, int sms) {
    p.u_whole = n_u;
    p.u_parts = 1;
    const int nseg = p.G + 2;
    const int tail = n_u % sms;
    if (tail == 0 || p.upart == nullptr) return;
    const int parts = std::min(std::min(nseg, kMaxUParts), std::min(sms / tail, kMaxUPieces / tail));
    if (parts < 2) return;
    long total = 0;
    for (int sg = 0; sg < nseg; ++sg) total += sg < p.G ? p.L / 64 : p.Fs / 64;
    p.u_segb[0] = 0;
    long acc = 0;
    int b = 1;
    for (int sg = 0; sg < nseg && b < parts; ++sg) {
        acc += sg < p.G ? p.L / 64 : p.Fs / 64;
        // close piece b - 1 once it holds its share, leaving a segment for each later piece
        if (acc * parts >= total * b && nseg - (sg + 1) >= parts - b) p.u_segb[b++] = sg + 1;
    }
    if (b < parts) return;                            // fewer natural cuts than pieces: keep whole tiles
    p.u_segb[parts] = nseg;
    p.u_whole = n_u - tail;
    p.u_parts = parts;
}

cudaError_t run_prefill_path(PrefillParams p, cudaStream_t st, void* memset_base, size_t memset_bytes,
                             void (*mark)(cudaStream_t)) {
    const int T = p.T, H = p.H, L = p.L, G = p.G, F = p.F, Fs = p.Fs, K = p.K, E = p.E;
    cudaError_t e;
    const int ttiles = (T + kNtDense - 1) / kNtDense;
    TmaMaps m_router, m_shared, m_d, m_gu, m_down, m_u;
    std::memset(&m_router, 0, sizeof(TmaMaps));
    m_shared = m_d = m_gu = m_down = m_u = m_router;
    (void)mark;
    bool ok = true;
    ok &= make_map_2d(&m_router.a, p.router_w_bf16, true, E, H, H, 128);
    ok &= make_map_2d(&m_router.b, p.xr ? (const void*)p.xr : (const void*)p.x, true, T, H, H, kNtDense);
    ok &= make_map_2d(&m_shared.a, p.sg, true, Fs, H, H, 64);
    ok &= make_map_2d(&m_shared.a2, p.su, true, Fs, H, H, 64);
    ok &= make_map_2d(&m_shared.b, p.xr ? (const void*)p.xr : (const void*)p.x, true, T, H, H, kNtDense);
    if (p.xr) {
        ok &= make_map_2d(&m_router.b2, p.xr_lo, true, T, H, H, kNtDense);
        ok &= make_map_2d(&m_shared.b2, p.xr_lo, true, T, H, H, kNtDense);
    }
    ok &= make_map_2d(&m_d.b, p.xh, false, T, H, H, kNtDense);
    ok &= make_map_2d(&m_gu.b, p.hperm, false, (uint64_t)T * K, L, L, kNtExpert);
    ok &= make_map_2d(&m_down.b, p.zperm, false, (uint64_t)T * K, F, F, kNtExpert);
    ok &= make_map_s(&m_u.b, p.s, T, G, L, kNtDense);
    ok &= make_map_2d(&m_u.a, p.sd, true, H, Fs, Fs, 128);           // shared down weights (bf16)
    ok &= make_map_zsh(&m_u.b2, p.zsh, T, Fs, kNtDense);               // shared hidden, bf16 high / low
    if (!ok) return cudaErrorInvalidValue;

    if (memset_bytes) {
        e = cudaMemsetAsync(memset_base, 0, memset_bytes, st);
        if (e != cudaSuccess) return e;
    }
    mark(st);
    k_x_to_fp16<<<T, 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(st);
    if ((e = launch_gemm<G_ROUTER, kNtDense, 4, 0>(m_router, p, st, (E / 128) * ttiles)) != cudaSuccess) return e;
    mark(st);
    k_topk<<<(T * 32 + 255) / 256, 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int pairs = T * K;
    k_bucket_count<<<(pairs + 255) / 256, 256, 0, st>>>(p);
    k_bucket_scan<<<1, 1024, 0, st>>>(p);
    k_bucket_scatter<<<(pairs + 255) / 256, 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(st);
    if ((e = launch_gemm<G_SHARED_GATEUP, kNtDense, 4, 0>(m_shared, p, st, (Fs / 64) * ttiles)) != cudaSuccess) return e;
    mark(st);
    if ((e = launch_gemm<G_DPROJ, kNtDense, 4, 0>(m_d, p, st, G * (L / 128) * ttiles)) != cudaSuccess) return e;
    mark(st);
    const int max_etiles = min(E, pairs) + pairs / kNtExpert + 1;
    if (p.act == LMOE_ACT_NVFP4) {
        // W4A4: h, then z, as NVFP4 activations, times the NVFP4 weights
        if ((e = run_act_quant(p.hperm, pairs, L, p.aq, p.asf, p.aG, st)) != cudaSuccess) return e;
        if ((e = run_w4a4_gateup(p, p.aq, p.asf, p.aG, pairs, st)) != cudaSuccess) return e;
        mark(st);
        if ((e = run_act_quant(p.zperm, pairs, F, p.aq, p.asf, p.aG, st)) != cudaSuccess) return e;
        if ((e = run_w4a4_down(p, p.aq, p.asf, p.aG, pairs, st)) != cudaSuccess) return e;
        mark(st);
    } else {
        if (p.efmt == LMOE_EXPERTS_NVFP4) {
            // two 128-row A tiles per item (one B stage feeds both)
            if ((e = launch_gemm<G_GATEUP, kNtExpert, 3, 4, 2>(m_gu, p, st, (F / 128 + 1) * max_etiles)) != cudaSuccess)
                return e;
            mark(st);
            if ((e = launch_gemm<G_DOWN, kNtExpert, 3, 4, 2>(m_down, p, st, (L / 256 + 1) * max_etiles)) != cudaSuccess)
                return e;
        } else {
            if ((e = launch_gemm<G_GATEUP, kNtExpert, 4, 0>(m_gu, p, st, (F / 64) * max_etiles)) != cudaSuccess) return e;
            mark(st);
            if ((e = launch_gemm<G_DOWN, kNtExpert, 4, 0>(m_down, p, st, (L / 128) * max_etiles)) != cudaSuccess) return e;
        }
        mark(st);
    }
    k_combine<<<T, 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    mark(st);
    {
        // the last, partial wave of U tiles runs split into pieces by K
        // segment, so that every SM gets a share of it
        if (g_num_sms == 0) {
            int dev = 0;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        }
        const int n_u = (H / 128) * ttiles;
        u_split_plan(p, n_u, g_num_sms);
        const int items = p.u_whole + (n_u - p.u_whole) * p.u_parts;
        if ((e = launch_gemm<G_UPROJ, kNtDense, 4, 0>(m_u, p, st, items)) != cudaSuccess) return e;
        if (p.u_parts > 1) {
            k_u_reduce<<<dim3(n_u - p.u_whole, kNtDense), 128, 0, st>>>(p);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
    }
    mark(st);
    return cudaSuccess;
}

// Router only (logits GEMM + top-k) for many tokens.
cudaError_t run_prefill_route(PrefillParams p, cudaStream_t st) {
    TmaMaps m;
    std::memset(&m, 0, sizeof(m));
    bool ok = make_map_2d(&m.a, p.router_w_bf16, true, p.E, p.H, p.H, 128);
    ok &= make_map_2d(&m.b, p.x, true, p.T, p.H, p.H, kNtDense);
    if (!ok) return cudaErrorInvalidValue;
    const int ttiles = (p.T + kNtDense - 1) / kNtDense;
    cudaError_t e = launch_gemm<G_ROUTER, kNtDense, 4, 0>(m, p, st, (p.E / 128) * ttiles);
    if (e != cudaSuccess) return e;
    k_topk<<<(p.T * 32 + 255) / 256, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace lmoe
