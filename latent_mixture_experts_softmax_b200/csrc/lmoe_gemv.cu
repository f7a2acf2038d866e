// Latent-MoE block for few tokens (decode / MTP verify windows): five
// weight-streaming kernels on CUDA cores.  Every weight byte of the block is
// read once per pass of up to kChunk tokens; activations are staged in shared
// memory as fp32 and every accumulation is fp32.
//
//   k_router_shared   router logits (+ bias) for all experts, the shared
//                     expert's gate/up + SwiGLU; the last router CTA runs the
//                     softmax / top-k / renormalisation and the bucketing
//   k_dproj           h[t][g] = D_g x_t for every group g hit by some token
//   k_expert_gateup   z = silu(W_gate h) * (W_up h) per routed (token, expert)
//   k_expert_down     o = W_down z
//   k_uproj           per output row tile: U_g (sum of w_k o_k over the
//                     experts of group g) for every hit g, the shared down
//                     projection, then (last CTA of the tile) the sum of the
//                     parts + residual -> bf16 y
//
// Method: teardown article "Edge0-145B: a Qwen MoE with its experts squeezed",
// section "A latent in front of the experts" (layer equation, per-group D/U);
// Edge0 145B / 120B model page, architecture tables (SwiGLU width 640, one
// shared expert at full width, top-10 of 512).

#include <algorithm>

#include "lmoe_internal.cuh"
#include "lmoe_q3k.cuh"
#include "lmoe_route.cuh"
#include "lmoe_rowdot.cuh"

namespace lmoe {

// ---------------------------------------------------------------------------
// kernel 1: router logits + shared gate/up; last router CTA: top-k + buckets
// ---------------------------------------------------------------------------

__device__ void topk_and_buckets(const FwdParams& p);

template <int NT, bool kRouterBF16>
__global__ void __launch_bounds__(256) k_router_shared(FwdParams p) {
    extern __shared__ float smem[];
    float* xs = smem;                 // [H][NT]
    __shared__ float rs[kChunk];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = p.H;
    const bool router_cta = (int)blockIdx.x < p.n_router_ctas;
    // the D_g kernel may launch now; it waits for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!router_cta && !p.do_shared) return;
    // expert -> group table, for the CTA that ends up routing (loaded while
    // the logits are computed)
    __shared__ uint8_t sgrp[kMaxExpertsTopk];
    if (router_cta && p.route_smem)
        for (int e = threadIdx.x; e < p.E; e += blockDim.x) sgrp[e] = p.group[e];
    if (p.prefetch_l2 && blockIdx.x == 0 && p.T <= kChunk)
        l2_prefetch_range(p.sd, (size_t)p.H * p.Fs * 2);
    for (int t0 = 0; t0 < p.T; t0 += NT) {
        const int nt = min(NT, p.T - t0);
        stage_x<NT>(p, t0, nt, xs, rs);
        __syncthreads();
        if (router_cta) {
            const int e = blockIdx.x * 8 + warp;
            if (e < p.E) {
                float acc[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t) acc[t] = 0.f;
                if (kRouterBF16) row_dot<NT, true>(static_cast<const uint16_t*>(p.router_w) + (size_t)e * H, H, xs, xs_ld(H), lane, acc);
                else row_dot<NT, false>(static_cast<const float*>(p.router_w) + (size_t)e * H, H, xs, xs_ld(H), lane, acc);
                const float b = p.router_b ? __ldg(p.router_b + e) : 0.f;
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float v = warp_sum(acc[t]);
                    if (lane == 0 && t < nt) p.r.logits[(size_t)(t0 + t) * p.E + e] = v + b;
                }
            }
        } else {
            // shared expert: warp -> feature f (one gate row and one up row)
            const int f = ((int)blockIdx.x - p.n_router_ctas) * 8 + warp;
            if (f < p.Fs) {
                float a[NT], u[NT];
#pragma unroll
                for (int t = 0; t < NT; ++t) { a[t] = 0.f; u[t] = 0.f; }
                row_dot2_bf16<NT>(p.sg + (size_t)f * H, p.su + (size_t)f * H, H, xs, xs_ld(H), lane, a, u);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float av = warp_sum(a[t]), uv = warp_sum(u[t]);
                    if (lane == 0 && t < nt) {
                        const float z = silu(av) * uv;
                        p.zsh[(size_t)(t0 + t) * p.Fs + f] = z;
                        if (p.zsh16) {
                            bool bad = false;
                            p.zsh16[(size_t)(t0 + t) * p.Fs + f] = half_checked(z, bad);
                            report_range(p.ctrl, bad);
                        }
                    }
                }
            }
        }
        __syncthreads();
    }
    if (!router_cta) return;

    // the last router CTA to finish selects the experts
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int done = atomicAdd(&p.ctrl->route_ticket, 1);
        s_last = (done == p.n_router_ctas - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (p.route_smem) {
        __shared__ StreamShared rsh;
        route_in_cta(p, rsh, sgrp, true);
    } else {
        topk_and_buckets(p);
    }
    if (threadIdx.x == 0) p.ctrl->route_ticket = 0;
}

// Warp-wide arg-max with ties to the lower index.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}

// Softmax top-K of token t by one warp: NV logits per lane in registers; K
// rounds of a warp arg-max (ties to the lower index); w_k = exp(l_k - l_1) /
// sum over the kept of exp(l_j - l_1).
template <int NV>
__device__ __forceinline__ void topk_warp(const FwdParams& p, int t, int lane) {
    const int E = p.E, K = p.K;
    float v[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        v[j] = e < E ? __ldcg(p.r.logits + (size_t)t * E + e) : -INFINITY;
    }
    // each lane keeps its own best untaken (value, index); only the lane that
    // supplied a round's winner rescans its values
    uint32_t taken = 0;
    float lv = -INFINITY;
    int li = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        if (e < E && v[j] > lv) { lv = v[j]; li = e; }
    }
    float lmax = 0.f, denom = 0.f, my_l = 0.f;
    int my_e = 0;
    for (int k = 0; k < K; ++k) {
        float bv = lv;
        int bi = li;
        warp_argmax(bv, bi);
        if (bi < E && (bi & 31) == lane) {
            taken |= 1u << (bi >> 5);
            lv = -INFINITY;
            li = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                const int e = lane + 32 * j;
                if (e < E && !(taken >> j & 1u) && (v[j] > lv || (v[j] == lv && e < li))) { lv = v[j]; li = e; }
            }
        }
        if (k == 0) lmax = bv;
        if (k == lane) { my_l = bv; my_e = bi; }
        denom += expf(bv - lmax);
    }
    if (lane < K) {
        p.r.idx[(size_t)t * K + lane] = my_e;
        p.r.w[(size_t)t * K + lane] = expf(my_l - lmax) / denom;
    }
}

// Bucketing of at most 64 (token, k) pairs by one warp: slots ordered by
// (expert, pair index), distinct experts ascending; O(n^2) comparisons.
__device__ void buckets_small_warp(const FwdParams& p, int lane) {
    const int K = p.K, G = p.G, T = p.T, E = p.E, n = T * K;
    const Routing& r = p.r;
    __shared__ int se[64];
    __shared__ uint8_t sf[64];
    int e_i[2], g_i[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = lane + 32 * h;
        e_i[h] = 0x7fffffff;
        g_i[h] = 0;
        if (i < n) {
            int e = r.idx[i];
            if (e < 0 || e >= E) { set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK); e = 0; r.idx[i] = 0; }
            int g = p.group[e];
            if (g >= G) { set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK); g = 0; }
            e_i[h] = e;
            g_i[h] = g;
        }
        se[i] = e_i[h];
    }
    for (int i = lane; i < T * G; i += 32) r.tghit[i] = 0;
    for (int g = lane; g < G; g += 32) r.ghit[g] = 0;
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = lane + 32 * h;
        int before = 0;
        for (int j = 0; j < i && j < n; ++j) before += se[j] == e_i[h];
        sf[i] = (i < n && before == 0);
    }
    __syncwarp();
    int n_first = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = lane + 32 * h;
        if (i >= n) continue;
        int less = 0, same_before = 0, cnt = 0, u = 0;
        for (int j = 0; j < n; ++j) {
            const int ej = se[j];
            less += ej < e_i[h];
            same_before += (j < i && ej == e_i[h]);
            cnt += ej == e_i[h];
            u += (sf[j] && ej < e_i[h]);
        }
        const int slot = less + same_before;
        r.slot_pair[slot] = i;
        r.pair_slot[i] = slot;
        if (sf[i]) {
            r.uexp[u] = e_i[h];
            r.ucnt[u] = cnt;
            r.uoff[u] = less;
            ++n_first;
        }
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = lane + 32 * h;
        if (i < n) {
            r.tghit[(i / K) * G + g_i[h]] = 1;
            atomicAdd(r.ghit + g_i[h], 1);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_first += __shfl_xor_sync(0xffffffffu, n_first, o);
    if (lane == 0) *r.n_unique = n_first;
}

__device__ void topk_and_buckets(const FwdParams& p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int E = p.E, K = p.K, G = p.G, T = p.T;
    const Routing& r = p.r;

    // --- softmax top-k per token: warp per token, logits in registers
    if (p.inject_idx != nullptr && p.inject_w != nullptr) {
        for (int i = threadIdx.x; i < T * K; i += blockDim.x) {
            r.idx[i] = p.inject_idx[i];
            r.w[i] = p.inject_w[i];
        }
    } else {
        for (int t = warp; t < T; t += nw) {
            if (E <= 64) topk_warp<2>(p, t, lane);
            else if (E <= 128) topk_warp<4>(p, t, lane);
            else if (E <= 256) topk_warp<8>(p, t, lane);
            else if (E <= 512) topk_warp<16>(p, t, lane);
            else topk_warp<32>(p, t, lane);
        }
    }
    __syncthreads();
    if (p.out_idx != nullptr || p.out_w != nullptr) {
        for (int i = threadIdx.x; i < T * K; i += blockDim.x) {
            if (p.out_idx) p.out_idx[i] = r.idx[i];
            if (p.out_w) p.out_w[i] = r.w[i];
        }
    }
    if (!p.do_buckets) return;
    if (T * K <= 64) {
        if (warp == 0) buckets_small_warp(p, lane);
        return;
    }

    // --- bucketing: counts, distinct experts, slots, group hits
    __shared__ int cnt[kMaxExpertsTopk];
    __shared__ int gh[kMaxGroups];
    __shared__ int scan_scratch[32];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    for (int g = threadIdx.x; g < G; g += blockDim.x) gh[g] = 0;
    for (int i = threadIdx.x; i < T * G; i += blockDim.x) r.tghit[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < T * K; i += blockDim.x) {
        int e = r.idx[i];
        if (e < 0 || e >= E) { set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK); e = 0; r.idx[i] = 0; }
        int g = p.group[e];
        if (g >= G) { set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK); g = 0; }
        atomicAdd(&cnt[e], 1);
        atomicAdd(&gh[g], 1);
        r.tghit[(i / K) * G + g] = 1;
    }
    __syncthreads();
    // scan over experts: each thread owns a contiguous range
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e_lo = threadIdx.x * per, e_hi = min(E, e_lo + per);
    int my_cnt = 0, my_flags = 0;
    for (int e = e_lo; e < e_hi; ++e) { my_cnt += cnt[e]; my_flags += cnt[e] > 0; }
    int off0, uoff0;
    block_exclusive_scan(my_cnt, &off0, scan_scratch);
    const int n_unique = block_exclusive_scan(my_flags, &uoff0, scan_scratch);
    __shared__ int offs[kMaxExpertsTopk];
    for (int e = e_lo, o = off0, u = uoff0; e < e_hi; ++e) {
        offs[e] = o;
        if (cnt[e] > 0) {
            r.uexp[u] = e;
            r.ucnt[u] = cnt[e];
            r.uoff[u] = o;
            ++u;
        }
        o += cnt[e];
    }
    if (threadIdx.x == 0) *r.n_unique = n_unique;
    for (int g = threadIdx.x; g < G; g += blockDim.x) r.ghit[g] = gh[g];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < T * K; i += blockDim.x) {
        const int e = r.idx[i];
        const int slot = offs[e] + atomicAdd(&cnt[e], 1);
        r.slot_pair[slot] = i;
        r.pair_slot[i] = slot;
    }
    // Start streaming every weight the rest of the step reads into L2 now, in
    // the order the kernels need them: D_g of the hit groups, the routed
    // experts' records, U_g of the hit groups.  The later kernels then find
    // their weights on chip while HBM stays busy across kernel boundaries.
    if (p.prefetch_l2 && T <= kChunk) {
        __syncthreads();
        for (int g = 0; g < G; ++g)
            if (gh[g]) l2_prefetch_range(p.D + (size_t)g * p.du_bytes_D, p.du_bytes_D);
        for (int u = 0; u < n_unique; ++u)
            l2_prefetch_range(p.experts + (size_t)__ldcg(r.uexp + u) * p.rec_bytes, p.rec_bytes);
        for (int g = 0; g < G; ++g)
            if (gh[g]) l2_prefetch_range(p.U + (size_t)g * p.du_bytes_U, p.du_bytes_U);
    }
}

// ---------------------------------------------------------------------------
// kernels 2-5 on the tensor pipe (mma.sync m16n8k16, fp16 operands, fp32
// accumulation): at decode the arithmetic per weight byte, not the tensor
// throughput, limits a CUDA-core GEMV (4-bit weights allow ~2.8 instructions
// per weight at HBM speed; a CUDA-core dot product with the dequantisation
// needs 4-6), so the dot products go to the tensor pipe and the CUDA cores
// only unpack.  A warp owns 16 weight rows; the 8 token columns of the MMA
// are the (up to 8) tokens of the pass, zero-padded.
//
// Fragment ownership (lane = 4 g + t): A rows g and g + 8; B column (token)
// g; C rows g, g + 8 and columns 2t, 2t + 1.  Within a 32-element block the
// thread feeds the k slots it owns with physical elements it loads itself;
// the activation operand is read with the same permutation, so the sum over
// k is unchanged.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// 4 signed int8 -> two f16x2 holding the exact integers (elements 0,1 and 2,3).
__device__ __forceinline__ void i8x4_to_h2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;                   // q + 128
    const uint32_t off = 0x64806480u;                     // fp16 1152 = 1024 + 128, twice
    lo = hsub2_bits(__byte_perm(u, 0x64646464u, 0x4140), off);
    hi = hsub2_bits(__byte_perm(u, 0x64646464u, 0x4342), off);
}

// 4 nibbles (in the low nibble of each byte) -> (q - 8) as two f16x2.
__device__ __forceinline__ void u4x4_to_h2x2(uint32_t n, uint32_t& lo, uint32_t& hi) {
    const uint32_t off = 0x64086408u;                     // fp16 1032 = 1024 + 8, twice
    lo = hsub2_bits(__byte_perm(n, 0x64646464u, 0x4140), off);
    hi = hsub2_bits(__byte_perm(n, 0x64646464u, 0x4342), off);
}

constexpr int kMmaWarps = 8;                      // warps per CTA: split of the reduction
constexpr int kXPad = 32;                         // halves of padding per staged activation row

// Stage 8 token rows of a 16-bit activation matrix (row stride `ld` halves,
// K columns) into dst[8][K + kXPad]; rows at or beyond nt are zero.  Eight
// 16-byte loads per thread are in flight before any store.
__device__ __forceinline__ void stage_act16(__half* dst, int K, const __half* src, size_t ld, int nt) {
    const int KP = K + kXPad;
    const int n8 = K / 8, total = 8 * n8;
    constexpr int kB = 8;
    for (int i0 = threadIdx.x; i0 < total; i0 += kB * blockDim.x) {
        uint4 v[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int i = i0 + u * blockDim.x, t = i / n8, c = i - t * n8;
            v[u] = (i < total && t < nt) ? __ldcg(reinterpret_cast<const uint4*>(src + t * ld) + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
            const int i = i0 + u * blockDim.x, t = i / n8, c = i - t * n8;
            if (i < total) *reinterpret_cast<uint4*>(dst + (size_t)t * KP + 8 * c) = v[u];
        }
    }
}

// Q8_0 / Q4_0 rows [r0, r0 + 16) of a matrix [R][C] against the staged
// activations xs[8][C + kXPad], columns [kb0 * 32, kb1 * 32); acc += C frags.
template <int FMT>
__device__ __forceinline__ void mma_du_rows(const uint8_t* mat, int R, int C, int r0, int kb0, int kb1,
                                            const __half* xs, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int KP = C + kXPad;
    const size_t qrow = FMT == LMOE_Q8_0 ? 32 : 16;
    const uint16_t* dsc = reinterpret_cast<const uint16_t*>(mat + (size_t)R * C / 32 * qrow);
    const __half* xrow = xs + (size_t)g * KP;
    constexpr int kU = 4;                                  // blocks whose loads are issued together
    for (int kb = kb0; kb < kb1; kb += kU) {
        uint32_t w[kU][4];
        uint16_t d[kU][2];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (kb + u < kb1) {
                const size_t b = (size_t)(kb + u);
                if (FMT == LMOE_Q8_0) {
                    const uint2 lo = __ldg(reinterpret_cast<const uint2*>(mat + (b * R + r0 + g) * 32 + 8 * t));
                    const uint2 hi = __ldg(reinterpret_cast<const uint2*>(mat + (b * R + r0 + g + 8) * 32 + 8 * t));
                    w[u][0] = lo.x; w[u][1] = lo.y; w[u][2] = hi.x; w[u][3] = hi.y;
                } else {
                    w[u][0] = __ldg(reinterpret_cast<const uint32_t*>(mat + (b * R + r0 + g) * 16 + 4 * t));
                    w[u][2] = __ldg(reinterpret_cast<const uint32_t*>(mat + (b * R + r0 + g + 8) * 16 + 4 * t));
                }
                d[u][0] = __ldg(dsc + b * R + r0 + g);
                d[u][1] = __ldg(dsc + b * R + r0 + g + 8);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (kb + u < kb1) {
                const int k0 = (kb + u) * 32;
                float c[4] = {0.f, 0.f, 0.f, 0.f};
                if (FMT == LMOE_Q8_0) {
                    // thread t: elements 8t .. 8t+7 of rows g and g + 8
                    uint32_t ga0, ga1, ga2, ga3, ha0, ha1, ha2, ha3;
                    i8x4_to_h2x2(w[u][0], ga0, ga1);
                    i8x4_to_h2x2(w[u][1], ga2, ga3);
                    i8x4_to_h2x2(w[u][2], ha0, ha1);
                    i8x4_to_h2x2(w[u][3], ha2, ha3);
                    const uint4 xv = *reinterpret_cast<const uint4*>(xrow + k0 + 8 * t);
                    mma16816(c, ga0, ha0, ga1, ha1, xv.x, xv.y);
                    mma16816(c, ga2, ha2, ga3, ha3, xv.z, xv.w);
                } else {
                    // thread t: elements 4t .. 4t+3 (low nibbles) and 16+4t .. (high)
                    uint32_t gl0, gl1, gh0, gh1, hl0, hl1, hh0, hh1;
                    u4x4_to_h2x2(w[u][0] & 0x0F0F0F0Fu, gl0, gl1);
                    u4x4_to_h2x2((w[u][0] >> 4) & 0x0F0F0F0Fu, gh0, gh1);
                    u4x4_to_h2x2(w[u][2] & 0x0F0F0F0Fu, hl0, hl1);
                    u4x4_to_h2x2((w[u][2] >> 4) & 0x0F0F0F0Fu, hh0, hh1);
                    const uint2 xl = *reinterpret_cast<const uint2*>(xrow + k0 + 4 * t);
                    const uint2 xh = *reinterpret_cast<const uint2*>(xrow + k0 + 16 + 4 * t);
                    mma16816(c, gl0, hl0, gl1, hl1, xl.x, xl.y);
                    mma16816(c, gh0, hh0, gh1, hh1, xh.x, xh.y);
                }
                const float dg = fp16_bits_to_f32(d[u][0]), dh = fp16_bits_to_f32(d[u][1]);
                acc[0] = fmaf(dg, c[0], acc[0]);
                acc[1] = fmaf(dg, c[1], acc[1]);
                acc[2] = fmaf(dh, c[2], acc[2]);
                acc[3] = fmaf(dh, c[3], acc[3]);
            }
        }
    }
}

// NVFP4 rows [r0, r0 + 16) of a matrix [R][C] (codes q, scales s), 32-column
// chunks [kc0, kc1).  The E4M3 scale multiplies the E2M1 value in fp16
// (exact); the tensor scale is left to the caller.
__device__ __forceinline__ void mma_nvfp4_rows(const uint8_t* q, const uint8_t* s, int R, int C, int r0, int kc0,
                                               int kc1, const __half* xs, float (&acc)[4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int KP = C + kXPad;
    const __half* xrow = xs + (size_t)g * KP;
    constexpr int kU = 4;
    for (int kc = kc0; kc < kc1; kc += kU) {
        uint32_t wg[kU], wh[kU], sg[kU], sh[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (kc + u < kc1) {
                const size_t c = (size_t)(kc + u);
                wg[u] = __ldg(reinterpret_cast<const uint32_t*>(q + (c * R + r0 + g) * 16 + 4 * t));
                wh[u] = __ldg(reinterpret_cast<const uint32_t*>(q + (c * R + r0 + g + 8) * 16 + 4 * t));
                sg[u] = __ldg(reinterpret_cast<const uint32_t*>(s + ((c / 2) * R + r0 + g) * 4));
                sh[u] = __ldg(reinterpret_cast<const uint32_t*>(s + ((c / 2) * R + r0 + g + 8) * 4));
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (kc + u < kc1) {
                const int kcu = kc + u;
                // this thread's 8 elements (8t .. 8t+7 of the chunk) share one scale byte
                const int sb = 2 * (kcu & 1) + (t >> 1);
                uint32_t scg, sch;
                {
                    const uint32_t bg = (sg[u] >> (8 * sb)) & 0xFF, bh = (sh[u] >> (8 * sb)) & 0xFF;
                    uint32_t hg, hh;
                    asm("{\n\t.reg .b16 a, b;\n\tcvt.u16.u32 a, %2;\n\tcvt.u16.u32 b, %3;\n\t"
                        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
                        : "=r"(hg), "=r"(hh)
                        : "r"(bg), "r"(bh));
                    scg = (hg & 0xFFFF) | (hg << 16);
                    sch = (hh & 0xFFFF) | (hh << 16);
                }
                uint32_t a[4], b[4];
                e2m1x8_to_f16x8(wg[u], a);
                e2m1x8_to_f16x8(wh[u], b);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    a[j] = hmul2_bits(a[j], scg);
                    b[j] = hmul2_bits(b[j], sch);
                }
                const uint4 xv = *reinterpret_cast<const uint4*>(xrow + kcu * 32 + 8 * t);
                mma16816(acc, a[0], b[0], a[1], b[1], xv.x, xv.y);
                mma16816(acc, a[2], b[2], a[3], b[3], xv.z, xv.w);
            }
        }
    }
}

// Sum the kMmaWarps partial C fragments into warp 0's (others get zeros).
__device__ __forceinline__ void reduce_frags(float (&acc)[4], float* red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < 4; ++i) red[(warp * 32 + lane) * 4 + i] = acc[i];
    __syncthreads();
    if (warp == 0) {
        for (int w = 1; w < kMmaWarps; ++w)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] += red[(w * 32 + lane) * 4 + i];
    }
    __syncthreads();
}

// kernel 2: h16[t][g] = D_g x_t for hit groups; CTA = 16 rows of one group
template <int FMT>
__global__ void __launch_bounds__(32 * kMmaWarps, 4) k_dproj_mma(FwdParams p) {
    extern __shared__ __align__(16) uint8_t smem_u8[];
    const int g = blockIdx.y;
    if (__ldcg(p.r.ghit + g) == 0) return;
    const int H = p.H, L = p.L, r0 = blockIdx.x * 16;
    __half* xs = reinterpret_cast<__half*>(smem_u8);
    float* red = reinterpret_cast<float*>(smem_u8 + (size_t)8 * (H + kXPad) * 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t* Dg = p.D + (size_t)g * p.du_bytes_D;
    const int nb = H / 32, per = (nb + kMmaWarps - 1) / kMmaWarps;
    for (int t0 = 0; t0 < p.T; t0 += 8) {
        const int nt = min(8, p.T - t0);
        stage_act16(xs, H, p.x16 + (size_t)t0 * H, H, nt);
        __syncthreads();
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        mma_du_rows<FMT>(Dg, L, H, r0, warp * per, min(nb, (warp + 1) * per), xs, acc);
        reduce_frags(acc, red);
        if (warp == 0) {
            const int gg = lane >> 2, tt = lane & 3;
            bool bad = false;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = 2 * tt + (i & 1), row = r0 + gg + 8 * (i >> 1);
                if (tok < nt) p.h16[((size_t)(t0 + tok) * p.G + g) * L + row] = half_checked(acc[i], bad);
            }
            report_range(p.ctrl, bad);
        }
    }
}

// kernel 3: z16[slot] = silu(W_gate h) * (W_up h) for the expert's slots;
// CTA = 16 features (gate and up rows) of one distinct expert
__global__ void __launch_bounds__(32 * kMmaWarps, 3) k_gateup_mma(FwdParams p) {
    extern __shared__ __align__(16) uint8_t smem_u8[];
    const int j = blockIdx.y;
    if (j >= __ldcg(p.r.n_unique)) return;
    const int e = __ldcg(p.r.uexp + j), cnt = __ldcg(p.r.ucnt + j), off = __ldcg(p.r.uoff + j);
    const int g = p.group[e] < p.G ? p.group[e] : 0;
    const int L = p.L, F = p.F, f0 = blockIdx.x * 16;
    __half* hs = reinterpret_cast<__half*>(smem_u8);
    float* red = reinterpret_cast<float*>(smem_u8 + (size_t)8 * (L + kXPad) * 2);
    __shared__ int tok[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint8_t* rec = p.experts + (size_t)e * p.rec_bytes;
    const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
    const float* tail = reinterpret_cast<const float*>(rec + 3 * nq + 3 * ns);
    const float ts_g = __ldg(tail), ts_u = __ldg(tail + 1);
    const int nc = L / 32, per = (nc + kMmaWarps - 1) / kMmaWarps;
    for (int c0 = 0; c0 < cnt; c0 += 8) {
        const int nt = min(8, cnt - c0);
        if (threadIdx.x < 8) tok[threadIdx.x] = threadIdx.x < nt ? __ldcg(p.r.slot_pair + off + c0 + threadIdx.x) / p.K : 0;
        __syncthreads();
        // gather the slots' latent inputs h16[token][g] (eight loads in flight per thread)
        {
            const int n8 = L / 8, total = 8 * n8;
            for (int i0 = threadIdx.x; i0 < total; i0 += 8 * blockDim.x) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + u * blockDim.x, t = i / n8, c = i - t * n8;
                    v[u] = (i < total && t < nt) ? __ldcg(reinterpret_cast<const uint4*>(p.h16 + ((size_t)tok[t] * p.G + g) * L) + c)
                                                 : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = i0 + u * blockDim.x, t = i / n8, c = i - t * n8;
                    if (i < total) *reinterpret_cast<uint4*>(hs + (size_t)t * (L + kXPad) + 8 * c) = v[u];
                }
            }
        }
        __syncthreads();
        float a[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
        const int kc0 = warp * per, kc1 = min(nc, (warp + 1) * per);
        mma_nvfp4_rows(rec, rec + 3 * nq, F, L, f0, kc0, kc1, hs, a);
        mma_nvfp4_rows(rec + nq, rec + 3 * nq + ns, F, L, f0, kc0, kc1, hs, u);
        reduce_frags(a, red);
        reduce_frags(u, red);
        if (warp == 0) {
            const int gg = lane >> 2, tt = lane & 3;
            bool bad = false;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = 2 * tt + (i & 1), f = f0 + gg + 8 * (i >> 1);
                if (col < nt) p.z16[(size_t)(off + c0 + col) * F + f] = half_checked(silu(a[i] * ts_g) * (u[i] * ts_u), bad);
            }
            report_range(p.ctrl, bad);
        }
        __syncthreads();
    }
}

// kernel 4: s16[t][g] = sum over the token's experts of group g of w * (W_down z);
// CTA = 16 latent rows of one group; each warp takes whole experts of the
// group (K = ffn in one warp, no reduction), the group sum is formed in a
// fixed order afterwards.
constexpr int kDownWarps = 4;

__global__ void __launch_bounds__(32 * kDownWarps, 4) k_down_mma(FwdParams p) {
    extern __shared__ __align__(16) uint8_t smem_u8[];
    const int g = blockIdx.y;
    const int L = p.L, F = p.F, T = p.T, r0 = blockIdx.x * 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KP = F + kXPad;
    __half* zs = reinterpret_cast<__half*>(smem_u8);                       // [kDownWarps][8][F + pad]
    float* part = reinterpret_cast<float*>(smem_u8 + (size_t)kDownWarps * 8 * KP * 2);  // [T * K][16] per slot
    __shared__ int elist[kMaxTopK * kChunk];
    __shared__ int n_e;
    // group label and slot of every (token, k) pair, for the final sum
    __shared__ uint8_t pg[kMaxTopK * 64];
    __shared__ int pslot[kMaxTopK * 64];
    const bool pairs_in_smem = T * p.K <= kMaxTopK * 64;
    for (int i = threadIdx.x; pairs_in_smem && i < T * p.K; i += blockDim.x) {
        const int e = __ldcg(p.r.idx + i);
        pg[i] = p.group[e] < p.G ? p.group[e] : 0;
        pslot[i] = __ldcg(p.r.pair_slot + i);
    }
    const int n_unique = __ldcg(p.r.n_unique);
    const bool hit = __ldcg(p.r.ghit + g) > 0;
    if (threadIdx.x == 0) {
        int n = 0;
        for (int j = 0; hit && j < n_unique; ++j)
            if (p.group[__ldcg(p.r.uexp + j)] == g && n < kMaxTopK * kChunk) elist[n++] = j;
        n_e = n;
    }
    __syncthreads();
    const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
    __half* zw = zs + (size_t)warp * 8 * KP;
    for (int ii = warp; ii < n_e; ii += kDownWarps) {
        const int j = elist[ii];
        const int e = __ldcg(p.r.uexp + j), cnt = __ldcg(p.r.ucnt + j), off = __ldcg(p.r.uoff + j);
        const uint8_t* rec = p.experts + (size_t)e * p.rec_bytes;
        const float ts_d = __ldg(reinterpret_cast<const float*>(rec + 3 * nq + 3 * ns) + 2);
        for (int c0 = 0; c0 < cnt; c0 += 8) {
            const int nt = min(8, cnt - c0);
            // this warp's 8 slot rows of z (fp16), zero beyond nt
            for (int i = lane; i < 8 * (F / 8); i += 32) {
                const int t = i / (F / 8), c = i - t * (F / 8);
                const uint4 v = t < nt ? __ldcg(reinterpret_cast<const uint4*>(p.z16 + (size_t)(off + c0 + t) * F) + c)
                                       : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(zw + (size_t)t * KP + 8 * c) = v;
            }
            __syncwarp();
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            mma_nvfp4_rows(rec + 2 * nq, rec + 3 * nq + 2 * ns, L, F, r0, 0, F / 32, zw, acc);
            const int gg = lane >> 2, tt = lane & 3;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = 2 * tt + (i & 1), row = gg + 8 * (i >> 1);
                if (col < nt) {
                    const int slot = off + c0 + col;
                    part[(size_t)slot * 16 + row] = __ldcg(p.r.w + __ldcg(p.r.slot_pair + slot)) * (acc[i] * ts_d);
                }
            }
            __syncwarp();
        }
    }
    __syncthreads();
    // group sum per (row, token), experts in ascending order (deterministic)
    bool bad = false;
    for (int i = threadIdx.x; i < 16 * T; i += blockDim.x) {
        const int row = i / T, t = i - row * T;
        float v = 0.f;
        if (hit) {
            for (int k = 0; k < p.K; ++k) {
                const int pair = t * p.K + k;
                if (pairs_in_smem) {
                    if (pg[pair] == g) v += part[(size_t)pslot[pair] * 16 + row];
                } else if (p.group[__ldcg(p.r.idx + pair)] == g) {
                    v += part[(size_t)__ldcg(p.r.pair_slot + pair) * 16 + row];
                }
            }
        }
        p.s16[((size_t)t * p.G + g) * L + r0 + row] = half_checked(v, bad);
    }
    report_range(p.ctrl, bad);
}

// kernel 5: per 16 output rows, one part per hit group (U_g s16[t][g]) and
// one for the shared expert's down projection; the last part of a row tile
// to finish sums the parts in a fixed order, adds the residual, writes y.
template <int FMT>
__global__ void __launch_bounds__(32 * kMmaWarps, 3) k_uproj_mma(FwdParams p) {
    extern __shared__ __align__(16) uint8_t smem_u8[];
    const int part = blockIdx.y;
    const int H = p.H, L = p.L, G = p.G, T = p.T, r0 = blockIdx.x * 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool active = part == G || __ldcg(p.r.ghit + part) > 0;
    if (active) {
        for (int t0 = 0; t0 < T; t0 += 8) {
            const int nt = min(8, T - t0);
            if (part < G) {
                __half* ss = reinterpret_cast<__half*>(smem_u8);
                float* red = reinterpret_cast<float*>(smem_u8 + (size_t)8 * (L + kXPad) * 2);
                stage_act16(ss, L, p.s16 + ((size_t)t0 * G + part) * L, (size_t)G * L, nt);
                __syncthreads();
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const int nb = L / 32, per = (nb + kMmaWarps - 1) / kMmaWarps;
                mma_du_rows<FMT>(p.U + (size_t)part * p.du_bytes_U, H, L, r0, warp * per, min(nb, (warp + 1) * per),
                                 ss, acc);
                reduce_frags(acc, red);
                if (warp == 0) {
                    const int gg = lane >> 2, tt = lane & 3;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int tok = 2 * tt + (i & 1), row = r0 + gg + 8 * (i >> 1);
                        if (tok < nt) p.ypart[((size_t)part * T + t0 + tok) * H + row] = acc[i];
                    }
                }
            } else {
                // shared expert: 4 rows per warp on CUDA cores (bf16 weights, fp32 hidden)
                float* as = reinterpret_cast<float*>(smem_u8);      // [8][Fs + 4]
                const int Fs = p.Fs, ld = xs_ld(Fs), n4 = Fs / 4;
                for (int i0 = threadIdx.x; i0 < 8 * n4; i0 += 4 * blockDim.x) {
                    float4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u * blockDim.x, t = i / n4, c = i - t * n4;
                        v[u] = (i < 8 * n4 && t < nt) ? __ldcg(reinterpret_cast<const float4*>(p.zsh + (size_t)(t0 + t) * Fs) + c)
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u * blockDim.x, t = i / n4, c = i - t * n4;
                        if (i < 8 * n4) *reinterpret_cast<float4*>(as + t * ld + 4 * c) = v[u];
                    }
                }
                __syncthreads();
                for (int rr = warp; rr < 16; rr += kMmaWarps) {
                    const int row = r0 + rr;
                    float a2[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) a2[t] = 0.f;
                    row_dot<8, true, 3>(p.sd + (size_t)row * Fs, Fs, as, ld, lane, a2);
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        const float v = warp_sum(a2[t]);
                        if (lane == 0 && t < nt) p.ypart[((size_t)G * T + t0 + t) * H + row] = v;
                    }
                }
            }
            __syncthreads();
        }
    }
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int done = atomicAdd(&p.ctrl->tile_ticket[blockIdx.x], 1);
        s_last = (done == G);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    __shared__ uint8_t th[64 * kMaxGroups];
    const bool hits_in_smem = T * G <= 64 * kMaxGroups;
    for (int i = threadIdx.x; hits_in_smem && i < T * G; i += blockDim.x)
        th[i] = p.r.tghit[i] && __ldcg(p.r.ghit + i % G) > 0;
    __syncthreads();
    for (int i = threadIdx.x; i < T * 16; i += blockDim.x) {
        const int t = i >> 4, row = r0 + (i & 15);
        float v = __ldcg(p.ypart + ((size_t)G * T + t) * H + row);
        for (int g = 0; g < G; ++g) {
            const bool h = hits_in_smem ? th[t * G + g] != 0 : (p.r.tghit[(size_t)t * G + g] && __ldcg(p.r.ghit + g) > 0);
            if (h) v += __ldcg(p.ypart + ((size_t)g * T + t) * H + row);
        }
        if (p.residual) v += bf16_bits_to_f32(p.residual[(size_t)t * H + row]);
        p.y[(size_t)t * H + row] = f32_to_bf16_bits(v);
    }
    if (threadIdx.x == 0) p.ctrl->tile_ticket[blockIdx.x] = 0;
}

// ---------------------------------------------------------------------------
// host launch of the decode path
// ---------------------------------------------------------------------------

// Optional CUDA events recorded around each kernel (profiling).
static cudaEvent_t g_stage_events[kMaxStageEvents];
static int g_n_stage_events = 0;
static int g_stage_cursor = 0;

void set_stage_events(void* const* events, int n) {
    g_n_stage_events = n;
    for (int i = 0; i < n; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
}

void stage_mark(cudaStream_t st) {
    if (g_stage_cursor < g_n_stage_events) cudaEventRecord(g_stage_events[g_stage_cursor++], st);
}

void stage_reset() { g_stage_cursor = 0; }

// Raise a kernel's dynamic shared-memory limit when needed (static + dynamic
// above 48 KiB needs the opt-in); remembered per kernel and device.
cudaError_t ensure_smem(const void* kernel, size_t smem) {
    struct Entry { const void* k; int dev; size_t bytes; };
    static Entry table[128];
    static int n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    for (int i = 0; i < n; ++i)
        if (table[i].k == kernel && table[i].dev == dev && table[i].bytes >= smem) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    for (int i = 0; i < n; ++i)
        if (table[i].k == kernel && table[i].dev == dev) { table[i].bytes = smem; return cudaSuccess; }
    if (n < 128) table[n++] = {kernel, dev, smem};
    return cudaSuccess;
}

template <typename Kern>
static cudaError_t launch(Kern k, dim3 grid, int threads, size_t smem, cudaStream_t st, const FwdParams& p) {
    stage_mark(st);
    if (smem > 0) {
        cudaError_t e = ensure_smem(reinterpret_cast<const void*>(k), smem);
        if (e != cudaSuccess) return e;
    }
    k<<<grid, threads, smem, st>>>(p);
    return cudaGetLastError();
}

template <int NT>
static cudaError_t run_gemv_path_nt(FwdParams p, cudaStream_t st, bool route_only) {
    // 1. router (+ shared gate/up, top-k, buckets): one warp per router row / shared feature
    p.router_rows_per_warp = 1;
    p.n_router_ctas = (p.E + 7) / 8;
    // the shared expert's gate/up run in the router kernel's other CTAs (as
    // items of the D kernel, whose items are split by count, their 80-step
    // items left a few CTAs four times the work of the rest)
    p.shared_in_d = false;
    p.do_shared = !route_only;
    p.do_buckets = !route_only;
    // few tokens, whole block: the routing is built in shared memory and
    // published with every table the weight-streaming kernels read
    p.route_smem = !route_only && p.T <= 8;
    // the weight-streaming kernels read the block input themselves
    if (p.route_smem) p.x16 = nullptr;
    p.prefetch_l2 = false;
    const int n_shared_ctas = p.do_shared ? (p.Fs + 7) / 8 : 0;
    if (p.route_smem && p.wtick) {
        // tickets of the split reductions of the weight-streaming kernels
        cudaError_t e = cudaMemsetAsync(p.wtick, 0, p.wtick_bytes, st);
        if (e != cudaSuccess) return e;
    }
    {
        size_t sm = (size_t)xs_ld(p.H) * NT * sizeof(float);
        cudaError_t e = p.router_bf16
            ? launch(k_router_shared<NT, true>, dim3(p.n_router_ctas + n_shared_ctas), 256, sm, st, p)
            : launch(k_router_shared<NT, false>, dim3(p.n_router_ctas + n_shared_ctas), 256, sm, st, p);
        if (e != cudaSuccess || route_only) return e;
    }
    if (p.T <= 8) return run_stream_path(p, st);
    const int max_unique = min(p.T * p.K, p.E);
    const size_t red = (size_t)kMmaWarps * 32 * 4 * sizeof(float);
    const int thr = 32 * kMmaWarps;
    cudaError_t e;
    const size_t sm_d = (size_t)8 * (p.H + kXPad) * 2 + red;
    e = p.du_fmt == LMOE_Q8_0 ? launch(k_dproj_mma<LMOE_Q8_0>, dim3(p.L / 16, p.G), thr, sm_d, st, p)
                              : launch(k_dproj_mma<LMOE_Q4_0>, dim3(p.L / 16, p.G), thr, sm_d, st, p);
    if (e != cudaSuccess) return e;
    e = launch(k_gateup_mma, dim3(p.F / 16, max_unique), thr, (size_t)8 * (p.L + kXPad) * 2 + red, st, p);
    if (e != cudaSuccess) return e;
    e = launch(k_down_mma, dim3(p.L / 16, p.G), 32 * kDownWarps,
               (size_t)kDownWarps * 8 * (p.F + kXPad) * 2 + (size_t)p.T * p.K * 16 * 4, st, p);
    if (e != cudaSuccess) return e;
    const size_t sm_u = max((size_t)8 * (p.L + kXPad) * 2 + red, (size_t)xs_ld(p.Fs) * 8 * 4);
    e = p.du_fmt == LMOE_Q8_0 ? launch(k_uproj_mma<LMOE_Q8_0>, dim3(p.H / 16, p.G + 1), thr, sm_u, st, p)
                              : launch(k_uproj_mma<LMOE_Q4_0>, dim3(p.H / 16, p.G + 1), thr, sm_u, st, p);
    return e;
}

cudaError_t run_gemv_path(const FwdParams& p, cudaStream_t st, bool route_only) {
    const int T = p.T;
    g_stage_cursor = 0;
    cudaError_t e;
    if (T <= 1) e = run_gemv_path_nt<1>(p, st, route_only);
    else if (T <= 2) e = run_gemv_path_nt<2>(p, st, route_only);
    else if (T <= 4) e = run_gemv_path_nt<4>(p, st, route_only);
    else e = run_gemv_path_nt<8>(p, st, route_only);
    stage_mark(st);
    return e;
}

// ---------------------------------------------------------------------------
// diagnostics: decode a stored matrix with the kernels' decoders
// ---------------------------------------------------------------------------

__global__ void k_debug_decode(int fmt, const uint8_t* blob, int R, int C, float ts, float* out) {
    const int r = blockIdx.x;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        float v;
        if (fmt == 2) {
            v = q3k_element(blob, R, C, r, c);
        } else if (fmt == 3) {
            v = iq4nl_element(blob, R, C, r, c);
        } else if (fmt == LMOE_Q8_0 || fmt == LMOE_Q4_0) {
            const int b = c / 32, j = c % 32;
            const size_t qrow = fmt == LMOE_Q8_0 ? 32 : 16;
            const uint16_t d = reinterpret_cast<const uint16_t*>(blob + (size_t)R * (C / 32) * qrow)[(size_t)b * R + r];
            const uint8_t* q = blob + ((size_t)b * R + r) * qrow;
            if (fmt == LMOE_Q8_0) {
                v = fp16_bits_to_f32(d) * (float)(int8_t)q[j];
            } else {
                const int nib = j < 16 ? (q[j] & 0xF) : (q[j - 16] >> 4);
                v = fp16_bits_to_f32(d) * (float)(nib - 8);
            }
        } else {
            const uint8_t* q = blob;
            const uint8_t* s = blob + (size_t)R * C / 2;
            const uint32_t word = reinterpret_cast<const uint32_t*>(q + ((size_t)(c / 32) * R + r) * 16)[(c % 32) / 8];
            uint32_t h[4];
            e2m1x8_to_f16x8(word, h);
            const float2 pr = f16x2_to_f32x2(h[(c % 8) / 2]);
            float sc[4];
            e4m3x4_to_f32x4(reinterpret_cast<const uint32_t*>(s)[(size_t)(c / 64) * R + r], sc);
            v = ((c & 1) ? pr.y : pr.x) * sc[(c % 64) / 16] * ts;
        }
        out[(size_t)r * C + c] = v;
    }
}

cudaError_t run_debug_decode(int fmt, const void* blob, int R, int C, float ts, float* out, cudaStream_t st) {
    k_debug_decode<<<R, 128, 0, st>>>(fmt, static_cast<const uint8_t*>(blob), R, C, ts, out);
    return cudaGetLastError();
}

}  // namespace lmoe
