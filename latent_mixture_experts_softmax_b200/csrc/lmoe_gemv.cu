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

#include "lmoe_internal.cuh"

namespace lmoe {

// ---------------------------------------------------------------------------
// activation staging: dst[k * NT + t] = act(t0 + t, k) for t < nt, 0 beyond
// ---------------------------------------------------------------------------

// x rows are bf16 [T][H]; with gamma != nullptr the row is RMS-normalised
// first: gamma[k] * x[k] / sqrt(mean(x^2) + eps).
template <int NT>
__device__ void stage_x(const FwdParams& p, int t0, int nt, float* xs, float* rs) {
    const int H = p.H;
    const int tid = threadIdx.x, nthr = blockDim.x;
    if (p.gamma != nullptr) {
        const int warp = tid >> 5, lane = tid & 31;
        for (int t = warp; t < NT; t += nthr >> 5) {
            float ss = 0.f;
            if (t < nt) {
                const uint16_t* row = p.x + (size_t)(t0 + t) * H;
                for (int k = lane; k < H; k += 32) {
                    float v = bf16_bits_to_f32(row[k]);
                    ss += v * v;
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) rs[t] = rsqrtf(ss / (float)H + p.eps);
        }
        __syncthreads();
    }
    for (int i = tid; i < NT * H; i += nthr) {
        const int t = i / H, k = i - t * H;
        float v = 0.f;
        if (t < nt) {
            v = bf16_bits_to_f32(p.x[(size_t)(t0 + t) * H + k]);
            if (p.gamma != nullptr) v *= rs[t] * bf16_bits_to_f32(p.gamma[k]);
        }
        xs[k * NT + t] = v;
    }
}

// ---------------------------------------------------------------------------
// inner products of one stored row segment with NT staged activations
// ---------------------------------------------------------------------------

// 8 bf16 weights (one 16-byte load) against xs[(k0 + j) * NT + t].
template <int NT>
__device__ __forceinline__ void dot8_bf16(uint4 wv, const float* xs, int k0, float (&acc)[NT]) {
    const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int j2 = 0; j2 < 4; ++j2) {
        const float2 w = bf16x2_to_f32x2(w4[j2]);
        const float* x0 = xs + (k0 + 2 * j2) * NT;
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = fmaf(w.x, x0[t], acc[t]);
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = fmaf(w.y, x0[NT + t], acc[t]);
    }
}

// 4 fp32 weights against xs.
template <int NT>
__device__ __forceinline__ void dot4_f32(float4 w, const float* xs, int k0, float (&acc)[NT]) {
    const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = fmaf(wv[j], xs[(k0 + j) * NT + t], acc[t]);
    }
}

// One Q8_0 block (32 int8 in a, b; scale d) against xs[(k0 + j) * NT + t].
template <int NT>
__device__ __forceinline__ void dot_q8_0_regs(uint4 a, uint4 b, float d, const float* xs, int k0, float (&acc)[NT]) {
    const uint32_t w8[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float blk[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) blk[t] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float wq = (float)(int8_t)((w8[i] >> (8 * j)) & 0xFF);
            const float* xk = xs + (k0 + 4 * i + j) * NT;
#pragma unroll
            for (int t = 0; t < NT; ++t) blk[t] = fmaf(wq, xk[t], blk[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = fmaf(d, blk[t], acc[t]);
}

// One Q4_0 block (16 bytes: byte j = elements j (low) and j+16 (high)).
template <int NT>
__device__ __forceinline__ void dot_q4_0_regs(uint4 a, float d, const float* xs, int k0, float (&acc)[NT]) {
    const uint32_t w4[4] = {a.x, a.y, a.z, a.w};
    float blk[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) blk[t] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t byte = (w4[i] >> (8 * j)) & 0xFF;
            const float lo = (float)((int)(byte & 0xF) - 8);
            const float hi = (float)((int)(byte >> 4) - 8);
            const float* xl = xs + (k0 + 4 * i + j) * NT;
            const float* xh = xs + (k0 + 16 + 4 * i + j) * NT;
#pragma unroll
            for (int t = 0; t < NT; ++t) blk[t] = fmaf(lo, xl[t], blk[t]);
#pragma unroll
            for (int t = 0; t < NT; ++t) blk[t] = fmaf(hi, xh[t], blk[t]);
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = fmaf(d, blk[t], acc[t]);
}

// One 32-element NVFP4 chunk (16 bytes of codes) with the two E4M3 scales of
// its halves (s0: elements 0..15, s1: 16..31).
template <int NT>
__device__ __forceinline__ void dot_nvfp4_chunk(uint4 qv, float s0, float s1, const float* xs, int k0,
                                                float (&acc)[NT]) {
    const uint32_t w4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float blk[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) blk[t] = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t h[4];
            e2m1x8_to_f16x8(w4[2 * half + i], h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 v = f16x2_to_f32x2(h[j]);
                const float* xk = xs + (k0 + 16 * half + 8 * i + 2 * j) * NT;
#pragma unroll
                for (int t = 0; t < NT; ++t) blk[t] = fmaf(v.x, xk[t], blk[t]);
#pragma unroll
                for (int t = 0; t < NT; ++t) blk[t] = fmaf(v.y, xk[NT + t], blk[t]);
            }
        }
        const float s = half ? s1 : s0;
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = fmaf(s, blk[t], acc[t]);
    }
}

// One row of a plain bf16 / fp32 matrix (K contiguous) against xs, the warp's
// lanes splitting K; ten 16-byte loads per lane are issued before any
// arithmetic.  The per-lane partial sums are left in acc (reduce with warp_sum).
template <int NT, bool kBF16>
__device__ __forceinline__ void row_dot(const void* wrow, int K, const float* xs, int lane, float (&acc)[NT]) {
    constexpr int kB = 10;
    constexpr int kPer = kBF16 ? 8 : 4;          // elements per 16-byte load
    constexpr int kStep = 32 * kPer;
    for (int base = 0; base < K; base += kB * kStep) {
        uint4 w[kB];
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            const int k0 = base + i * kStep + lane * kPer;
            if (k0 < K) w[i] = ldg_stream(reinterpret_cast<const uint4*>(static_cast<const char*>(wrow) + (size_t)k0 * (kBF16 ? 2 : 4)));
        }
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            const int k0 = base + i * kStep + lane * kPer;
            if (k0 < K) {
                if (kBF16) dot8_bf16<NT>(w[i], xs, k0, acc);
                else dot4_f32<NT>(make_float4(__uint_as_float(w[i].x), __uint_as_float(w[i].y), __uint_as_float(w[i].z),
                                              __uint_as_float(w[i].w)), xs, k0, acc);
            }
        }
    }
}

// Row-tile GEMV over a D/U matrix [R rows][C cols] stored as Q8_0 / Q4_0:
// lane = row, warps split the 64-wide column groups.  Each warp takes two
// groups per pass and issues all their loads before any arithmetic.
template <int NT>
__device__ __forceinline__ void du_rows(int fmt, const uint8_t* mat, int R, int C, int row, const float* xs,
                                        float (&acc)[NT]) {
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int ng = C / 64;
    const uint16_t* dsc = reinterpret_cast<const uint16_t*>(mat + (size_t)R * C / 32 * (fmt == LMOE_Q8_0 ? 32 : 16));
    for (int base = warp; base < ng; base += 2 * nwarps) {
        const int kg[2] = {base, base + nwarps};
        if (fmt == LMOE_Q8_0) {
            uint4 q[2][4];
            uint16_t d[2][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (kg[u] < ng) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint4* src = reinterpret_cast<const uint4*>(mat + ((size_t)(2 * kg[u] + c) * R + row) * 32);
                        q[u][2 * c] = ldg_stream(src);
                        q[u][2 * c + 1] = ldg_stream(src + 1);
                        d[u][c] = __ldg(dsc + (size_t)(2 * kg[u] + c) * R + row);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (kg[u] < ng) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        dot_q8_0_regs<NT>(q[u][2 * c], q[u][2 * c + 1], fp16_bits_to_f32(d[u][c]), xs,
                                          64 * kg[u] + 32 * c, acc);
                }
            }
        } else {
            uint4 q[2][2];
            uint16_t d[2][2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (kg[u] < ng) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        q[u][c] = ldg_stream(reinterpret_cast<const uint4*>(mat + ((size_t)(2 * kg[u] + c) * R + row) * 16));
                        d[u][c] = __ldg(dsc + (size_t)(2 * kg[u] + c) * R + row);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (kg[u] < ng) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        dot_q4_0_regs<NT>(q[u][c], fp16_bits_to_f32(d[u][c]), xs, 64 * kg[u] + 32 * c, acc);
                }
            }
        }
    }
}

// NVFP4 matrix [R rows][C cols] (codes at q, scales at s), rows as above.
template <int NT>
__device__ __forceinline__ void nvfp4_rows(const uint8_t* q, const uint8_t* s, int R, int C, int row,
                                           const float* xs, float (&acc)[NT]) {
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int ng = C / 64;
    for (int base = warp; base < ng; base += 2 * nwarps) {
        const int kg[2] = {base, base + nwarps};
        uint4 qv[2][2];
        uint32_t sw[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (kg[u] < ng) {
                sw[u] = __ldg(reinterpret_cast<const uint32_t*>(s + ((size_t)kg[u] * R + row) * 4));
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    qv[u][c] = ldg_stream(reinterpret_cast<const uint4*>(q + ((size_t)(2 * kg[u] + c) * R + row) * 16));
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (kg[u] < ng) {
                float sc[4];
                e4m3x4_to_f32x4(sw[u], sc);
#pragma unroll
                for (int c = 0; c < 2; ++c) dot_nvfp4_chunk<NT>(qv[u][c], sc[2 * c], sc[2 * c + 1], xs, 64 * kg[u] + 32 * c, acc);
            }
        }
    }
}

// Sum per-warp partials red[warp][lane][t] into warp 0's acc (others get junk).
template <int NT>
__device__ __forceinline__ void reduce_warps(float (&acc)[NT], float* red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
#pragma unroll
    for (int t = 0; t < NT; ++t) red[(warp * 32 + lane) * NT + t] = acc[t];
    __syncthreads();
    if (warp == 0) {
        for (int w = 1; w < nwarps; ++w) {
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] += red[(w * 32 + lane) * NT + t];
        }
    }
    __syncthreads();
}

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
    if (!router_cta && !p.do_shared) return;
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
                if (kRouterBF16) row_dot<NT, true>(static_cast<const uint16_t*>(p.router_w) + (size_t)e * H, H, xs, lane, acc);
                else row_dot<NT, false>(static_cast<const float*>(p.router_w) + (size_t)e * H, H, xs, lane, acc);
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
                row_dot<NT, true>(p.sg + (size_t)f * H, H, xs, lane, a);
                row_dot<NT, true>(p.su + (size_t)f * H, H, xs, lane, u);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float av = warp_sum(a[t]), uv = warp_sum(u[t]);
                    if (lane == 0 && t < nt) p.zsh[(size_t)(t0 + t) * p.Fs + f] = silu(av) * uv;
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
    topk_and_buckets(p);
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
            float v[kMaxExpertsTopk / 32];
            uint32_t taken = 0;
#pragma unroll
            for (int j = 0; j < kMaxExpertsTopk / 32; ++j) {
                const int e = lane + 32 * j;
                v[j] = e < E ? __ldcg(r.logits + (size_t)t * E + e) : -INFINITY;
            }
            float lmax = 0.f, denom = 0.f;
            float sel_l[kMaxTopK];
            int sel_e[kMaxTopK];
            for (int k = 0; k < K; ++k) {
                float bv = -INFINITY;
                int bi = 0x7fffffff;
#pragma unroll
                for (int j = 0; j < kMaxExpertsTopk / 32; ++j) {
                    const int e = lane + 32 * j;
                    if (e < E && !(taken >> j & 1u) && (v[j] > bv || (v[j] == bv && e < bi))) { bv = v[j]; bi = e; }
                }
                warp_argmax(bv, bi);
                if ((bi & 31) == lane && bi < E) taken |= 1u << (bi >> 5);
                if (k == 0) lmax = bv;
                sel_l[k] = bv;
                sel_e[k] = bi;
                denom += expf(bv - lmax);
            }
            if (lane < K) {
                float lk = 0.f;
                int ek = 0;
#pragma unroll
                for (int k = 0; k < kMaxTopK; ++k) if (k == lane) { lk = sel_l[k]; ek = sel_e[k]; }
                r.idx[(size_t)t * K + lane] = ek;
                r.w[(size_t)t * K + lane] = expf(lk - lmax) / denom;
            }
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
// kernel 2: h[t][g] = D_g x_t
// ---------------------------------------------------------------------------

template <int NT>
__global__ void __launch_bounds__(512) k_dproj(FwdParams p) {
    extern __shared__ float smem[];
    __shared__ float rs[kChunk];
    const int g = blockIdx.y;
    if (__ldcg(p.r.ghit + g) == 0) return;
    float* xs = smem;                       // [H][NT]
    float* red = smem + (size_t)p.H * NT;   // [8][32][NT]
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 32 + lane;
    const uint8_t* Dg = p.D + (size_t)g * p.du_bytes_D;
    for (int t0 = 0; t0 < p.T; t0 += NT) {
        const int nt = min(NT, p.T - t0);
        stage_x<NT>(p, t0, nt, xs, rs);
        __syncthreads();
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
        du_rows<NT>(p.du_fmt, Dg, p.L, p.H, row, xs, acc);
        reduce_warps<NT>(acc, red);
        if (threadIdx.x < 32) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (t < nt) p.h[((size_t)(t0 + t) * p.G + g) * p.L + row] = acc[t];
        }
    }
}

// ---------------------------------------------------------------------------
// kernels 3 and 4: experts (one CTA = 32 rows of one distinct expert)
// ---------------------------------------------------------------------------

template <int NT>
__global__ void __launch_bounds__(512) k_expert_gateup(FwdParams p) {
    extern __shared__ float smem[];
    const int j = blockIdx.y;
    const int n_unique = __ldcg(p.r.n_unique);
    if (j >= n_unique) return;
    const int e = __ldcg(p.r.uexp + j), cnt = __ldcg(p.r.ucnt + j), off = __ldcg(p.r.uoff + j);
    const int g = p.group[e] < p.G ? p.group[e] : 0;
    const int L = p.L, F = p.F;
    float* hs = smem;                        // [L][NT]
    float* red = smem + (size_t)L * NT;      // [8][32][NT]
    __shared__ int tok[kChunk];
    const int lane = threadIdx.x & 31;
    const int f = blockIdx.x * 32 + lane;
    const uint8_t* rec = p.experts + (size_t)e * p.rec_bytes;
    const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
    float ts[2];
    ts[0] = __ldg(reinterpret_cast<const float*>(rec + 3 * nq + 3 * ns));
    ts[1] = __ldg(reinterpret_cast<const float*>(rec + 3 * nq + 3 * ns) + 1);
    for (int c0 = 0; c0 < cnt; c0 += NT) {
        const int nt = min(NT, cnt - c0);
        if (threadIdx.x < NT) tok[threadIdx.x] = threadIdx.x < nt ? __ldcg(p.r.slot_pair + off + c0 + threadIdx.x) / p.K : -1;
        __syncthreads();
        for (int i = threadIdx.x; i < NT * L; i += blockDim.x) {
            const int t = i / L, k = i - t * L;
            hs[k * NT + t] = tok[t] >= 0 ? __ldcg(p.h + ((size_t)tok[t] * p.G + g) * L + k) : 0.f;
        }
        __syncthreads();
        float a[NT], u[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) { a[t] = 0.f; u[t] = 0.f; }
        nvfp4_rows<NT>(rec, rec + 3 * nq, F, L, f, hs, a);
        nvfp4_rows<NT>(rec + nq, rec + 3 * nq + ns, F, L, f, hs, u);
        reduce_warps<NT>(a, red);
        reduce_warps<NT>(u, red);
        if (threadIdx.x < 32) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (t < nt) p.z[(size_t)(off + c0 + t) * F + f] = silu(a[t] * ts[0]) * (u[t] * ts[1]);
        }
        __syncthreads();
    }
}

template <int NT>
__global__ void __launch_bounds__(512) k_expert_down(FwdParams p) {
    extern __shared__ float smem[];
    const int j = blockIdx.y;
    const int n_unique = __ldcg(p.r.n_unique);
    if (j >= n_unique) return;
    const int e = __ldcg(p.r.uexp + j), cnt = __ldcg(p.r.ucnt + j), off = __ldcg(p.r.uoff + j);
    const int L = p.L, F = p.F;
    float* zs = smem;                        // [F][NT]
    float* red = smem + (size_t)F * NT;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 32 + lane;
    const uint8_t* rec = p.experts + (size_t)e * p.rec_bytes;
    const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
    const float ts = __ldg(reinterpret_cast<const float*>(rec + 3 * nq + 3 * ns) + 2);
    for (int c0 = 0; c0 < cnt; c0 += NT) {
        const int nt = min(NT, cnt - c0);
        for (int i = threadIdx.x; i < NT * F; i += blockDim.x) {
            const int t = i / F, k = i - t * F;
            zs[k * NT + t] = t < nt ? __ldcg(p.z + (size_t)(off + c0 + t) * F + k) : 0.f;
        }
        __syncthreads();
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.f;
        nvfp4_rows<NT>(rec + 2 * nq, rec + 3 * nq + 2 * ns, L, F, row, zs, acc);
        reduce_warps<NT>(acc, red);
        if (threadIdx.x < 32) {
#pragma unroll
            for (int t = 0; t < NT; ++t)
                if (t < nt) p.o[(size_t)(off + c0 + t) * L + row] = acc[t] * ts;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// kernel 5: U_g of the per-group weighted sums, shared down, combine
// ---------------------------------------------------------------------------

template <int NT>
__global__ void __launch_bounds__(512) k_uproj(FwdParams p) {
    extern __shared__ float smem[];
    const int part = blockIdx.y;            // 0..G-1: group; G: shared expert
    const int H = p.H, L = p.L, G = p.G, K = p.K, T = p.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * 32;
    const bool active = part == G || __ldcg(p.r.ghit + part) > 0;
    __shared__ int lst_slot[kChunk * kMaxTopK];
    __shared__ float lst_w[kChunk * kMaxTopK];
    __shared__ int lst_n[kChunk];
    if (active) {
        float* as = smem;                                   // [max(L, Fs)][NT]
        float* red = smem + (size_t)max(L, p.Fs) * NT;
        for (int t0 = 0; t0 < T; t0 += NT) {
            const int nt = min(NT, T - t0);
            float acc[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = 0.f;
            if (part < G) {
                // s[t][k] = sum over the token's experts of group `part` of w * o
                if (threadIdx.x < NT) {
                    const int t = threadIdx.x;
                    int n = 0;
                    if (t < nt && p.r.tghit[(size_t)(t0 + t) * G + part]) {
                        for (int kk = 0; kk < K; ++kk) {
                            const int pair = (t0 + t) * K + kk;
                            const int e = __ldcg(p.r.idx + pair);
                            if (p.group[e] == part) {
                                lst_slot[t * kMaxTopK + n] = __ldcg(p.r.pair_slot + pair);
                                lst_w[t * kMaxTopK + n] = __ldcg(p.r.w + pair);
                                ++n;
                            }
                        }
                    }
                    lst_n[t] = n;
                }
                __syncthreads();
                for (int i = threadIdx.x; i < NT * L; i += blockDim.x) {
                    const int t = i / L, k = i - t * L;
                    float s = 0.f;
                    for (int j = 0; j < lst_n[t]; ++j)
                        s = fmaf(lst_w[t * kMaxTopK + j], __ldcg(p.o + (size_t)lst_slot[t * kMaxTopK + j] * L + k), s);
                    as[k * NT + t] = s;
                }
                __syncthreads();
                du_rows<NT>(p.du_fmt, p.U + (size_t)part * p.du_bytes_U, H, L, row0 + lane, as, acc);
                reduce_warps<NT>(acc, red);
                if (threadIdx.x < 32) {
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        if (t < nt) p.ypart[((size_t)part * T + t0 + t) * H + row0 + lane] = acc[t];
                }
            } else {
                const int Fs = p.Fs;
                for (int i = threadIdx.x; i < NT * Fs; i += blockDim.x) {
                    const int t = i / Fs, k = i - t * Fs;
                    as[k * NT + t] = t < nt ? __ldcg(p.zsh + (size_t)(t0 + t) * Fs + k) : 0.f;
                }
                __syncthreads();
                for (int rr = warp; rr < 32; rr += blockDim.x >> 5) {
                    const int row = row0 + rr;
                    float a2[NT];
#pragma unroll
                    for (int t = 0; t < NT; ++t) a2[t] = 0.f;
                    row_dot<NT, true>(p.sd + (size_t)row * Fs, Fs, as, lane, a2);
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float v = warp_sum(a2[t]);
                        if (lane == 0 && t < nt) p.ypart[((size_t)G * T + t0 + t) * H + row] = v;
                    }
                }
            }
            __syncthreads();
        }
    }
    // the last part of this row tile to finish writes y
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
    for (int i = threadIdx.x; i < T * 32; i += blockDim.x) {
        const int t = i >> 5, row = row0 + (i & 31);
        float v = 0.f;
        for (int g = 0; g < G; ++g)
            if (__ldcg(p.r.ghit + g) > 0 && p.r.tghit[(size_t)t * G + g]) v += __ldcg(p.ypart + ((size_t)g * T + t) * H + row);
        v += __ldcg(p.ypart + ((size_t)G * T + t) * H + row);
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

// Warps per CTA of a row-tile GEMV over C columns: two 64-column groups per warp.
static int gemv_warps(int C) { return max(1, min(16, (C / 64 + 1) / 2)); }

template <int NT>
static cudaError_t run_gemv_path_nt(FwdParams p, cudaStream_t st, bool route_only) {
    auto red = [](int warps) { return (size_t)warps * 32 * NT * sizeof(float); };
    // 1. router (+ shared gate/up, top-k, buckets): one warp per router row / shared feature
    p.router_rows_per_warp = 1;
    p.n_router_ctas = (p.E + 7) / 8;
    p.do_shared = !route_only;
    p.do_buckets = !route_only;
    p.prefetch_l2 = !route_only;
    const int n_shared_ctas = route_only ? 0 : (p.Fs + 7) / 8;
    {
        const size_t sm = (size_t)p.H * NT * sizeof(float);
        cudaError_t e = p.router_bf16
            ? launch(k_router_shared<NT, true>, dim3(p.n_router_ctas + n_shared_ctas), 256, sm, st, p)
            : launch(k_router_shared<NT, false>, dim3(p.n_router_ctas + n_shared_ctas), 256, sm, st, p);
        if (e != cudaSuccess || route_only) return e;
    }
    const int max_unique = min(p.T * p.K, p.E);
    cudaError_t e;
    int w = gemv_warps(p.H);
    e = launch(k_dproj<NT>, dim3(p.L / 32, p.G), 32 * w, (size_t)p.H * NT * 4 + red(w), st, p);
    if (e != cudaSuccess) return e;
    w = gemv_warps(p.L);
    e = launch(k_expert_gateup<NT>, dim3(p.F / 32, max_unique), 32 * w, (size_t)p.L * NT * 4 + red(w), st, p);
    if (e != cudaSuccess) return e;
    w = gemv_warps(p.F);
    e = launch(k_expert_down<NT>, dim3(p.L / 32, max_unique), 32 * w, (size_t)p.F * NT * 4 + red(w), st, p);
    if (e != cudaSuccess) return e;
    w = max(gemv_warps(p.L), 8);
    e = launch(k_uproj<NT>, dim3(p.H / 32, p.G + 1), 32 * w, (size_t)max(p.L, p.Fs) * NT * 4 + red(w), st, p);
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
        if (fmt == LMOE_Q8_0 || fmt == LMOE_Q4_0) {
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
