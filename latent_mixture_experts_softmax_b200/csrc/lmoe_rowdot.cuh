// Row-at-a-time inner products for few tokens: staging of the block input
// (bf16, optionally RMS-normalised) as fp32 rows in shared memory, and one
// warp's dot products of a stored weight row (bf16 or fp32) with the staged
// rows.  Used by the router / shared-expert stage of the few-token path.
#pragma once

#include "lmoe_internal.cuh"

namespace lmoe {

// ---------------------------------------------------------------------------
// activation staging: xs[t * ld + k] = act(t0 + t, k) as fp32 for t < nt, 0
// beyond (token-major rows padded by 4 floats so lanes reading 8 consecutive
// columns of one row hit distinct bank pairs)
// ---------------------------------------------------------------------------

__host__ __device__ constexpr int xs_ld(int K) { return K + 4; }

// x rows are bf16 [T][H]; with gamma != nullptr the row is RMS-normalised:
// gamma[k] * x[k] / sqrt(mean(x^2) + eps).  Every load of the CTA is issued
// before any is used.  CTA 0 also writes the fp16 copy used by the D_g kernel.
template <int NT>
__device__ void stage_x(const FwdParams& p, int t0, int nt, float* xs, float* rs) {
    const int H = p.H, ld = xs_ld(H);
    const int nc = H / 8;                     // 16-byte chunks per row
    __shared__ float ssq[NT][32];
    float part[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) part[t] = 0.f;
    for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        uint4 v[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t)
            v[t] = t < nt ? __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)(t0 + t) * H) + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const uint32_t w4[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
            float f[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 q = bf16x2_to_f32x2(w4[j]);
                f[2 * j] = q.x;
                f[2 * j + 1] = q.y;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) part[t] = fmaf(f[j], f[j], part[t]);
            *reinterpret_cast<float4*>(xs + t * ld + 8 * c) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4*>(xs + t * ld + 8 * c + 4) = make_float4(f[4], f[5], f[6], f[7]);
        }
    }
    if (p.gamma != nullptr) {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float v = warp_sum(part[t]);
            if (lane == 0) ssq[t][warp] = v;
        }
        __syncthreads();
        if (threadIdx.x < NT) {
            float tot = 0.f;
            for (int w = 0; w < nw; ++w) tot += ssq[threadIdx.x][w];
            rs[threadIdx.x] = rsqrtf(tot / (float)H + p.eps);
        }
        __syncthreads();
        for (int c = threadIdx.x; c < nc; c += blockDim.x) {
            const uint4 gv = __ldg(reinterpret_cast<const uint4*>(p.gamma) + c);
            const uint32_t g4[4] = {gv.x, gv.y, gv.z, gv.w};
            float gf[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 q = bf16x2_to_f32x2(g4[j]);
                gf[2 * j] = q.x;
                gf[2 * j + 1] = q.y;
            }
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int j = 0; j < 8; ++j) xs[t * ld + 8 * c + j] *= rs[t] * gf[j];
        }
    }
    if (blockIdx.x == 0 && p.x16) {
        __syncthreads();
        bool bad = false;
        for (int i = threadIdx.x; i < nt * nc; i += blockDim.x) {
            const int t = i / nc, c = i - t * nc;
            const float* src = xs + t * ld + 8 * c;
            __half2 h[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) h[j] = half2_checked(src[2 * j], src[2 * j + 1], bad);
            *reinterpret_cast<uint4*>(p.x16 + (size_t)(t0 + t) * H + 8 * c) = *reinterpret_cast<uint4*>(h);
        }
        report_range(p.ctrl, bad);
    }
}

// ---------------------------------------------------------------------------
// inner products of one stored row segment with NT staged activations
// ---------------------------------------------------------------------------

// 8 bf16 weights (one 16-byte load) against xs[t * ld + k0 + j].
template <int NT>
__device__ __forceinline__ void dot8_bf16(uint4 wv, const float* xs, int ld, int k0, float (&acc)[NT]) {
    const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
    float w[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 q = bf16x2_to_f32x2(w4[j]);
        w[2 * j] = q.x;
        w[2 * j + 1] = q.y;
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const float4 a = *reinterpret_cast<const float4*>(xs + t * ld + k0);
        const float4 b = *reinterpret_cast<const float4*>(xs + t * ld + k0 + 4);
        acc[t] = fmaf(w[0], a.x, acc[t]);
        acc[t] = fmaf(w[1], a.y, acc[t]);
        acc[t] = fmaf(w[2], a.z, acc[t]);
        acc[t] = fmaf(w[3], a.w, acc[t]);
        acc[t] = fmaf(w[4], b.x, acc[t]);
        acc[t] = fmaf(w[5], b.y, acc[t]);
        acc[t] = fmaf(w[6], b.z, acc[t]);
        acc[t] = fmaf(w[7], b.w, acc[t]);
    }
}

// 4 fp32 weights against xs.
template <int NT>
__device__ __forceinline__ void dot4_f32(float4 w, const float* xs, int ld, int k0, float (&acc)[NT]) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const float4 a = *reinterpret_cast<const float4*>(xs + t * ld + k0);
        acc[t] = fmaf(w.x, a.x, acc[t]);
        acc[t] = fmaf(w.y, a.y, acc[t]);
        acc[t] = fmaf(w.z, a.z, acc[t]);
        acc[t] = fmaf(w.w, a.w, acc[t]);
    }
}

// One row of a plain bf16 / fp32 matrix (K contiguous) against xs, the warp's
// lanes splitting K; ten 16-byte loads per lane are issued before any
// arithmetic.  The per-lane partial sums are left in acc (reduce with warp_sum).
template <int NT, bool kBF16, int kB = 10>
__device__ __forceinline__ void row_dot(const void* wrow, int K, const float* xs, int ld, int lane, float (&acc)[NT]) {
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
                if (kBF16) dot8_bf16<NT>(w[i], xs, ld, k0, acc);
                else dot4_f32<NT>(make_float4(__uint_as_float(w[i].x), __uint_as_float(w[i].y), __uint_as_float(w[i].z),
                                              __uint_as_float(w[i].w)), xs, ld, k0, acc);
            }
        }
    }
}

// Two rows of plain bf16 matrices (K contiguous) against xs, as row_dot:
// both rows' loads are issued before any arithmetic.
template <int NT, int kB = 10>
__device__ __forceinline__ void row_dot2_bf16(const uint16_t* ra, const uint16_t* rb, int K, const float* xs, int ld,
                                              int lane, float (&acc_a)[NT], float (&acc_b)[NT]) {
    constexpr int kStep = 32 * 8;
    for (int base = 0; base < K; base += kB * kStep) {
        uint4 wa[kB], wb[kB];
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            const int k0 = base + i * kStep + lane * 8;
            if (k0 < K) {
                wa[i] = ldg_stream(reinterpret_cast<const uint4*>(ra + k0));
                wb[i] = ldg_stream(reinterpret_cast<const uint4*>(rb + k0));
            }
        }
#pragma unroll
        for (int i = 0; i < kB; ++i) {
            const int k0 = base + i * kStep + lane * 8;
            if (k0 < K) {
                dot8_bf16<NT>(wa[i], xs, ld, k0, acc_a);
                dot8_bf16<NT>(wb[i], xs, ld, k0, acc_b);
            }
        }
    }
}

}  // namespace lmoe
