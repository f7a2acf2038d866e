// Ablation of D_g: the design of the reference kernel printed in the
// teardown article (section "A latent in front of the experts", its code
// excerpt: every token row quantised to Q8_1, then D over all 8 groups as
// integer dot products) against this library's (fp16 activations, only the
// groups the batch hits).  Both run the same weight-streaming structure so
// that the activation format and the group set are the only differences:
//
//   k_quantize_q8_1    x bf16 [T][H] -> int8 q [T][H], fp32 d and block sums
//                      [T][H/32]   (d = fp16(amax / 127), q = rint(x / d))
//   k_dproj_ablation   h fp32 [T][G][L] = D_g x for the groups in a mask;
//                      one CTA per SM, work items of 16 rows of one group,
//                      8 warps splitting the reduction; Q8_1 activations on
//                      mma.sync m16n8k32 (s8 x s8, or u8 x s8 with the -8
//                      offset of Q4_0 taken out through the block sums), or
//                      fp16 activations on mma.sync m16n8k16

#include <algorithm>

#include "lmoe_internal.cuh"

namespace lmoe {

namespace {

constexpr int kAblWarps = 8;
constexpr int kAblThreads = 32 * kAblWarps;

struct AblParams {
    const uint16_t* x;    // bf16 [T][H]
    const uint8_t* D;     // G matrices [L][H]
    int T, H, L, G, fmt;
    uint32_t gmask;       // groups to project (bit g)
    size_t du_bytes;
    int8_t* q;            // Q8_1 codes [T][H]
    float* dq;            // Q8_1 scales [T][H/32]
    int* sq;              // Q8_1 block sums [T][H/32]
    float* h;             // [T][G][L]
};

__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t hsub2w(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// Q8_1 of one 32-element block per thread (every rounding an fp32 operation).
__global__ void k_quantize_q8_1(AblParams a) {
    const int nb = a.H / 32;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.T * nb) return;
    const int t = i / nb, b = i - t * nb;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H + b * 32);
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 w = __ldg(src + c);
        const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = bf16x2_to_f32x2(w4[j]);
            v[8 * c + 2 * j] = f.x;
            v[8 * c + 2 * j + 1] = f.y;
        }
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const float d = __half2float(__float2half_rn(__fdiv_rn(amax, 127.0f)));
    int sum = 0;
    int8_t q[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        float r = d > 0.f ? rintf(__fdiv_rn(v[j], d)) : 0.f;
        r = fminf(127.f, fmaxf(-127.f, r));
        q[j] = (int8_t)r;
        sum += (int)r;
    }
    int4* dst = reinterpret_cast<int4*>(a.q + (size_t)t * a.H + b * 32);
    dst[0] = *reinterpret_cast<int4*>(q);
    dst[1] = *reinterpret_cast<int4*>(q + 16);
    a.dq[i] = d;
    a.sq[i] = sum;
}

template <int FMT, bool kQ81>
__global__ void __launch_bounds__(kAblThreads, 1) k_dproj_ablation(AblParams a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int H = a.H, L = a.L, nb = H / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g8 = lane >> 2, t4 = lane & 3;
    // activations of up to 8 tokens, row stride padded against bank conflicts
    const int ldq = H + 16, ldh = H + 32;
    int8_t* xq = reinterpret_cast<int8_t*>(smem);                          // [8][ldq]   (Q8_1)
    float* xd = reinterpret_cast<float*>(smem + 8 * ldq);                   // [8][nb]
    int* xs = reinterpret_cast<int*>(xd + 8 * nb);                          // [8][nb]
    __half* xh = reinterpret_cast<__half*>(smem);                           // [8][ldh]   (fp16)
    float* red = reinterpret_cast<float*>(smem + (kQ81 ? (size_t)8 * ldq + 64 * nb : (size_t)16 * ldh));
    const int n_items = a.G * (L / 16);
    const int per = (nb + kAblWarps - 1) / kAblWarps;
    const int kb0 = warp * per, kb1 = min(nb, kb0 + per);
    for (int t0 = 0; t0 < a.T; t0 += 8) {
        const int nt = min(8, a.T - t0);
        __syncthreads();
        if (kQ81) {
            for (int i = threadIdx.x; i < 8 * (H / 16); i += blockDim.x) {
                const int t = i / (H / 16), c = i - t * (H / 16);
                const int4 v = t < nt ? __ldcg(reinterpret_cast<const int4*>(a.q + (size_t)(t0 + t) * H) + c)
                                      : make_int4(0, 0, 0, 0);
                *reinterpret_cast<int4*>(xq + (size_t)t * ldq + 16 * c) = v;
            }
            for (int i = threadIdx.x; i < 8 * nb; i += blockDim.x) {
                const int t = i / nb, b = i - t * nb;
                xd[i] = t < nt ? __ldcg(a.dq + (size_t)(t0 + t) * nb + b) : 0.f;
                xs[i] = t < nt ? __ldcg(a.sq + (size_t)(t0 + t) * nb + b) : 0;
            }
        } else {
            for (int i = threadIdx.x; i < 8 * (H / 8); i += blockDim.x) {
                const int t = i / (H / 8), c = i - t * (H / 8);
                uint4 v = make_uint4(0, 0, 0, 0);
                if (t < nt) {
                    const uint4 w = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)(t0 + t) * H) + c);
                    const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
                    uint32_t o[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = bf16x2_to_f32x2(w4[j]);
                        __half2 hv = __floats2half2_rn(f.x, f.y);
                        o[j] = *reinterpret_cast<uint32_t*>(&hv);
                    }
                    v = make_uint4(o[0], o[1], o[2], o[3]);
                }
                *reinterpret_cast<uint4*>(xh + (size_t)t * ldh + 8 * c) = v;
            }
        }
        __syncthreads();
        for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
            const int g = item / (L / 16), r0 = (item - g * (L / 16)) * 16;
            if (!((a.gmask >> g) & 1u)) continue;
            const uint8_t* mat = a.D + (size_t)g * a.du_bytes;
            const size_t qrow = FMT == LMOE_Q8_0 ? 32 : 16;
            const uint16_t* dsc = reinterpret_cast<const uint16_t*>(mat + (size_t)L * H / 32 * qrow);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            constexpr int kU = 4;
            for (int kb = kb0; kb < kb1; kb += kU) {
                uint2 wg[kU], wh[kU];
                uint16_t dg[kU], dh[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (kb + u < kb1) {
                        const size_t b = (size_t)(kb + u);
                        // lane t4 takes elements 8 t4 .. 8 t4 + 7 (Q8_0) or the
                        // nibbles of bytes 8 (t4 & 1) .. + 7 (Q4_0: low t4 < 2)
                        const size_t off = FMT == LMOE_Q8_0 ? 8 * t4 : 8 * (t4 & 1);
                        wg[u] = __ldg(reinterpret_cast<const uint2*>(mat + (b * L + r0 + g8) * qrow + off));
                        wh[u] = __ldg(reinterpret_cast<const uint2*>(mat + (b * L + r0 + g8 + 8) * qrow + off));
                        dg[u] = __ldg(dsc + b * L + r0 + g8);
                        dh[u] = __ldg(dsc + b * L + r0 + g8 + 8);
                    }
                }
#pragma unroll
                for (int u = 0; u < kU; ++u) {
                    if (kb + u >= kb1) continue;
                    const int b = kb + u;
                    const float fdg = __half2float(__ushort_as_half(dg[u])), fdh = __half2float(__ushort_as_half(dh[u]));
                    if (kQ81) {
                        // A: the lane's 8 weights of rows g8 and g8 + 8; B: the
                        // same 8 positions of token g8's codes (both permuted alike)
                        uint32_t a0 = wg[u].x, a1 = wh[u].x, a2 = wg[u].y, a3 = wh[u].y;
                        const int pos = FMT == LMOE_Q8_0 ? 8 * t4 : (t4 < 2 ? 8 * t4 : 16 + 8 * (t4 - 2));
                        if (FMT == LMOE_Q4_0) {
                            const int sh = t4 < 2 ? 0 : 4;
                            a0 = (a0 >> sh) & 0x0F0F0F0Fu;
                            a1 = (a1 >> sh) & 0x0F0F0F0Fu;
                            a2 = (a2 >> sh) & 0x0F0F0F0Fu;
                            a3 = (a3 >> sh) & 0x0F0F0F0Fu;
                        }
                        const uint2 bx = *reinterpret_cast<const uint2*>(xq + (size_t)g8 * ldq + 32 * b + pos);
                        int c[4] = {0, 0, 0, 0};
                        if (FMT == LMOE_Q8_0) mma_s8(c, a0, a1, a2, a3, bx.x, bx.y);
                        else mma_u8s8(c, a0, a1, a2, a3, bx.x, bx.y);
                        // token columns 2 t4, 2 t4 + 1
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int col = 2 * t4 + (i & 1);
                            int v = c[i];
                            if (FMT == LMOE_Q4_0) v -= 8 * xs[col * nb + b];
                            acc[i] = fmaf((i < 2 ? fdg : fdh) * xd[col * nb + b], (float)v, acc[i]);
                        }
                    } else {
                        float c[4] = {0.f, 0.f, 0.f, 0.f};
                        const __half* xr = xh + (size_t)g8 * ldh + 32 * b;
                        if (FMT == LMOE_Q8_0) {
                            // lane t4: elements 8 t4 .. 8 t4 + 7 of rows g8, g8 + 8
                            auto cv = [](uint32_t w, uint32_t& lo, uint32_t& hi) {
                                const uint32_t u8 = w ^ 0x80808080u;
                                lo = hsub2w(__byte_perm(u8, 0x64646464u, 0x4140), 0x64806480u);
                                hi = hsub2w(__byte_perm(u8, 0x64646464u, 0x4342), 0x64806480u);
                            };
                            uint32_t ga0, ga1, ga2, ga3, ha0, ha1, ha2, ha3;
                            cv(wg[u].x, ga0, ga1);
                            cv(wg[u].y, ga2, ga3);
                            cv(wh[u].x, ha0, ha1);
                            cv(wh[u].y, ha2, ha3);
                            const uint4 xv = *reinterpret_cast<const uint4*>(xr + 8 * t4);
                            mma_f16(c, ga0, ha0, ga1, ha1, xv.x, xv.y);
                            mma_f16(c, ga2, ha2, ga3, ha3, xv.z, xv.w);
                        } else {
                            // lane t4: the nibbles of bytes 8 (t4 & 1) .. + 7, low
                            // (elements 8 (t4 & 1) + j) or high (16 + ...)
                            const int sh = t4 < 2 ? 0 : 4;
                            auto cv = [sh](uint32_t w, uint32_t& lo, uint32_t& hi) {
                                const uint32_t n = (w >> sh) & 0x0F0F0F0Fu;
                                lo = hsub2w(__byte_perm(n, 0x64646464u, 0x4140), 0x64086408u);
                                hi = hsub2w(__byte_perm(n, 0x64646464u, 0x4342), 0x64086408u);
                            };
                            uint32_t ga0, ga1, ga2, ga3, ha0, ha1, ha2, ha3;
                            cv(wg[u].x, ga0, ga1);
                            cv(wg[u].y, ga2, ga3);
                            cv(wh[u].x, ha0, ha1);
                            cv(wh[u].y, ha2, ha3);
                            const int pos = t4 < 2 ? 8 * t4 : 16 + 8 * (t4 - 2);
                            const uint4 xv = *reinterpret_cast<const uint4*>(xr + pos);
                            mma_f16(c, ga0, ha0, ga1, ha1, xv.x, xv.y);
                            mma_f16(c, ga2, ha2, ga3, ha3, xv.z, xv.w);
                        }
                        acc[0] = fmaf(fdg, c[0], acc[0]);
                        acc[1] = fmaf(fdg, c[1], acc[1]);
                        acc[2] = fmaf(fdh, c[2], acc[2]);
                        acc[3] = fmaf(fdh, c[3], acc[3]);
                    }
                }
            }
            // the warps' partial sums of the item, added in warp order
#pragma unroll
            for (int i = 0; i < 4; ++i) red[(warp * 32 + lane) * 4 + i] = acc[i];
            __syncthreads();
            if (warp == 0) {
                for (int w = 1; w < kAblWarps; ++w)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i] += red[(w * 32 + lane) * 4 + i];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int col = 2 * t4 + (i & 1), row = r0 + g8 + 8 * (i >> 1);
                    if (col < nt) a.h[((size_t)(t0 + col) * a.G + g) * L + row] = acc[i];
                }
            }
            __syncthreads();
        }
    }
}

}  // namespace

size_t dproj_ablation_ws_bytes(int T, int H) {
    return (size_t)T * H + 2 * (size_t)T * (H / 32) * 4 + 256;
}

cudaError_t run_dproj_ablation(const uint16_t* x, const uint8_t* D, int T, int H, int L, int G, int fmt, int q81,
                               uint32_t gmask, size_t du_bytes, float* h, void* ws, cudaStream_t st) {
    AblParams a;
    a.x = x;
    a.D = D;
    a.T = T;
    a.H = H;
    a.L = L;
    a.G = G;
    a.fmt = fmt;
    a.gmask = gmask;
    a.du_bytes = du_bytes;
    char* b = static_cast<char*>(ws);
    a.q = reinterpret_cast<int8_t*>(b);
    a.dq = reinterpret_cast<float*>(b + (((size_t)T * H + 15) & ~(size_t)15));
    a.sq = reinterpret_cast<int*>(a.dq + (size_t)T * (H / 32));
    a.h = h;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int nb = H / 32;
    const size_t red = (size_t)kAblWarps * 32 * 4 * sizeof(float);
    size_t smem;
    cudaError_t e;
    if (q81) {
        const int n = T * nb;
        k_quantize_q8_1<<<(n + 127) / 128, 128, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        smem = (size_t)8 * (H + 16) + (size_t)64 * nb + red;
    } else {
        smem = (size_t)16 * (H + 32) + red;
    }
    const void* k = q81 ? (fmt == LMOE_Q8_0 ? reinterpret_cast<const void*>(k_dproj_ablation<LMOE_Q8_0, true>)
                                             : reinterpret_cast<const void*>(k_dproj_ablation<LMOE_Q4_0, true>))
                        : (fmt == LMOE_Q8_0 ? reinterpret_cast<const void*>(k_dproj_ablation<LMOE_Q8_0, false>)
                                             : reinterpret_cast<const void*>(k_dproj_ablation<LMOE_Q4_0, false>));
    if ((e = ensure_smem(k, smem)) != cudaSuccess) return e;
    const int grid = std::min(sms, G * (L / 16));
    if (q81) {
        if (fmt == LMOE_Q8_0) k_dproj_ablation<LMOE_Q8_0, true><<<grid, kAblThreads, smem, st>>>(a);
        else k_dproj_ablation<LMOE_Q4_0, true><<<grid, kAblThreads, smem, st>>>(a);
    } else {
        if (fmt == LMOE_Q8_0) k_dproj_ablation<LMOE_Q8_0, false><<<grid, kAblThreads, smem, st>>>(a);
        else k_dproj_ablation<LMOE_Q4_0, false><<<grid, kAblThreads, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace lmoe
