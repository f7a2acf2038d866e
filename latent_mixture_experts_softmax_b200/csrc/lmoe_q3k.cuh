// Device decoders of the other expert build: Q3_K gate/up and IQ4_NL down
// (model page, "Model profile"; teardown article, "What is 4-bit":
// 985,600 + 645,120 = 1,630,720 bytes per record at latent 1792).  The
// pages give the type names and byte counts; the arrangement, documented in
// include/lmoe.h, is this library's:
//   Q3_K [R][C], 110 bytes per 256 weights of a row, planes over 128-column
//   halves h:  lo [C/128][R][32]: element 16w + 4i + b of the half in byte
//   4w + b, bits 2i..2i+1;  hi [C/128][R][16]: element 32v + 4i + b in byte
//   4v + b, bit i;  sc [C/128][R][6]: sub-block j (elements 16j..16j+15) at
//   bits 6j..6j+5, little-endian;  d fp16 [C/256][R];
//   w = d * (sc_j - 32) * (q - 4), q = lo | hi << 2
//   IQ4_NL [R][C], 18 bytes per 32: codes [C/32][R][16] (byte j: element j
//   low nibble, j + 16 high), d fp16 [C/32][R];  w = d * level[code]
// The IQ4_NL levels are the standard normal quantiles at (i + 1/2) / 16,
// scaled so that the outermost is 127 and rounded to integers.
#pragma once

#include "lmoe_internal.cuh"

namespace lmoe {

__host__ __device__ constexpr size_t q3k_matrix_bytes(int R, int C) { return (size_t)R * C / 256 * 110; }
__host__ __device__ constexpr size_t iq4nl_matrix_bytes(int R, int C) { return (size_t)R * C / 32 * 18; }

// the 16 IQ4_NL levels (definition in the header comment)
__device__ __forceinline__ int iq4nl_level(int i) {
    constexpr int kLevels[16] = {-127, -90, -69, -53, -39, -27, -16, -5, 5, 16, 27, 39, 53, 69, 90, 127};
    return kLevels[i & 15];
}

// One element of a Q3_K matrix (diagnostics; the streaming kernels decode
// whole tiles).
__device__ __forceinline__ float q3k_element(const uint8_t* m, int R, int C, int r, int c) {
    const size_t nh = (size_t)C / 128;
    const uint8_t* lo = m;
    const uint8_t* hi = lo + nh * R * 32;
    const uint8_t* sc = hi + nh * R * 16;
    const uint16_t* d = reinterpret_cast<const uint16_t*>(sc + nh * R * 6);
    const int h = c / 128, e = c % 128;
    const int q_lo = (lo[((size_t)h * R + r) * 32 + 4 * (e / 16) + e % 4] >> (2 * ((e % 16) / 4))) & 3;
    const int q_hi = (hi[((size_t)h * R + r) * 16 + 4 * (e / 32) + e % 4] >> ((e % 32) / 4)) & 1;
    const int j = e / 16;
    const uint8_t* sp = sc + ((size_t)h * R + r) * 6;
    int scj = 0;
    for (int b = 0; b < 6; ++b) scj |= ((sp[(6 * j + b) / 8] >> ((6 * j + b) % 8)) & 1) << b;
    return __half2float(__ushort_as_half(d[(size_t)(c / 256) * R + r])) * (float)((scj - 32) * ((q_lo | (q_hi << 2)) - 4));
}

__device__ __forceinline__ float iq4nl_element(const uint8_t* m, int R, int C, int r, int c) {
    const size_t blk = (size_t)(c / 32) * R + r;
    const int j = c % 32;
    const uint8_t byte = m[blk * 16 + (j % 16)];
    const int q = j < 16 ? (byte & 0xF) : (byte >> 4);
    const uint16_t d = reinterpret_cast<const uint16_t*>(m + (size_t)R * C / 2)[blk];
    return __half2float(__ushort_as_half(d)) * (float)iq4nl_level(q);
}

// The shared-memory lookup table of the IQ4_NL decode: lut[b] = (level of
// b's low nibble, level of its high nibble) as fp16 (exact integers).
__device__ __forceinline__ void iq4nl_fill_lut(uint32_t* lut) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) {
        __half2 v = __halves2half2(__int2half_rn(iq4nl_level(b & 15)), __int2half_rn(iq4nl_level(b >> 4)));
        lut[b] = *reinterpret_cast<uint32_t*>(&v);
    }
}

}  // namespace lmoe
