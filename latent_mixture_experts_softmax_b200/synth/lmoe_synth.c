/*
 * Seeded synthetic inputs for the latent mixture-of-experts FFN block.
 *
 * This file only draws random numbers and packs them into the storage
 * formats the block reads (bf16, fp32, Q8_0, Q4_0, NVFP4).  It holds none of
 * the block's arithmetic: no decoding, no routing, no projection.  Both the
 * CUDA path and the fp64 test oracle consume the bytes written here.
 *
 * Random numbers: a counter-based SplitMix64 (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014; finaliser
 * constants as published by Vigna).  Element n of stream `key` is
 *     bits(key, n) = mix(key + (n + 1) * 0x9E3779B97F4A7C15)
 * and a normal deviate is drawn by the Box-Muller transform from the pair
 * (bits(key, 2j), bits(key, 2j + 1)), cosine branch for even elements and
 * sine branch for odd ones.  Any element can be regenerated on its own.
 *
 * Storage layouts written here (the block's kernels and the oracle each
 * decode them on their own):
 *   Q8_0 matrix [R rows, C cols], blocks of 32 along C:
 *       qs  int8  [C/32][R][32]     then   d fp16 [C/32][R]
 *   Q4_0 matrix [R, C]:
 *       qs  uint8 [C/32][R][16]  (byte j: low nibble = element j,
 *                                 high nibble = element j+16; value (q-8)*d)
 *       then d fp16 [C/32][R]
 *   NVFP4 matrix [R, C]:
 *       q   uint8 [C/32][R][16]  (byte i: low nibble = element 2i,
 *                                 high nibble = element 2i+1; E2M1 codes)
 *       s   uint8 [C/64][R][4]   (byte j: E4M3 scale of elements 16j..16j+15
 *                                 of the 64-wide column group)
 *   NVFP4 expert record (latent L, ffn F):
 *       gate.q [L/32][F][16] | up.q [L/32][F][16] | down.q [F/32][L][16] |
 *       gate.s [L/64][F][4]  | up.s [L/64][F][4]  | down.s [F/64][L][4]  |
 *       tail: fp32 ts_gate, ts_up, ts_down, uint32 0       (16 bytes)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t sm_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t lmoe_synth_bits(uint64_t key, uint64_t n) { return sm_mix(key + (n + 1) * GOLDEN); }

uint64_t lmoe_synth_key(uint64_t a, uint64_t b) { return sm_mix(a ^ sm_mix(b + GOLDEN)); }

double lmoe_synth_normal(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    double u1 = (double)((lmoe_synth_bits(key, 2 * j) >> 11) + 1) * 0x1.0p-53;  /* (0, 1] */
    double u2 = (double)(lmoe_synth_bits(key, 2 * j + 1) >> 11) * 0x1.0p-53;    /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(a) : r * cos(a);
}

double lmoe_synth_uniform(uint64_t key, uint64_t i) {
    return (double)(lmoe_synth_bits(key, i) >> 11) * 0x1.0p-53;
}

/* ---------------- rounding into storage formats ---------------- */

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static inline uint16_t f64_to_fp16_rne(double v) {
    _Float16 h = (_Float16)v;   /* single correctly rounded conversion */
    uint16_t u;
    memcpy(&u, &h, 2);
    return u;
}

static inline double fp16_value(uint16_t u) {
    _Float16 h;
    memcpy(&h, &u, 2);
    return (double)h;
}

/* E4M3 (fn variant: no infinities, 0x7F is NaN), round to nearest even,
 * saturating at 448.  v must be >= 0. */
static uint8_t e4m3_rne_nonneg(double v) {
    if (!(v > 0.0)) return 0;
    if (v >= 448.0) return 0x7E;
    int e;
    frexp(v, &e);         /* v = f * 2^e, f in [0.5, 1) */
    int ex = e - 1;       /* v in [2^ex, 2^(ex+1)) */
    if (ex < -6) {        /* subnormal: units of 2^-9 */
        double m = rint(ldexp(v, 9));
        return (uint8_t)m; /* m == 8 is the smallest normal, code 0x08 */
    }
    double m = rint((ldexp(v, -ex) - 1.0) * 8.0);
    if (m >= 8.0) { m = 0.0; ex += 1; }
    int code = ((ex + 7) << 3) | (int)m;
    if (code > 0x7E) code = 0x7E;
    return (uint8_t)code;
}

static double e4m3_value(uint8_t c) {
    int e = (c >> 3) & 15, m = c & 7;
    double v = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp(m / 8.0, -6);
    return (c & 0x80) ? -v : v;
}

/* E2M1 code of |v| (3 magnitude bits), nearest with ties to the even code,
 * saturating at 6. */
static uint8_t e2m1_rne_mag(double a) {
    static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    if (a >= 6.0) return 7;
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        double dc = fabs(a - grid[c]), db = fabs(a - grid[best]);
        if (dc < db || (dc == db && (c & 1) == 0)) best = c;
    }
    return (uint8_t)best;
}

/* ---------------- plain tensors ---------------- */

void lmoe_synth_bf16(uint64_t key, double sigma, uint16_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne((float)(sigma * lmoe_synth_normal(key, (uint64_t)i)));
}

void lmoe_synth_f64(uint64_t key, double sigma, double* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = sigma * lmoe_synth_normal(key, (uint64_t)i);
}

void lmoe_synth_f32(uint64_t key, double sigma, float* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(sigma * lmoe_synth_normal(key, (uint64_t)i));
}

/* expert_group[e] = floor(8 * u) style draw in [0, G) */
void lmoe_synth_groups_uniform(uint64_t key, int E, int G, uint8_t* out) {
    for (int e = 0; e < E; ++e) {
        int g = (int)(lmoe_synth_uniform(key, (uint64_t)e) * G);
        out[e] = (uint8_t)(g < G ? g : G - 1);
    }
}

/* ---------------- Q8_0 / Q4_0 matrices ----------------
 * Element (r, c) of a generated matrix is sigma * normal(key, r * C + c). */

static void q8_0_block(const double* w, int8_t* q, uint16_t* d) {
    double amax = 0.0;
    for (int j = 0; j < 32; ++j) if (fabs(w[j]) > amax) amax = fabs(w[j]);
    uint16_t dh = f64_to_fp16_rne(amax / 127.0);
    double dv = fp16_value(dh);
    for (int j = 0; j < 32; ++j) {
        double v = dv > 0.0 ? rint(w[j] / dv) : 0.0;
        if (v > 127.0) v = 127.0;
        if (v < -127.0) v = -127.0;
        q[j] = (int8_t)v;
    }
    *d = dh;
}

static void q4_0_block(const double* w, uint8_t* q, uint16_t* d) {
    double m = 0.0;
    for (int j = 0; j < 32; ++j) if (fabs(w[j]) > fabs(m)) m = w[j];
    uint16_t dh = f64_to_fp16_rne(m / -8.0);
    double dv = fp16_value(dh);
    uint8_t qv[32];
    for (int j = 0; j < 32; ++j) {
        double v = dv != 0.0 ? rint(w[j] / dv) + 8.0 : 8.0;
        if (v > 15.0) v = 15.0;
        if (v < 0.0) v = 0.0;
        qv[j] = (uint8_t)v;
    }
    for (int j = 0; j < 16; ++j) q[j] = (uint8_t)(qv[j] | (qv[j + 16] << 4));
    *d = dh;
}

/* fmt 8: Q8_0, fmt 4: Q4_0.  w == NULL draws the weights from `key`. */
static void qblock_matrix(int fmt, const double* wsrc, uint64_t key, double sigma, int R, int C, uint8_t* out) {
    const int nb = C / 32;
    const size_t qrow = fmt == 8 ? 32 : 16;
    uint8_t* qs = out;
    uint16_t* d = (uint16_t*)(out + (size_t)R * nb * qrow);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < R; ++r) {
        double w[32];
        for (int b = 0; b < nb; ++b) {
            for (int j = 0; j < 32; ++j) {
                size_t i = (size_t)r * C + (size_t)b * 32 + j;
                w[j] = wsrc ? wsrc[i] : sigma * lmoe_synth_normal(key, i);
            }
            uint8_t* q = qs + ((size_t)b * R + r) * qrow;
            uint16_t* dd = d + (size_t)b * R + r;
            if (fmt == 8) q8_0_block(w, (int8_t*)q, dd);
            else q4_0_block(w, q, dd);
        }
    }
}

void lmoe_synth_q8_0(uint64_t key, double sigma, int R, int C, uint8_t* out) {
    qblock_matrix(8, NULL, key, sigma, R, C, out);
}
void lmoe_synth_q4_0(uint64_t key, double sigma, int R, int C, uint8_t* out) {
    qblock_matrix(4, NULL, key, sigma, R, C, out);
}
/* Encode a given fp64 matrix [R, C] (row-major). */
void lmoe_synth_q8_0_encode(const double* w, int R, int C, uint8_t* out) {
    qblock_matrix(8, w, 0, 0.0, R, C, out);
}
void lmoe_synth_q4_0_encode(const double* w, int R, int C, uint8_t* out) {
    qblock_matrix(4, w, 0, 0.0, R, C, out);
}

/* ---------------- NVFP4 ----------------
 * One matrix [R, C] into (q, s) with the per-tensor scale
 *   ts = amax / (6 * 448),  s = E4M3(amax16 / 6 / ts),  q = E2M1(w / (s * ts)).
 * `w` is scratch of R*C doubles already filled with the weights. */
static float nvfp4_pack(const double* w, int R, int C, uint8_t* q, uint8_t* s) {
    double amax = 0.0;
    for (size_t i = 0; i < (size_t)R * C; ++i) if (fabs(w[i]) > amax) amax = fabs(w[i]);
    float ts = amax > 0.0 ? (float)(amax / (6.0 * 448.0)) : 1.0f;
    for (int r = 0; r < R; ++r) {
        for (int c16 = 0; c16 < C / 16; ++c16) {
            const double* wb = w + (size_t)r * C + (size_t)c16 * 16;
            double a16 = 0.0;
            for (int j = 0; j < 16; ++j) if (fabs(wb[j]) > a16) a16 = fabs(wb[j]);
            uint8_t sc = e4m3_rne_nonneg(a16 / 6.0 / (double)ts);
            double sv = e4m3_value(sc) * (double)ts;
            s[((size_t)(c16 / 4) * R + r) * 4 + (c16 % 4)] = sc;
            for (int j = 0; j < 16; ++j) {
                int c = c16 * 16 + j;
                uint8_t code = 0;
                if (sv > 0.0) {
                    code = e2m1_rne_mag(fabs(wb[j]) / sv);
                    if (wb[j] < 0.0 && code) code |= 8;
                }
                uint8_t* byte = q + ((size_t)(c / 32) * R + r) * 16 + (c % 32) / 2;
                if (c & 1) *byte = (uint8_t)((*byte & 0x0F) | (code << 4));
                else       *byte = (uint8_t)((*byte & 0xF0) | code);
            }
        }
    }
    return ts;
}

size_t lmoe_synth_nvfp4_record_bytes(int L, int F) {
    return (size_t)3 * L * F / 2 + (size_t)3 * L * F / 16 + 16;
}

/* E experts; expert e, matrix m (0 gate [F,L], 1 up [F,L], 2 down [L,F]):
 * element (r, c) = sigma * normal(key_em, r * C + c) with
 * key_em = lmoe_synth_key(lmoe_synth_key(key, e), m). */
void lmoe_synth_nvfp4_experts(uint64_t key, double sigma, int E, int L, int F, uint8_t* out) {
    const size_t rec = lmoe_synth_nvfp4_record_bytes(L, F);
    const size_t nq = (size_t)L * F / 2, ns = (size_t)L * F / 16;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)L * F);
#pragma omp for schedule(dynamic, 1)
        for (int e = 0; e < E; ++e) {
            uint8_t* r = out + rec * (size_t)e;
            memset(r, 0, rec);
            float ts[3];
            for (int m = 0; m < 3; ++m) {
                int R = m < 2 ? F : L, C = m < 2 ? L : F;
                uint64_t km = lmoe_synth_key(lmoe_synth_key(key, (uint64_t)e), (uint64_t)m);
                for (size_t i = 0; i < (size_t)R * C; ++i) w[i] = sigma * lmoe_synth_normal(km, i);
                ts[m] = nvfp4_pack(w, R, C, r + nq * m, r + 3 * nq + ns * m);
            }
            memcpy(r + 3 * nq + 3 * ns, ts, 12);
        }
        free(w);
    }
}

/* Encode an arbitrary fp64 matrix [R, C] (row-major) to the NVFP4 matrix
 * layout; returns the tensor scale.  Used by tests that need hand-built
 * weights (identity-like or structured matrices). */
float lmoe_synth_nvfp4_encode(const double* w, int R, int C, uint8_t* q, uint8_t* s) {
    memset(q, 0, (size_t)R * C / 2);
    return nvfp4_pack(w, R, C, q, s);
}

/* ---------------- Q3_K gate/up + IQ4_NL down expert records ----------------
 * The other expert build of the pages: Q3_K for gate and up, IQ4_NL for
 * down, 985,600 + 645,120 = 1,630,720 bytes per record at latent 1792 and
 * ffn 640 (1,164,800 at latent 1280).  The pages give the type names and the
 * byte totals, not the bit arrangement; the arrangement below is this
 * project's, with exactly those byte counts:
 *
 *   Q3_K matrix [R, C] (C a multiple of 256): 110 bytes per 256 weights of a
 *   row, stored as planes over 128-column halves h = c / 128:
 *     lo [C/128][R][32]  2-bit low code parts; 32-bit word w (0..7) of a row's
 *                        32 bytes covers elements 16w..16w+15, element
 *                        16w + 4i + b in byte b, bits 2i..2i+1
 *     hi [C/128][R][16]  high code bits; word v (0..3) covers elements
 *                        32v..32v+31, element 32v + 4i + b in byte b, bit i
 *     sc [C/128][R][6]   eight 6-bit sub-block scales (sub-block j = elements
 *                        16j..16j+15 of the half) at bits 6j..6j+5 of the
 *                        48-bit little-endian word
 *     d  [C/256][R]      fp16 super-block scale
 *     weight = d * (sc_j - 32) * (q - 4),  q = lo | hi << 2  in 0..7
 *   IQ4_NL matrix [R, C] (C a multiple of 32): 18 bytes per 32 weights:
 *     q  [C/32][R][16]   4-bit indices, byte j: element j (low nibble) and
 *                        element j + 16 (high nibble)
 *     d  [C/32][R]       fp16 block scale
 *     weight = d * level[q]; the 16 levels are not printed on the pages: here
 *     they are the standard normal quantiles at (i + 1/2) / 16, scaled so the
 *     outermost is 127 and rounded (the table below, from that definition)
 *   record: gate (Q3_K [F, L]) | up (Q3_K [F, L]) | down (IQ4_NL [L, F]).
 */
static const int kIq4Levels[16] = {-127, -90, -69, -53, -39, -27, -16, -5, 5, 16, 27, 39, 53, 69, 90, 127};

size_t lmoe_synth_q3k_bytes(int R, int C) { return (size_t)R * C / 256 * 110; }
size_t lmoe_synth_iq4nl_bytes(int R, int C) { return (size_t)R * C / 32 * 18; }
size_t lmoe_synth_q3k_record_bytes(int L, int F) {
    return 2 * lmoe_synth_q3k_bytes(F, L) + lmoe_synth_iq4nl_bytes(L, F);
}

/* Encode w [R, C] (row-major fp64) into the Q3_K planes at out. */
void lmoe_synth_q3k_encode(const double* w, int R, int C, uint8_t* out) {
    const size_t nh = (size_t)C / 128;
    uint8_t* lo = out;
    uint8_t* hi = lo + nh * R * 32;
    uint8_t* sc = hi + nh * R * 16;
    uint16_t* dd = (uint16_t*)(sc + nh * R * 6);
    memset(out, 0, lmoe_synth_q3k_bytes(R, C));
    for (int r = 0; r < R; ++r) {
        for (int sb = 0; sb < C / 256; ++sb) {
            const double* ws = w + (size_t)r * C + (size_t)sb * 256;
            /* sub-block scales: the signed element of largest magnitude maps to -4 */
            double s[16], smax = 0.0;
            for (int j = 0; j < 16; ++j) {
                double m = 0.0;
                for (int k = 0; k < 16; ++k) if (fabs(ws[16 * j + k]) > fabs(m)) m = ws[16 * j + k];
                s[j] = m / -4.0;
                if (fabs(s[j]) > smax) smax = fabs(s[j]);
            }
            uint16_t dh = f64_to_fp16_rne(smax / 31.0);
            double dv = fp16_value(dh);
            dd[(size_t)sb * R + r] = dh;
            for (int j = 0; j < 16; ++j) {
                double f = dv > 0.0 ? rint(s[j] / dv) : 0.0;
                if (f > 31.0) f = 31.0;
                if (f < -32.0) f = -32.0;
                const int scj = (int)f + 32;
                const double e = dv * f;
                const int h = (sb * 256 + 16 * j) / 128, jj = j % 8;
                uint8_t* scp = sc + ((size_t)h * R + r) * 6;
                /* 6 bits at bit 6*jj of the 48-bit little-endian word */
                for (int b = 0; b < 6; ++b) {
                    const int bit = 6 * jj + b;
                    if ((scj >> b) & 1) scp[bit / 8] |= (uint8_t)(1u << (bit % 8));
                }
                for (int k = 0; k < 16; ++k) {
                    const int c = sb * 256 + 16 * j + k, e128 = c % 128;
                    double qv = e != 0.0 ? rint(ws[16 * j + k] / e) + 4.0 : 4.0;
                    if (qv > 7.0) qv = 7.0;
                    if (qv < 0.0) qv = 0.0;
                    const int q = (int)qv;
                    /* low bits: word e128/16, i = (e128 % 16) / 4, byte b = e128 % 4 */
                    const int wlo = e128 / 16, ilo = (e128 % 16) / 4, blo = e128 % 4;
                    lo[((size_t)h * R + r) * 32 + 4 * wlo + blo] |= (uint8_t)((q & 3) << (2 * ilo));
                    const int whi = e128 / 32, ihi = (e128 % 32) / 4, bhi = e128 % 4;
                    if (q & 4) hi[((size_t)h * R + r) * 16 + 4 * whi + bhi] |= (uint8_t)(1u << ihi);
                }
            }
        }
    }
}

/* Encode w [R, C] into the IQ4_NL planes at out: d = amax / 127, index of
 * the nearest level (the lower one on a tie). */
void lmoe_synth_iq4nl_encode(const double* w, int R, int C, uint8_t* out) {
    uint8_t* qs = out;
    uint16_t* dd = (uint16_t*)(out + (size_t)R * C / 2);
    memset(out, 0, lmoe_synth_iq4nl_bytes(R, C));
    for (int r = 0; r < R; ++r) {
        for (int b = 0; b < C / 32; ++b) {
            const double* wb = w + (size_t)r * C + (size_t)b * 32;
            double amax = 0.0;
            for (int j = 0; j < 32; ++j) if (fabs(wb[j]) > amax) amax = fabs(wb[j]);
            uint16_t dh = f64_to_fp16_rne(amax / 127.0);
            double dv = fp16_value(dh);
            dd[(size_t)b * R + r] = dh;
            uint8_t* q = qs + ((size_t)b * R + r) * 16;
            for (int j = 0; j < 32; ++j) {
                int best = 0;
                if (dv > 0.0) {
                    const double t = wb[j] / dv;
                    for (int i = 1; i < 16; ++i)
                        if (fabs(t - kIq4Levels[i]) < fabs(t - kIq4Levels[best])) best = i;
                }
                if (j < 16) q[j] |= (uint8_t)best;
                else q[j - 16] |= (uint8_t)(best << 4);
            }
        }
    }
}

/* E experts in the Q3_K build; matrix m (0 gate [F, L], 1 up, 2 down [L, F]) of
 * expert e drawn as sigma * normal(key(key(key, e), m), r * C + c). */
void lmoe_synth_q3k_experts(uint64_t key, double sigma, int E, int L, int F, uint8_t* out) {
    const size_t rec = lmoe_synth_q3k_record_bytes(L, F);
    const size_t gb = lmoe_synth_q3k_bytes(F, L);
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)L * F);
#pragma omp for schedule(dynamic, 1)
        for (int e = 0; e < E; ++e) {
            uint8_t* r = out + rec * (size_t)e;
            for (int m = 0; m < 3; ++m) {
                int R = m < 2 ? F : L, C = m < 2 ? L : F;
                uint64_t km = lmoe_synth_key(lmoe_synth_key(key, (uint64_t)e), (uint64_t)m);
                for (size_t i = 0; i < (size_t)R * C; ++i) w[i] = sigma * lmoe_synth_normal(km, i);
                if (m < 2) lmoe_synth_q3k_encode(w, R, C, r + gb * m);
                else lmoe_synth_iq4nl_encode(w, R, C, r + 2 * gb);
            }
        }
        free(w);
    }
}
