// fp64 CPU oracle of the latent mixture-of-experts FFN block, in plain C++.
//
// TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
// CPU-baseline legs of the benchmark may load this library.  It shares no
// code with the CUDA path: every storage format is decoded here from its
// definition, element by element, and every step of the block follows the
// method in the order the pages give it.  Loops are plain; OpenMP only
// spreads independent rows, tokens or experts over the host cores (each
// result is still one sequential sum in its natural order), so the output
// does not depend on the thread count.
//
// What the block computes (teardown article "Edge0-145B: a Qwen MoE with its
// experts squeezed, and a 51B table left on the SSD", section "A latent in
// front of the experts", layer equation; the Edge0 145B / 120B model page,
// "Model profile" and the architecture tables), per token x of width H:
//
//   1. router   l_e = W_r[e] . x + b_e for all E experts; the experts are
//               ordered by (l descending, index ascending) and the first K
//               kept; p = softmax(l) over all E; w_k = p_k / sum of kept p
//               (the routing function is not printed on the pages; it is
//               the one the task's workload statement gives)
//   2. groups   every expert e carries a label group[e]; the token's hit
//               groups are the labels of its K experts
//   3. D        h_g = D_g x for every hit group g
//   4. experts  o_k = W_down (silu(W_gate h) * (W_up h)),  h = h_{group[e_k]}
//   5. combine  s_g = sum over k with group[e_k] = g of w_k o_k
//   6. U        y = sum over hit g (ascending) of U_g s_g
//   7. shared   y += S_down (silu(S_gate x) * (S_up x))   (full width, no gate)
//   8. residual y += residual (optional)
//   stack layer: x + block(RMSNorm(x)), RMSNorm(v) = gamma v / sqrt(mean v^2 + eps)
//
// Storage formats (the model page, "Model profile": D and U in Q8 or Q4; the teardown
// article, "What is 4-bit": NVFP4 = E2M1 values with one E4M3 scale per 16,
// a 16-byte record tail):
//   Q8_0 [R][C]:  int8 q [C/32][R][32], then fp16 d [C/32][R]; w = d q
//   Q4_0 [R][C]:  uint8 [C/32][R][16] (byte j: low nibble element j, high
//                 nibble element j + 16), then fp16 d [C/32][R]; w = d (q - 8)
//   NVFP4 [R][C]: uint8 q [C/32][R][16] (byte i: low nibble element 2i, high
//                 nibble element 2i + 1), E4M3 scales [C/64][R][4] (byte j of
//                 a word: elements 16j..16j+15 of its 64 columns);
//                 w = e2m1(code) * e4m3(scale) * ts (fp32 tensor scale)
//   expert record: gate.q | up.q | down.q | gate.s | up.s | down.s |
//                  fp32 ts_gate, ts_up, ts_down, 4 zero bytes
//
// Build: g++ -O2 -fopenmp -shared -fPIC (no fast-math: IEEE fp64 throughout).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#include <omp.h>

namespace {

// ---------------------------------------------------------------------------
// scalar formats
// ---------------------------------------------------------------------------

// bfloat16: the high 16 bits of an IEEE binary32.
double bf16_value(uint16_t b) {
    const uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return (double)f;
}

// IEEE binary16: sign, 5-bit exponent (bias 15), 10-bit fraction.
double fp16_value(uint16_t h) {
    const int s = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double mag;
    if (e == 0) mag = std::ldexp((double)f, -24);
    else if (e == 31) mag = f == 0 ? std::numeric_limits<double>::infinity() : std::numeric_limits<double>::quiet_NaN();
    else mag = std::ldexp(1.0 + f / 1024.0, e - 15);
    return s ? -mag : mag;
}

// FP4 E2M1 (OCP Microscaling formats): sign, 2-bit exponent (bias 1),
// 1-bit mantissa; exponent 0 is subnormal (m * 0.5).  Magnitudes 0, 0.5, 1,
// 1.5, 2, 3, 4, 6.
double e2m1_value(int code) {
    const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

// FP8 E4M3, "fn" variant (no infinities; S.1111.111 is NaN): sign, 4-bit
// exponent (bias 7), 3-bit mantissa; exponent 0 is subnormal (m/8 * 2^-6).
double e4m3fn_value(int code) {
    const int s = (code >> 7) & 1, e = (code >> 3) & 0xF, m = code & 7;
    if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
    const double mag = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

uint16_t load_u16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

float load_f32(const uint8_t* p) {
    float f;
    std::memcpy(&f, p, 4);
    return f;
}

// ---------------------------------------------------------------------------
// matrix formats: one element (r, c) of a stored matrix [R][C]
// ---------------------------------------------------------------------------

constexpr int kQ8_0 = 8;
constexpr int kQ4_0 = 4;

int64_t du_matrix_bytes(int fmt, int R, int C) { return (int64_t)R * C / 32 * (fmt == kQ8_0 ? 34 : 18); }

int64_t nvfp4_matrix_bytes(int R, int C) { return (int64_t)R * C / 2 + (int64_t)R * C / 16; }

int64_t expert_record_bytes(int L, int F) { return 3 * nvfp4_matrix_bytes(F, L) + 16; }

double q8_0_weight(const uint8_t* m, int R, int C, int r, int c) {
    const int64_t blk = (int64_t)(c / 32) * R + r;
    const int8_t q = (int8_t)m[blk * 32 + c % 32];
    const double d = fp16_value(load_u16(m + (int64_t)R * C + 2 * blk));
    return d * q;
}

double q4_0_weight(const uint8_t* m, int R, int C, int r, int c) {
    const int64_t blk = (int64_t)(c / 32) * R + r;
    const int j = c % 32;
    const uint8_t byte = m[blk * 16 + (j % 16)];
    const int q = j < 16 ? (byte & 0xF) : (byte >> 4);
    const double d = fp16_value(load_u16(m + (int64_t)R * C / 2 + 2 * blk));
    return d * (q - 8);
}

double du_weight(int fmt, const uint8_t* m, int R, int C, int r, int c) {
    return fmt == kQ8_0 ? q8_0_weight(m, R, C, r, c) : q4_0_weight(m, R, C, r, c);
}

double nvfp4_weight(const uint8_t* q, const uint8_t* s, double ts, int R, int r, int c) {
    const uint8_t byte = q[((int64_t)(c / 32) * R + r) * 16 + (c % 32) / 2];
    const int code = (c % 2) ? (byte >> 4) : (byte & 0xF);
    const int scode = s[((int64_t)(c / 64) * R + r) * 4 + (c % 64) / 16];
    return e2m1_value(code) * e4m3fn_value(scode) * ts;
}

// The other expert build (model page, "Model profile": Q3_K gate/up and
// IQ4_NL down; teardown article, "What is 4-bit": 985,600 + 645,120 bytes is
// the 1,630,720-byte record).  The pages give the type names and byte counts
// only; the block arrangement is this project's (documented with the C ABI):
//   Q3_K [R][C], 110 bytes per 256 weights of a row, planes over 128-column
//   halves h: lo [C/128][R][32] (element 16w + 4i + b: byte 4w + b, bits
//   2i..2i+1), hi [C/128][R][16] (element 32v + 4i + b: byte 4v + b, bit i),
//   sc [C/128][R][6] (sub-block j of the half: bits 6j..6j+5, little-endian),
//   d fp16 [C/256][R];  w = d * (sc_j - 32) * (q - 4), q = lo | hi << 2
//   IQ4_NL [R][C], 18 bytes per 32: q [C/32][R][16] (as Q4_0), d fp16
//   [C/32][R];  w = d * level[q]
// The 16 IQ4_NL levels are not printed on the pages; they are read here as
// the standard normal quantiles at (i + 1/2) / 16, scaled so that the
// outermost is 127, rounded to integers (computed below from that definition).
double normal_quantile(double p) {
    double lo = -10.0, hi = 10.0;       // Phi(x) = erfc(-x / sqrt 2) / 2, by bisection
    for (int it = 0; it < 200; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p) lo = mid;
        else hi = mid;
    }
    return 0.5 * (lo + hi);
}

const double* iq4nl_levels() {
    static double levels[16];
    static bool done = false;
    if (!done) {
        const double top = normal_quantile(15.5 / 16.0);
        for (int i = 0; i < 16; ++i) levels[i] = std::nearbyint(127.0 * normal_quantile((i + 0.5) / 16.0) / top);
        done = true;
    }
    return levels;
}

int64_t q3k_matrix_bytes(int R, int C) { return (int64_t)R * C / 256 * 110; }
int64_t iq4nl_matrix_bytes(int R, int C) { return (int64_t)R * C / 32 * 18; }

double q3k_weight(const uint8_t* m, int R, int C, int r, int c) {
    const int64_t nh = C / 128;
    const uint8_t* lo = m;
    const uint8_t* hi = lo + nh * R * 32;
    const uint8_t* sc = hi + nh * R * 16;
    const uint8_t* d = sc + nh * R * 6;
    const int h = c / 128, e = c % 128;
    const int q_lo = (lo[((int64_t)h * R + r) * 32 + 4 * (e / 16) + e % 4] >> (2 * ((e % 16) / 4))) & 3;
    const int q_hi = (hi[((int64_t)h * R + r) * 16 + 4 * (e / 32) + e % 4] >> ((e % 32) / 4)) & 1;
    const int q = q_lo | (q_hi << 2);
    const int j = e / 16;
    int scj = 0;
    for (int b = 0; b < 6; ++b) {
        const int bit = 6 * j + b;
        scj |= ((sc[((int64_t)h * R + r) * 6 + bit / 8] >> (bit % 8)) & 1) << b;
    }
    const double dv = fp16_value(load_u16(d + 2 * ((int64_t)(c / 256) * R + r)));
    return dv * (scj - 32) * (q - 4);
}

double iq4nl_weight(const uint8_t* m, int R, int C, int r, int c) {
    const int64_t blk = (int64_t)(c / 32) * R + r;
    const int j = c % 32;
    const uint8_t byte = m[blk * 16 + (j % 16)];
    const int q = j < 16 ? (byte & 0xF) : (byte >> 4);
    const double d = fp16_value(load_u16(m + (int64_t)R * C / 2 + 2 * blk));
    return d * iq4nl_levels()[q];
}

// Row r of a stored matrix into out[0..C).
void du_row(int fmt, const uint8_t* m, int R, int C, int r, double* out) {
    for (int c = 0; c < C; ++c) out[c] = du_weight(fmt, m, R, C, r, c);
}

// One matrix of an expert record: which = 0 gate [F][L], 1 up [F][L], 2 down
// [L][F].  efmt 0: NVFP4 record (codes, scales, tensor-scale tail); efmt 1:
// the Q3_K build (gate and up Q3_K, down IQ4_NL, no tail).
struct ExpertMatrix {
    int kind;            // 0 NVFP4, 1 Q3_K, 2 IQ4_NL
    const uint8_t* q;    // NVFP4 codes, or the whole Q3_K / IQ4_NL matrix
    const uint8_t* s;    // NVFP4 scales
    double ts;
    int R, C;
};

int64_t expert_record_bytes_fmt(int efmt, int L, int F) {
    return efmt == 1 ? 2 * q3k_matrix_bytes(F, L) + iq4nl_matrix_bytes(L, F) : expert_record_bytes(L, F);
}

ExpertMatrix expert_matrix(const uint8_t* rec, int L, int F, int which, int efmt = 0) {
    ExpertMatrix v;
    v.R = which < 2 ? F : L;
    v.C = which < 2 ? L : F;
    v.s = nullptr;
    v.ts = 1.0;
    if (efmt == 1) {
        v.kind = which < 2 ? 1 : 2;
        v.q = rec + which * q3k_matrix_bytes(F, L);
        return v;
    }
    const int64_t nq = (int64_t)L * F / 2, ns = (int64_t)L * F / 16;
    v.kind = 0;
    v.q = rec + which * nq;
    v.s = rec + 3 * nq + which * ns;
    v.ts = (double)load_f32(rec + 3 * nq + 3 * ns + 4 * which);
    return v;
}

void nvfp4_row(const ExpertMatrix& v, int r, double* out) {
    for (int c = 0; c < v.C; ++c) {
        if (v.kind == 0) out[c] = nvfp4_weight(v.q, v.s, v.ts, v.R, r, c);
        else if (v.kind == 1) out[c] = q3k_weight(v.q, v.R, v.C, r, c);
        else out[c] = iq4nl_weight(v.q, v.R, v.C, r, c);
    }
}

double dot(const double* a, const double* b, int n) {
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += a[i] * b[i];
    return acc;
}

double silu(double a) { return a / (1.0 + std::exp(-a)); }

// ---------------------------------------------------------------------------
// NVFP4 activations (the W4A4 mode)
// ---------------------------------------------------------------------------
//
// The teardown article's "What is 4-bit" section gives the NVFP4 format (E2M1
// values, one E4M3 scale per 16) for the weights.  The W4A4 mode applies it to
// the routed experts' inputs as well (h before gate/up, z before down); the
// pages give no rule for choosing activation scales, so this library uses
// the plainest one that keeps every block scale in the E4M3 range: one fp32
// scale per row, G = max|v| / (6 * 448), and per 16-element block the
// smallest E4M3 value s >= max|v_block| / (6 G), codes = E2M1 nearest (ties
// to the even code, saturating at 6) of v / (s G).  The kernels take these
// decisions in fp32 on the fp16 activations they store, so the oracle rounds
// the row to fp16 first and repeats the same fp32 operations; the products
// and sums after that are fp64.

// Round to the nearest IEEE binary16 value (ties to even), as a double.
double fp16_round(double x) {
    if (!std::isfinite(x)) return x;
    const double a = std::fabs(x);
    if (a >= 65520.0) return std::copysign(std::numeric_limits<double>::infinity(), x);
    int e;
    std::frexp(a, &e);                          // a = f 2^e, f in [0.5, 1)
    const int lead = std::max(e - 1, -14);      // exponent of the leading bit (subnormals: -14)
    const double quantum = std::ldexp(1.0, lead - 10);
    return std::copysign(std::nearbyint(a / quantum) * quantum, x);
}

// Code of the smallest E4M3 value not below s (0 < s), at most 448.
int e4m3_code_up(float s) {
    for (int c = 1; c < 0x7E; ++c)
        if ((float)e4m3fn_value(c) >= s) return c;
    return 0x7E;
}

// E2M1 code nearest to v (ties to the even code), saturating at +-6.
int e2m1_code_rn(float v) {
    const float a = std::fabs(v);
    int best = 0;
    double bd = std::numeric_limits<double>::infinity();
    for (int c = 0; c < 8; ++c) {
        const double d = std::fabs((double)a - e2m1_value(c));
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1)) {
            bd = d;
            best = c;
        }
    }
    return (v < 0.f ? 8 : 0) | best;
}

// One activation row v [K] (K % 16 == 0, fp16-representable values) ->
// out [K] = its NVFP4 value q * s * G; codes [K] (E2M1, low 4 bits),
// scales [K/16] (E4M3 codes) and G when not NULL.
void nvfp4_act_row(const double* v, int K, double* out, uint8_t* codes, uint8_t* scales, float* Gout) {
    float amax = 0.f;
    for (int k = 0; k < K; ++k) amax = std::max(amax, std::fabs((float)v[k]));
    const float G = amax > 0.f ? amax * (1.f / (6.f * 448.f)) : 1.f;
    if (Gout) *Gout = G;
    for (int b = 0; b < K / 16; ++b) {
        float bmax = 0.f;
        for (int e = 0; e < 16; ++e) bmax = std::max(bmax, std::fabs((float)v[16 * b + e]));
        int sc = 0;
        float sd = 0.f;
        if (bmax > 0.f) {
            sc = e4m3_code_up(bmax / (6.f * G));
            sd = (float)e4m3fn_value(sc) * G;
        }
        if (scales) scales[b] = (uint8_t)sc;
        const float inv = sc ? 1.f / sd : 0.f;
        for (int e = 0; e < 16; ++e) {
            const int q = sc ? e2m1_code_rn((float)v[16 * b + e] * inv) : 0;
            if (codes) codes[16 * b + e] = (uint8_t)q;
            out[16 * b + e] = sc ? e2m1_value(q) * e4m3fn_value(sc) * (double)G : 0.0;
        }
    }
}

}  // namespace

extern "C" {

struct orc_shape {
    int hidden, latent, n_experts, top_k, n_groups, ffn, shared_ffn;
    int du_fmt;        // 8: Q8_0, 4: Q4_0
    int router_bf16;   // 1: router weights are bf16 bits, 0: fp32
    int expert_fmt;    // 0: NVFP4 records, 1: Q3_K gate/up + IQ4_NL down records
    int act_fmt;       // 0: expert inputs as computed, 1: NVFP4 expert inputs (W4A4)
};

struct orc_layer {
    const void* router_w;          // [E][H]
    const float* router_b;         // [E] or NULL
    const uint8_t* expert_group;   // [E]
    const uint8_t* D;              // G matrices [latent][hidden]
    const uint8_t* U;              // G matrices [hidden][latent]
    const uint8_t* experts;        // E records
    const uint16_t* shared_gate;   // bf16 [Fs][H]
    const uint16_t* shared_up;     // bf16 [Fs][H]
    const uint16_t* shared_down;   // bf16 [H][Fs]
};

int orc_threads(void) { return omp_get_max_threads(); }

// ---- sizes and offsets ------------------------------------------------------

int64_t orc_du_matrix_bytes(int fmt, int R, int C) { return du_matrix_bytes(fmt, R, C); }
int64_t orc_expert_record_bytes(int L, int F) { return expert_record_bytes(L, F); }
// Byte offset of group g's matrix in a D or U blob, and of expert e's record.
int64_t orc_du_offset(int fmt, int g, int R, int C) { return (int64_t)g * du_matrix_bytes(fmt, R, C); }
int64_t orc_expert_offset(int e, int L, int F) { return (int64_t)e * expert_record_bytes(L, F); }
int64_t orc_expert_offset_fmt(int efmt, int e, int L, int F) { return (int64_t)e * expert_record_bytes_fmt(efmt, L, F); }

// ---- scalar decoders over arrays -----------------------------------------------

void orc_bf16_to_f64(const uint16_t* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_value(in[i]);
}
void orc_fp16_to_f64(const uint16_t* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = fp16_value(in[i]);
}
void orc_e2m1_to_f64(const uint8_t* codes, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e2m1_value(codes[i] & 0xF);
}
void orc_e4m3fn_to_f64(const uint8_t* codes, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3fn_value(codes[i]);
}

// ---- matrix decoders --------------------------------------------------------------

// Q8_0 / Q4_0 matrix [R][C] -> out [R][C] row-major.
int orc_decode_du(int fmt, const uint8_t* blob, int R, int C, double* out) {
    if ((fmt != kQ8_0 && fmt != kQ4_0) || C % 32) return -1;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < R; ++r) du_row(fmt, blob, R, C, r, out + (int64_t)r * C);
    return 0;
}

// NVFP4 matrix [R][C] (codes q, scales s, tensor scale ts) -> out [R][C].
int orc_decode_nvfp4(const uint8_t* q, const uint8_t* s, double ts, int R, int C, double* out) {
    if (C % 64) return -1;
    ExpertMatrix v{0, q, s, ts, R, C};
#pragma omp parallel for schedule(static)
    for (int r = 0; r < R; ++r) nvfp4_row(v, r, out + (int64_t)r * C);
    return 0;
}

// Q3_K (kind 1) or IQ4_NL (kind 2) matrix [R][C] -> out [R][C].
int orc_decode_q3k_iq4nl(int kind, const uint8_t* blob, int R, int C, double* out) {
    if ((kind == 1 && C % 256) || (kind == 2 && C % 32) || (kind != 1 && kind != 2)) return -1;
    ExpertMatrix v{kind, blob, nullptr, 1.0, R, C};
#pragma omp parallel for schedule(static)
    for (int r = 0; r < R; ++r) nvfp4_row(v, r, out + (int64_t)r * C);
    return 0;
}

// The 16 IQ4_NL levels as this oracle computes them from their definition.
void orc_iq4nl_levels(double* out) {
    for (int i = 0; i < 16; ++i) out[i] = iq4nl_levels()[i];
}

int64_t orc_expert_record_bytes_fmt(int efmt, int L, int F) { return expert_record_bytes_fmt(efmt, L, F); }

// Expert record (efmt 0 NVFP4, 1 Q3_K build) -> gate [F][L], up [F][L], down [L][F].
void orc_decode_expert_fmt(int efmt, const uint8_t* rec, int L, int F, double* wg, double* wu, double* wd) {
    double* outs[3] = {wg, wu, wd};
    for (int m = 0; m < 3; ++m) {
        const ExpertMatrix v = expert_matrix(rec, L, F, m, efmt);
#pragma omp parallel for schedule(static)
        for (int r = 0; r < v.R; ++r) nvfp4_row(v, r, outs[m] + (int64_t)r * v.C);
    }
}

// NVFP4 expert record -> gate [F][L], up [F][L], down [L][F].
void orc_decode_expert(const uint8_t* rec, int L, int F, double* wg, double* wu, double* wd) {
    double* outs[3] = {wg, wu, wd};
    for (int m = 0; m < 3; ++m) {
        const ExpertMatrix v = expert_matrix(rec, L, F, m);
#pragma omp parallel for schedule(static)
        for (int r = 0; r < v.R; ++r) nvfp4_row(v, r, outs[m] + (int64_t)r * v.C);
    }
}

// ---- router -----------------------------------------------------------------------

// Router over all experts (step 1).  x [T][H], Wr [E][H] fp64, b [E] or NULL.
// idx [T][K] in selection order, w [T][K], gap [T] = l_(K) - l_(K+1) (inf
// when K = E), logits [T][E] or NULL.
void orc_route(const double* x, const double* Wr, const double* b, int T, int H, int E, int K, int64_t* idx,
               double* w, double* gap, double* logits) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        std::vector<double> l(E);
        for (int e = 0; e < E; ++e) l[e] = dot(x + (int64_t)t * H, Wr + (int64_t)e * H, H) + (b ? b[e] : 0.0);
        std::vector<int> order(E);
        for (int e = 0; e < E; ++e) order[e] = e;
        std::sort(order.begin(), order.end(), [&](int a, int c) { return l[a] > l[c] || (l[a] == l[c] && a < c); });
        // softmax over all E experts (max subtracted), then renormalised over the kept K
        const double lmax = l[order[0]];
        double z = 0.0;
        for (int e = 0; e < E; ++e) z += std::exp(l[e] - lmax);
        double kept = 0.0;
        for (int k = 0; k < K; ++k) kept += std::exp(l[order[k]] - lmax) / z;
        for (int k = 0; k < K; ++k) {
            idx[(int64_t)t * K + k] = order[k];
            w[(int64_t)t * K + k] = (std::exp(l[order[k]] - lmax) / z) / kept;
        }
        gap[t] = K < E ? l[order[K - 1]] - l[order[K]] : std::numeric_limits<double>::infinity();
        if (logits)
            for (int e = 0; e < E; ++e) logits[(int64_t)t * E + e] = l[e];
    }
}

// ---- pieces of the block (also used by the tests' special cases) -------------------

// Shared expert on x [T][H] (step 7): y [T][H] = S_down (silu(S_gate x) * (S_up x)).
void orc_shared_expert(const orc_shape* s, const orc_layer* ly, const double* x, int T, double* y) {
    const int H = s->hidden, Fs = s->shared_ffn;
    std::vector<double> z((size_t)T * Fs);
#pragma omp parallel
    {
        std::vector<double> rg(H), ru(H);
#pragma omp for schedule(static)
        for (int f = 0; f < Fs; ++f) {
            orc_bf16_to_f64(ly->shared_gate + (int64_t)f * H, H, rg.data());
            orc_bf16_to_f64(ly->shared_up + (int64_t)f * H, H, ru.data());
            for (int t = 0; t < T; ++t) {
                const double* xt = x + (int64_t)t * H;
                z[(size_t)t * Fs + f] = silu(dot(rg.data(), xt, H)) * dot(ru.data(), xt, H);
            }
        }
    }
#pragma omp parallel
    {
        std::vector<double> rd(Fs);
#pragma omp for schedule(static)
        for (int r = 0; r < H; ++r) {
            orc_bf16_to_f64(ly->shared_down + (int64_t)r * Fs, Fs, rd.data());
            for (int t = 0; t < T; ++t) y[(int64_t)t * H + r] = dot(rd.data(), z.data() + (size_t)t * Fs, Fs);
        }
    }
}

// One expert on n latent vectors h [n][L] (step 4): o [n][L].  act = 1:
// h and then z are taken as their NVFP4 activation values (W4A4 mode).
void orc_expert_apply_act(int efmt, int act, const uint8_t* rec, int L, int F, const double* h_in, int n, double* o) {
    const ExpertMatrix vg = expert_matrix(rec, L, F, 0, efmt), vu = expert_matrix(rec, L, F, 1, efmt),
                       vd = expert_matrix(rec, L, F, 2, efmt);
    std::vector<double> rg(L), ru(L), rd(F), z((size_t)n * F), hq;
    const double* h = h_in;
    if (act == 1) {
        hq.resize((size_t)n * L);
        std::vector<double> r16(L);
        for (int i = 0; i < n; ++i) {
            for (int k = 0; k < L; ++k) r16[k] = fp16_round(h_in[(int64_t)i * L + k]);
            nvfp4_act_row(r16.data(), L, hq.data() + (size_t)i * L, nullptr, nullptr, nullptr);
        }
        h = hq.data();
    }
    for (int f = 0; f < F; ++f) {
        nvfp4_row(vg, f, rg.data());
        nvfp4_row(vu, f, ru.data());
        for (int i = 0; i < n; ++i) {
            const double* hi = h + (int64_t)i * L;
            z[(size_t)i * F + f] = silu(dot(rg.data(), hi, L)) * dot(ru.data(), hi, L);
        }
    }
    if (act == 1) {
        std::vector<double> r16(F);
        for (int i = 0; i < n; ++i) {
            for (int f = 0; f < F; ++f) r16[f] = fp16_round(z[(size_t)i * F + f]);
            nvfp4_act_row(r16.data(), F, z.data() + (size_t)i * F, nullptr, nullptr, nullptr);
        }
    }
    for (int r = 0; r < L; ++r) {
        nvfp4_row(vd, r, rd.data());
        for (int i = 0; i < n; ++i) o[(int64_t)i * L + r] = dot(rd.data(), z.data() + (size_t)i * F, F);
    }
}

void orc_expert_apply_fmt(int efmt, const uint8_t* rec, int L, int F, const double* h, int n, double* o) {
    orc_expert_apply_act(efmt, 0, rec, L, F, h, n, o);
}

void orc_expert_apply(const uint8_t* rec, int L, int F, const double* h, int n, double* o) {
    orc_expert_apply_fmt(0, rec, L, F, h, n, o);
}

// One activation row quantised as the W4A4 mode does (fp16 rounding first):
// out [K] its NVFP4 values, codes [K], scales [K/16], G [1] (any may be NULL
// except out).  K % 16 == 0.
void orc_nvfp4_act_quantize(const double* v, int K, double* out, uint8_t* codes, uint8_t* scales, float* G) {
    std::vector<double> r16(K);
    for (int k = 0; k < K; ++k) r16[k] = fp16_round(v[k]);
    nvfp4_act_row(r16.data(), K, out, codes, scales, G);
}

double orc_fp16_round(double x) { return fp16_round(x); }

// y [n][R] = M x for the stored Q8_0 / Q4_0 matrix M [R][C] and n vectors x [n][C].
void orc_du_apply(int fmt, const uint8_t* m, int R, int C, const double* x, int n, double* y) {
#pragma omp parallel
    {
        std::vector<double> row(C);
#pragma omp for schedule(static)
        for (int r = 0; r < R; ++r) {
            du_row(fmt, m, R, C, r, row.data());
            for (int i = 0; i < n; ++i) y[(int64_t)i * R + r] = dot(row.data(), x + (int64_t)i * C, C);
        }
    }
}

// ---- the block ----------------------------------------------------------------------

// One latent-MoE block on x [T][H] (fp64): steps 1-8.  residual: bf16 bits
// [T][H] or NULL.  inject_idx / inject_w ([T][K]) replace the router's
// choice when non-NULL (the router still runs for gap).  Outputs y [T][H],
// idx, w [T][K] (the routing used) and gap [T].  Returns 0, or -1 for an
// expert index or group label out of range.
int orc_forward(const orc_shape* s, const orc_layer* ly, const double* x, const uint16_t* residual,
                const int64_t* inject_idx, const double* inject_w, int T, double* y, int64_t* idx, double* w,
                double* gap) {
    const int H = s->hidden, L = s->latent, E = s->n_experts, K = s->top_k, G = s->n_groups, F = s->ffn;
    // step 1: router
    std::vector<double> Wr((size_t)E * H);
    if (s->router_bf16) orc_bf16_to_f64(static_cast<const uint16_t*>(ly->router_w), (int64_t)E * H, Wr.data());
    else
        for (int64_t i = 0; i < (int64_t)E * H; ++i) Wr[i] = (double)static_cast<const float*>(ly->router_w)[i];
    std::vector<double> b;
    if (ly->router_b) {
        b.resize(E);
        for (int e = 0; e < E; ++e) b[e] = (double)ly->router_b[e];
    }
    orc_route(x, Wr.data(), ly->router_b ? b.data() : nullptr, T, H, E, K, idx, w, gap, nullptr);
    if (inject_idx) {
        for (int64_t i = 0; i < (int64_t)T * K; ++i) {
            idx[i] = inject_idx[i];
            w[i] = inject_w[i];
        }
    }
    for (int64_t i = 0; i < (int64_t)T * K; ++i)
        if (idx[i] < 0 || idx[i] >= E || ly->expert_group[idx[i]] >= G) return -1;
    // step 2: hit groups of each token
    std::vector<char> hit((size_t)T * G, 0);
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) hit[(size_t)t * G + ly->expert_group[idx[(int64_t)t * K + k]]] = 1;
    // step 3: h[t][g] = D_g x_t for the tokens that hit g
    std::vector<double> h((size_t)T * G * L, 0.0);
    const int64_t du_b = du_matrix_bytes(s->du_fmt, L, H);
    for (int g = 0; g < G; ++g) {
        std::vector<int> toks;
        for (int t = 0; t < T; ++t)
            if (hit[(size_t)t * G + g]) toks.push_back(t);
        if (toks.empty()) continue;
        std::vector<double> xs(toks.size() * (size_t)H), hs(toks.size() * (size_t)L);
        for (size_t i = 0; i < toks.size(); ++i) std::memcpy(&xs[i * H], x + (int64_t)toks[i] * H, sizeof(double) * H);
        orc_du_apply(s->du_fmt, ly->D + g * du_b, L, H, xs.data(), (int)toks.size(), hs.data());
        for (size_t i = 0; i < toks.size(); ++i)
            std::memcpy(&h[((size_t)toks[i] * G + g) * L], &hs[i * L], sizeof(double) * L);
    }
    // step 4: o[t][k] for every routed pair, each distinct expert once over its pairs
    std::vector<std::vector<int>> pairs(E);
    for (int64_t i = 0; i < (int64_t)T * K; ++i) pairs[idx[i]].push_back((int)i);
    std::vector<int> used;
    for (int e = 0; e < E; ++e)
        if (!pairs[e].empty()) used.push_back(e);
    std::vector<double> o((size_t)T * K * L);
    const int64_t rec_b = expert_record_bytes_fmt(s->expert_fmt, L, F);
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < (int)used.size(); ++u) {
        const int e = used[u];
        const int g = ly->expert_group[e];
        const std::vector<int>& pe = pairs[e];
        std::vector<double> hin(pe.size() * (size_t)L), out(pe.size() * (size_t)L);
        for (size_t i = 0; i < pe.size(); ++i)
            std::memcpy(&hin[i * L], &h[((size_t)(pe[i] / K) * G + g) * L], sizeof(double) * L);
        orc_expert_apply_act(s->expert_fmt, s->act_fmt, ly->experts + e * rec_b, L, F, hin.data(), (int)pe.size(),
                             out.data());
        for (size_t i = 0; i < pe.size(); ++i) std::memcpy(&o[(size_t)pe[i] * L], &out[i * L], sizeof(double) * L);
    }
    // step 7 first (the output starts as the shared expert), then steps 5, 6
    orc_shared_expert(s, ly, x, T, y);
    for (int g = 0; g < G; ++g) {
        std::vector<int> toks;
        for (int t = 0; t < T; ++t)
            if (hit[(size_t)t * G + g]) toks.push_back(t);
        if (toks.empty()) continue;
        // step 5: s[t][g] = sum over k in group g of w_k o_k (k order)
        std::vector<double> sg(toks.size() * (size_t)L, 0.0), ug(toks.size() * (size_t)H);
        for (size_t i = 0; i < toks.size(); ++i) {
            const int t = toks[i];
            for (int k = 0; k < K; ++k) {
                const int64_t pi = (int64_t)t * K + k;
                if (ly->expert_group[idx[pi]] != g) continue;
                for (int l = 0; l < L; ++l) sg[i * L + l] += w[pi] * o[(size_t)pi * L + l];
            }
        }
        // step 6: y += U_g s[t][g]
        orc_du_apply(s->du_fmt, ly->U + g * du_b, H, L, sg.data(), (int)toks.size(), ug.data());
        for (size_t i = 0; i < toks.size(); ++i)
            for (int r = 0; r < H; ++r) y[(int64_t)toks[i] * H + r] += ug[i * H + r];
    }
    // step 8: residual
    if (residual)
        for (int64_t i = 0; i < (int64_t)T * H; ++i) y[i] += bf16_value(residual[i]);
    return 0;
}

// ---- ablation: D over all groups with Q8_1 activations -------------------------------
//
// The teardown article's reference kernel (section "A latent in front of the
// experts", its code excerpt) quantises each token row to Q8_1 and runs D over
// all 8 groups with integer dot products.  Q8_1 as read here, per block of 32
// consecutive elements of a row (the pages do not print it; every rounding
// is an fp32 operation, so the GPU takes the same integer decisions):
//   d = fp16(amax / 127)              amax = max |x_j| of the block (fp32)
//   q_j = clamp(rint(x_j / float(d)), -127, 127)     (all zero when d == 0)
// and the sum s = sum_j q_j (an integer; the fp16 d*s of the stored format
// only matters for Q4_0 weights, whose -8 offset it cancels exactly here).
// orc_quantize_q8_1: x [T][H] fp32 -> q int8 [T][H], d fp16 bits [T][H/32].
void orc_quantize_q8_1(const float* x, int T, int H, int8_t* q, uint16_t* d_bits) {
    for (int t = 0; t < T; ++t) {
        for (int b = 0; b < H / 32; ++b) {
            const float* xb = x + (int64_t)t * H + b * 32;
            float amax = 0.f;
            for (int j = 0; j < 32; ++j) amax = std::max(amax, std::fabs(xb[j]));
            const float d32 = amax / 127.0f;
            // fp32 -> fp16, round to nearest even (_Float16 conversion)
            const _Float16 d16 = (_Float16)d32;
            uint16_t bits;
            std::memcpy(&bits, &d16, 2);
            d_bits[(int64_t)t * (H / 32) + b] = bits;
            const float dv = (float)d16;
            for (int j = 0; j < 32; ++j) {
                float v = dv > 0.f ? std::rint(xb[j] / dv) : 0.f;
                v = std::min(127.f, std::max(-127.f, v));
                q[(int64_t)t * H + b * 32 + j] = (int8_t)v;
            }
        }
    }
}

// h [T][G][L] = D_g xq for every group g, where xq is the Q8_1 reading of the
// fp32 rows x [T][H]: per block, d_w * d_x * sum_j w_j q_j (integer sum, exact).
void orc_dproj_q8_1(int fmt, const uint8_t* D, int G, int L, int H, const float* x, int T, double* h) {
    std::vector<int8_t> q((size_t)T * H);
    std::vector<uint16_t> dx((size_t)T * (H / 32));
    orc_quantize_q8_1(x, T, H, q.data(), dx.data());
    const int64_t mb = du_matrix_bytes(fmt, L, H);
    for (int g = 0; g < G; ++g) {
        const uint8_t* m = D + g * mb;
#pragma omp parallel for schedule(static)
        for (int r = 0; r < L; ++r) {
            for (int t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int b = 0; b < H / 32; ++b) {
                    const int64_t blk = (int64_t)b * L + r;
                    int64_t isum = 0;
                    double dw;
                    for (int j = 0; j < 32; ++j) {
                        int wq;
                        if (fmt == kQ8_0) {
                            wq = (int8_t)m[blk * 32 + j];
                        } else {
                            const uint8_t byte = m[blk * 16 + (j % 16)];
                            wq = (j < 16 ? (byte & 0xF) : (byte >> 4)) - 8;
                        }
                        isum += (int64_t)wq * q[(size_t)t * H + b * 32 + j];
                    }
                    dw = fp16_value(load_u16(m + (int64_t)L * H / 32 * (fmt == kQ8_0 ? 32 : 16) + 2 * blk));
                    acc += dw * fp16_value(dx[(size_t)t * (H / 32) + b]) * (double)isum;
                }
                h[((int64_t)t * G + g) * L + r] = acc;
            }
        }
    }
}

// RMSNorm per row: out = gamma * v / sqrt(mean(v^2) + eps).
void orc_rmsnorm(const double* v, const double* gamma, double eps, int T, int H, double* out) {
    for (int t = 0; t < T; ++t) {
        const double* vt = v + (int64_t)t * H;
        double ss = 0.0;
        for (int i = 0; i < H; ++i) ss += vt[i] * vt[i];
        const double r = std::sqrt(ss / H + eps);
        for (int i = 0; i < H; ++i) out[(int64_t)t * H + i] = gamma[i] * vt[i] / r;
    }
}

// One pre-norm residual layer of the stack: y = x + block(RMSNorm(x)), x
// given as bf16 bits (the stack keeps its residual stream in bf16).
int orc_stack_layer(const orc_shape* s, const orc_layer* ly, const uint16_t* x_bits, const double* gamma, double eps,
                    const int64_t* inject_idx, const double* inject_w, int T, double* y, int64_t* idx, double* w,
                    double* gap) {
    const int H = s->hidden;
    std::vector<double> x((size_t)T * H), xn((size_t)T * H);
    orc_bf16_to_f64(x_bits, (int64_t)T * H, x.data());
    orc_rmsnorm(x.data(), gamma, eps, T, H, xn.data());
    const int rc = orc_forward(s, ly, xn.data(), nullptr, inject_idx, inject_w, T, y, idx, w, gap);
    if (rc) return rc;
    for (int64_t i = 0; i < (int64_t)T * H; ++i) y[i] += x[i];
    return 0;
}

}  // extern "C"
