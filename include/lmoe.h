/*
 * lmoe.h -- C ABI of the latent mixture-of-experts FFN block on NVIDIA B200
 * (sm_100a).
 *
 * The block (teardown article "Edge0-145B: a Qwen MoE with its experts
 * squeezed, and a 51B table left on the SSD", section "A latent in front of
 * the experts", layer equation; Edge0 145B / 120B model page, "Model
 * profile" and the architecture tables), per token x (width `hidden`):
 *
 *   router   l = W_r x + b; softmax over all experts; keep the top_k by
 *            (logit desc, index asc); w_k = p_k / sum of the kept p
 *   groups   every expert e carries a label group[e] in [0, n_groups)
 *   D        h_g = D_g x                 for each group g hit by the token
 *   experts  o_k = W_down (silu(W_gate h) * (W_up h)),  h = h_{group[e_k]}
 *   U        y = sum_g U_g (sum_{k: group[e_k] = g} w_k o_k)
 *   shared   y += S_down (silu(S_gate x) * (S_up x))    (full width)
 *   residual y += residual                               (optional)
 *
 * Conventions for every call:
 *   - Pointers named *_host are host memory; every other pointer is device
 *     memory on the current device, owned by the caller.  The library never
 *     allocates device memory; scratch comes from the caller's workspace
 *     (size from lmoe_workspace_bytes, 256-byte aligned).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it.  A negative return means nothing was launched.
 *   - All device pointers must be 16-byte aligned.
 *   - A workspace may be used by one call at a time (calls on one stream
 *     serialise; calls on different streams need different workspaces).
 *   - Faults the kernels detect (an expert_group label >= n_groups, a
 *     routed index out of range) are recorded in the workspace's status
 *     word, read with lmoe_last_device_status.
 *
 * Storage layouts (all little-endian):
 *   x, y, residual       bf16 [T][hidden]
 *   router_w             fp32 or bf16 (cfg.router_dtype) [n_experts][hidden]
 *   router_b             fp32 [n_experts] or NULL
 *   expert_group         uint8 [n_experts]
 *   shared.gate, .up     bf16 [shared_ffn][hidden]
 *   shared.down          bf16 [hidden][shared_ffn]
 *   D                    n_groups matrices [latent rows][hidden cols], then
 *   U                    n_groups matrices [hidden rows][latent cols], each
 *     Q8_0:  int8 q [cols/32][rows][32], then fp16 d [cols/32][rows];
 *            weight(r, c) = d * q                       (34 bytes per 32)
 *     Q4_0:  uint8 q [cols/32][rows][16] (byte j: low nibble element j,
 *            high nibble element j+16), then fp16 d [cols/32][rows];
 *            weight = d * (q - 8)                      (18 bytes per 32)
 *   experts              n_experts records of lmoe_expert_record_bytes():
 *     gate.q [latent/32][ffn][16] | up.q [latent/32][ffn][16] |
 *     down.q [ffn/32][latent][16] | gate.s [latent/64][ffn][4] |
 *     up.s [latent/64][ffn][4] | down.s [ffn/64][latent][4] |
 *     fp32 ts_gate, ts_up, ts_down, uint32 0
 *     q bytes hold E2M1 codes, element 2i in the low nibble of byte i;
 *     s bytes are E4M3 scales, byte j of a word scales elements 16j..16j+15
 *     of its 64-wide column group; weight = e2m1 * e4m3 * ts.
 *     (1,935,376 bytes at latent 1792, ffn 640: the record size printed in
 *     the teardown article, section "What is 4-bit".)
 *   experts, cfg.expert_fmt == LMOE_EXPERTS_Q3K: records of
 *     gate (Q3_K [ffn][latent]) | up (Q3_K [ffn][latent]) | down (IQ4_NL
 *     [latent][ffn]), no tail (1,630,720 bytes at latent 1792, 1,164,800 at
 *     1280: the Q3_K record sizes the pages print; they give the type names
 *     and byte counts only, the arrangement is this library's):
 *     Q3_K [R][C], 110 bytes per 256 weights of a row, planes over 128-column
 *       halves h:  lo [C/128][R][32] (element 16w + 4i + b of the half in
 *       byte 4w + b, bits 2i..2i+1) | hi [C/128][R][16] (element 32v + 4i + b
 *       in byte 4v + b, bit i) | sc [C/128][R][6] (sub-block j = elements
 *       16j..16j+15 at bits 6j..6j+5, little-endian) | d fp16 [C/256][R];
 *       weight = d * (sc_j - 32) * (q - 4), q = lo | hi << 2
 *     IQ4_NL [R][C], 18 bytes per 32: codes [C/32][R][16] (byte j: element j
 *       low nibble, element j+16 high) | d fp16 [C/32][R];
 *       weight = d * level[code], the 16 levels being the standard normal
 *       quantiles at (i + 1/2) / 16 scaled to an outermost 127 and rounded:
 *       -127 -90 -69 -53 -39 -27 -16 -5 5 16 27 39 53 69 90 127
 *
 * Shape limits (lmoe_cfg_check): hidden, latent multiples of 128; ffn,
 * shared_ffn multiples of 64; 1 <= top_k <= 16 and top_k <= n_experts <=
 * 1024; 1 <= n_groups <= 64; with Q3_K experts latent a multiple of 256.
 */
#ifndef LMOE_H
#define LMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LMOE_API __attribute__((visibility("default")))
#else
#define LMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LMOE_OK = 0,
    LMOE_ERR_ARG = -1,           /* null pointer, bad size, misaligned pointer */
    LMOE_ERR_UNSUPPORTED = -2,   /* shape or format outside the limits above */
    LMOE_ERR_CUDA = -3,          /* a CUDA runtime call failed */
    LMOE_ERR_WORKSPACE = -4,     /* workspace smaller than lmoe_workspace_bytes */
    LMOE_ERR_TIMEOUT = -5,       /* a bounded device wait gave up */
    LMOE_ERR_DEVICE_CHECK = -6   /* a kernel found an invalid input (see header) */
} lmoe_status;

typedef enum { LMOE_Q8_0 = 8, LMOE_Q4_0 = 4 } lmoe_du_fmt;   /* D/U block formats */
typedef enum { LMOE_F32 = 0, LMOE_BF16 = 1 } lmoe_dtype;     /* router weight type */
typedef enum { LMOE_EXPERTS_NVFP4 = 0, LMOE_EXPERTS_Q3K = 1 } lmoe_expert_fmt;   /* expert records */
/* Expert inputs.  LMOE_ACT_FP16: h and z enter the expert contractions as
 * computed (staged in fp16, fp32 accumulation).  LMOE_ACT_NVFP4 (W4A4, NVFP4
 * expert records only): the teardown article's NVFP4 format ("What is
 * 4-bit") applied to h before gate/up and to z before down, each row
 * quantised on its fp16 values in fp32: G = max|v| / (6 * 448), per 16
 * elements the smallest E4M3 scale s >= max|v_block| / (6 G), E2M1 codes
 * nearest (ties to even, saturating) to v / (s G); the contractions then run
 * as NVFP4 x NVFP4 on the tensor cores (tcgen05 kind::mxf4nvf4).  Needs
 * latent and ffn multiples of 128 up to 2048. */
typedef enum { LMOE_ACT_FP16 = 0, LMOE_ACT_NVFP4 = 1 } lmoe_act_fmt;

typedef struct {
    int hidden;        /* model width (2560 for Edge0 145B / 120B) */
    int latent;        /* latent width l (1792 / 1280) */
    int n_experts;     /* routed experts per layer (512) */
    int top_k;         /* experts per token (10) */
    int n_groups;      /* D/U pairs per layer (8) */
    int ffn;           /* expert SwiGLU width (640) */
    int shared_ffn;    /* shared expert SwiGLU width (640) */
    int du_fmt;        /* lmoe_du_fmt */
    int router_dtype;  /* lmoe_dtype */
    int expert_fmt;    /* lmoe_expert_fmt (0: NVFP4 records) */
    int act_fmt;       /* lmoe_act_fmt (0: fp16 expert inputs) */
} lmoe_cfg;

typedef struct {
    const void* gate;  /* bf16 [shared_ffn][hidden] */
    const void* up;    /* bf16 [shared_ffn][hidden] */
    const void* down;  /* bf16 [hidden][shared_ffn] */
} lmoe_shared;

/* One layer of a stack; all device pointers. */
typedef struct {
    const void* router_w;
    const float* router_b;        /* may be NULL */
    const uint8_t* expert_group;
    const void* D;
    const void* U;
    const void* experts;
    lmoe_shared shared;
    const void* norm_gamma;       /* bf16 [hidden]: RMSNorm weight before the block */
} lmoe_layer;

/* LMOE_OK if the shape is supported, else LMOE_ERR_UNSUPPORTED / LMOE_ERR_ARG.
 * (Shapes: Edge0 145B / 120B model page, architecture tables: hidden 2560,
 * 512 experts, top-10, 8 D/U groups, latent 1792 or 1280, SwiGLU 640.) */
LMOE_API int lmoe_cfg_check(const lmoe_cfg* cfg);

/* Bytes of one expert record, of one D (or U) blob holding all n_groups
 * matrices, and of the workspace needed for up to T_max tokens.  0 if the
 * configuration is unsupported.  (Record size: teardown article, section
 * "What is 4-bit": 1,935,376 bytes per expert at latent 1792; Q8_0 / Q4_0
 * sizes: 34 and 18 bytes per 32 weights; the model page, "Model profile",
 * stores D and U as Q8 or Q4.) */
LMOE_API size_t lmoe_expert_record_bytes(const lmoe_cfg* cfg);
LMOE_API size_t lmoe_du_bytes(const lmoe_cfg* cfg);
LMOE_API size_t lmoe_workspace_bytes(const lmoe_cfg* cfg, int T_max);

/* Router only: logits, softmax, top_k and renormalised weights.
 * Defining passage: model page, "Model profile" (the router picks 10 of the
 * 512 experts of a layer); the function itself (softmax over all experts,
 * top-k, renormalise over the kept, bias added to the logits, lowest index
 * on ties) is not printed on the pages and follows the task's workload
 * statement of the block.
 *   x         bf16 [T][hidden], device
 *   router_w  fp32 or bf16 [n_experts][hidden]; router_b fp32 [n_experts] or NULL
 *   topk_idx  int32 [T][top_k] and topk_w fp32 [T][top_k], written in
 *             selection order (logit descending, index ascending on ties)
 *   ws        workspace of at least lmoe_workspace_bytes(cfg, T) bytes
 * Errors: LMOE_ERR_ARG (null, misaligned, T < 0), LMOE_ERR_UNSUPPORTED,
 * LMOE_ERR_WORKSPACE; T = 0 launches nothing. */
LMOE_API int lmoe_route(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b, int T,
               int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream);

/* The block: y [T][hidden] bf16 = block(x).
 * Defining passage: teardown article, section "A latent in front of the
 * experts" (layer equation: the token is compressed by D_g, the experts run
 * at latent width, their weighted outputs are summed and widened back by
 * U_g), read per group (the same section gives every expert one of eight
 * group labels); shared expert at full width: model page, "Model profile"
 * (only the expert pool runs at the latent width).
 * Arguments: x bf16 [T][hidden]; weights as in the storage layouts above;
 * y bf16 [T][hidden] (must not overlap x); ws of lmoe_workspace_bytes(cfg, T).
 * Errors: LMOE_ERR_ARG / _UNSUPPORTED / _WORKSPACE before any launch; kernel
 * findings through lmoe_last_device_status.
 * Environment: LMOE_FEW_TOKEN_EXPERTS=tensor_cores (read at every call)
 * runs the NVFP4 expert contractions of steps of T <= 8 on the tensor cores
 * (kind::mxf4nvf4 on the stored bytes, the fp16 activations as six E2M1
 * terms) instead of the weight-streaming kernels; the result agrees within
 * the same tolerance, the default is faster on the Edge0 shapes. */
LMOE_API int lmoe_forward(const lmoe_cfg* cfg, const void* x, const void* router_w, const uint8_t* expert_group,
                 const void* D, const void* U, const void* experts, const lmoe_shared* shared,
                 void* y, int T, void* ws, size_t ws_bytes, void* stream);

/* The block with every option (same passage as lmoe_forward):
 *   router_b     per-expert bias added to the logits, or NULL
 *   residual     bf16 [T][hidden] added to y, or NULL; y overlaps neither x
 *                nor residual
 *   inject_idx / inject_w   when both non-NULL, the routing is taken from
 *                them ([T][top_k]) instead of the router (the router still
 *                runs; used where two logits are too close to compare)
 *   out_idx / out_w         when non-NULL, receive the routing used. */
LMOE_API int lmoe_forward_ex(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b,
                    const uint8_t* expert_group, const void* D, const void* U, const void* experts,
                    const lmoe_shared* shared, const void* residual,
                    const int32_t* inject_idx, const float* inject_w, int32_t* out_idx, float* out_w,
                    void* y, int T, void* ws, size_t ws_bytes, void* stream);

/* As lmoe_forward (same passage), with x_host and y_host in host memory
 * (page-locked for the copies to overlap): copies x in, runs the block,
 * copies y out, all on `stream`.  The call returns once y_host is written;
 * the workspace holds the device copies of x and y. */
LMOE_API int lmoe_forward_host(const lmoe_cfg* cfg, const void* x_host, const void* router_w, const float* router_b,
                      const uint8_t* expert_group, const void* D, const void* U, const void* experts,
                      const lmoe_shared* shared, void* y_host, int T, void* ws, size_t ws_bytes, void* stream);

/* n_layers pre-norm residual layers: x <- x + block_l(RMSNorm_l(x)), the
 * residual stream kept in bf16; RMSNorm(v) = gamma * v / sqrt(mean(v^2) + eps).
 * Defining passage: model page, architecture tables (48 layers, each with a
 * latent-MoE FFN); the norm, its place before the block and the residual
 * add are not printed there (attention is omitted) and follow the task's
 * statement of the stack.
 * x and y are bf16 [T][hidden] and may not alias.  `layers` is a host array
 * of device pointers (norm_gamma required).  Errors as lmoe_forward. */
LMOE_API int lmoe_stack_forward(const lmoe_cfg* cfg, int n_layers, const lmoe_layer* layers, const void* x, void* y,
                       int T, float rms_eps, void* ws, size_t ws_bytes, void* stream);

/* Waits for `stream`, then returns and clears the workspace status word
 * (LMOE_OK, or LMOE_ERR_DEVICE_CHECK / LMOE_ERR_TIMEOUT set by a kernel). */
LMOE_API int lmoe_last_device_status(void* ws, size_t ws_bytes, void* stream);

/* Static text for a status code. */
LMOE_API const char* lmoe_status_str(int status);

/* Diagnostics: decode one stored matrix to fp32 [rows][cols] on the device
 * with the same decoders the kernels use.  fmt: LMOE_Q8_0, LMOE_Q4_0, 1 for
 * an NVFP4 matrix (q then s as in an expert record, scaled by ts), 2 for a
 * Q3_K matrix, 3 for an IQ4_NL matrix (layouts above; ts unused). */
LMOE_API int lmoe_debug_decode(int fmt, const void* blob, int rows, int cols, float ts, float* out, void* stream);

/* Diagnostics: the W4A4 mode's activation quantiser on its own.  Defining
 * passage: teardown article, section "What is 4-bit" (NVFP4: E2M1 values,
 * one E4M3 scale per 16), applied to activations by the rule under
 * lmoe_act_fmt.  src: fp16 [n][cols] (device, 16-byte aligned), cols a
 * multiple of 64.  Outputs (device, caller-owned): codes [cols/32][n][16]
 * bytes (element 2i of a row's 32-column chunk in the low nibble of byte i),
 * scales [cols/64][n] 32-bit words (byte j: the E4M3 code of the row's
 * 16-column block 4k + j), G [n] fp32.  Returns LMOE_ERR_ARG for null,
 * misaligned or badly sized arguments. */
LMOE_API int lmoe_debug_act_quant(const void* src, int n, int cols, void* codes, void* scales, float* G, void* stream);

/* Profiling: while n > 0, every later forward call records events[0] before
 * its first kernel, events[i] before kernel i and one more event after its
 * last kernel, on the call's stream, until the n events are used (each call
 * starts again at events[0]).  `events` holds cudaEvent_t handles owned by
 * the caller; n = 0 turns recording off.  At most 16 events. */
LMOE_API int lmoe_profile_stage_events(void* const* events, int n);

/* Ablation of D_g.  Defining passage: teardown article, section "A latent
 * in front of the experts" -- its code excerpt shows the reference kernel
 * quantising each token row to Q8_1 and running D over all 8 groups with
 * integer dot products, where this library runs D on fp16 activations and
 * needs only the groups a token hits.  h fp32 [T][n_groups][latent] =
 * D_g x for every group g with bit g of group_mask set (other groups of h
 * are not written):
 *   act_fmt 0  fp16 activations, fp16 x fp16 tensor-core products, fp32 sums
 *   act_fmt 1  Q8_1 activations: per block of 32, d = fp16(amax / 127) and
 *              q = rint(x / d) clamped to +-127 (fp32 operations), then
 *              integer products per block scaled by d_w * d
 * x bf16 [T][hidden]; D as in lmoe_forward; ws of lmoe_workspace_bytes(cfg,
 * T).  n_groups <= 32.  Errors: LMOE_ERR_ARG, _UNSUPPORTED, _WORKSPACE. */
LMOE_API int lmoe_dproj_ablation(const lmoe_cfg* cfg, const void* x, const void* D, int act_fmt, uint32_t group_mask,
                                 float* h, int T, void* ws, size_t ws_bytes, void* stream);

/* Router only, for callers that cannot call cudaMalloc (code inside a host
 * framework that owns every device allocation, or a path where no workspace
 * can be handed in).  Same results as lmoe_route, but the scratch lives in a
 * fixed array of 274,432 bytes that is part of this library; every device
 * that loads the library holds one copy until the process exits.  The paper
 * has no counterpart to this call.
 *   - Limits: T <= 64, n_experts <= 1024, top_k <= 16; larger sizes return
 *     LMOE_ERR_WORKSPACE and launch nothing.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before
 *     any stream capture.
 *   - Every call on a device shares the one array and clears its control
 *     words itself; calls that overlap on the GPU (other streams, other host
 *     threads) race on it and must be serialised by the caller.
 *   - topk_idx / topk_w as in lmoe_route; all pointers device memory. */
LMOE_API int lmoe_route_noalloc(const lmoe_cfg* cfg, const void* x, const void* router_w, const float* router_b,
                                int T, int32_t* topk_idx, float* topk_w, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LMOE_H */
