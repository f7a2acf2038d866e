// Routing of a few-token step (T <= 8) in one CTA's shared memory: softmax
// top-K per token and the bucketing of the (token, k) pairs by expert.  Used
// by the last CTA of the router kernel, which publishes the result to the
// workspace for the kernels after it.
#pragma once

#include "lmoe_internal.cuh"

namespace lmoe {

constexpr int kMaxPairs = 8 * kMaxTopK;   // (token, k) pairs of at most 8 tokens

// Routing of the step in shared memory.
struct StreamShared {
    int hg[kMaxGroups];        // hit groups, ascending
    int n_hit;
    int n_unique;              // distinct experts
    int uexp[kMaxPairs];
    int ucnt[kMaxPairs];
    int uoff[kMaxPairs];
    int ugrp[kMaxPairs];       // group of each distinct expert
    int slot_tok[kMaxPairs];   // token of each slot (slots grouped by expert)
    float slot_w[kMaxPairs];   // routing weight of each slot
    // the routing itself (kernels that compute it rather than read it)
    int idx[kMaxPairs];        // [T][K] selected experts
    float w[kMaxPairs];        // [T][K] renormalised weights
    int pe[kMaxPairs];         // pair -> expert (validated)
    int pgrp[kMaxPairs];       // pair -> group
    int slot_pair[kMaxPairs];
    int pair_slot[kMaxPairs];
    int gcnt[kMaxGroups];      // pairs per group
    uint32_t emask[kMaxExpertsTopk / 32];  // experts selected by some pair
};

// ---------------------------------------------------------------------------
// routing inside one CTA, from the router logits in global memory
// ---------------------------------------------------------------------------

// Order-preserving map of a float onto an unsigned integer (larger float,
// larger key; -0 and +0 map to the same key), and back.
static __device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t b = __float_as_uint(f + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
static __device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

static __device__ __forceinline__ uint64_t pack_logit(float l, int e) {
    return ((uint64_t)order_key(l) << 32) | (uint32_t)~e;
}

// Softmax top-K of one token by one warp (the router of the model page's
// "Model profile": softmax over the E logits, top-K, renormalise over the
// kept).  A logit is packed as (order key, ~index), so the larger word is the
// larger logit and, between equal logits, the lower expert index; the words
// of a row are distinct.  Each lane holds NV words; K rounds each take the
// warp's largest word: the largest order key by a warp max reduction, then
// the lowest index among the lanes whose own largest word carries that key
// by a warp min reduction; the owning lane clears that word.  The rounds
// share one short loop body (this runs once per step, with its instructions
// fetched cold, so code size counts more than cycles).
//   w_k = exp(l_k - l_1) / sum over the kept of exp(l_j - l_1), summed in k
//   order.  Writes idx[0..K), w[0..K).
template <int NV>
static __device__ void topk_row(const float* logits, int E, int K, int lane, int* idx, float* w) {
    uint64_t pk[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int e = lane + 32 * j;
        pk[j] = e < E ? pack_logit(__ldcg(logits + e), e) : 0ull;
    }
    float l1 = 0.f, denom = 0.f, my_l = 0.f;
    int my_e = 0;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
        uint64_t m = pk[0];
#pragma unroll
        for (int j = 1; j < NV; ++j) m = pk[j] > m ? pk[j] : m;
        const uint32_t key = (uint32_t)(m >> 32);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        const uint32_t e = __reduce_min_sync(0xffffffffu, key == kmax ? ~(uint32_t)m : 0xffffffffu);
        if ((int)(e & 31) == lane) {
#pragma unroll
            for (int j = 0; j < NV; ++j)
                if (j == (int)(e >> 5)) pk[j] = 0ull;
        }
        const float l = key_value(kmax);
        if (k == 0) l1 = l;
        denom += expf(l - l1);
        if (k == lane) {
            my_l = l;
            my_e = (int)e;
        }
    }
    if (lane < K) {
        idx[lane] = my_e;
        w[lane] = expf(my_l - l1) / denom;
    }
}

// Bucketing of the T*K pairs by the whole CTA (one pair per thread), in
// shared memory: slots ordered by (expert, pair index), distinct experts
// ascending, pairs per group.  `grp` is the expert -> group table (in shared
// memory).  Invalid indices or labels are reported (report = true) and read
// as 0.  sh.emask and sh.n_unique must be zero on entry (and that ordered by
// a __syncthreads).  Contains __syncthreads.
static __device__ void bucket_pairs(const FwdParams& p, StreamShared& sh, const uint8_t* grp, bool report) {
    const int K = p.K, G = p.G, E = p.E, n = p.T * K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        int e = sh.idx[i];
        if (e < 0 || e >= E) {
            if (report) set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK);
            e = 0;
        }
        int g = grp[e];
        if (g >= G) {
            if (report) set_status(p.ctrl, LMOE_ERR_DEVICE_CHECK);
            g = 0;
        }
        sh.pe[i] = e;
        sh.pgrp[i] = g;
        atomicOr(&sh.emask[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        int c = 0;
        for (int i = 0; i < n; ++i) c += sh.pgrp[i] == g;
        sh.gcnt[g] = c;
    }
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int e = sh.pe[i];
        int less = 0, same_before = 0, cnt = 0;
#pragma unroll 2
        for (int j = 0; j < n; ++j) {
            const int ej = sh.pe[j];
            less += ej < e;
            same_before += (j < i) & (ej == e);
            cnt += ej == e;
        }
        // distinct experts below e
        int u = __popc(sh.emask[e >> 5] & ((1u << (e & 31)) - 1u));
        for (int v = 0; v < (e >> 5); ++v) u += __popc(sh.emask[v]);
        const int slot = less + same_before;
        sh.slot_pair[slot] = i;
        sh.pair_slot[i] = slot;
        sh.slot_tok[slot] = i / K;
        sh.slot_w[slot] = sh.w[i];
        if (same_before == 0) {
            sh.uexp[u] = e;
            sh.ucnt[u] = cnt;
            sh.uoff[u] = less;
            sh.ugrp[u] = sh.pgrp[i];
            atomicAdd(&sh.n_unique, 1);
        }
    }
    __syncthreads();
    // hit groups, ascending (warp 0, by ballots)
    if (warp == 0) {
        int base = 0;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            const bool hit = g < G && sh.gcnt[g] > 0;
            const uint32_t bal = __ballot_sync(0xffffffffu, hit);
            if (hit) sh.hg[base + __popc(bal & ((1u << lane) - 1u))] = g;
            base += __popc(bal);
        }
        if (lane == 0) sh.n_hit = base;
    }
    __syncthreads();
}

// The step's routing into `sh`, by every thread of the CTA (contains
// __syncthreads); `grp` is the expert -> group table in shared memory.
// With publish, also written to the workspace for the kernels that read it
// and to the caller's routing outputs.
static __device__ void route_in_cta(const FwdParams& p, StreamShared& sh, const uint8_t* grp, bool publish) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = p.T, K = p.K, E = p.E, G = p.G, n = T * K;
    for (int v = threadIdx.x; v < (E + 31) / 32; v += blockDim.x) sh.emask[v] = 0u;
    if (threadIdx.x == 0) sh.n_unique = 0;
    if (p.inject_idx != nullptr && p.inject_w != nullptr) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            sh.idx[i] = __ldg(p.inject_idx + i);
            sh.w[i] = __ldg(p.inject_w + i);
        }
    } else {
        for (int t = warp; t < T; t += blockDim.x >> 5) {
            const float* lg = p.r.logits + (size_t)t * E;
            int* ix = sh.idx + t * K;
            float* wt = sh.w + t * K;
            if (E <= 128) topk_row<4>(lg, E, K, lane, ix, wt);
            else if (E <= 256) topk_row<8>(lg, E, K, lane, ix, wt);
            else if (E <= 512) topk_row<16>(lg, E, K, lane, ix, wt);
            else topk_row<32>(lg, E, K, lane, ix, wt);
        }
    }
    __syncthreads();
    bucket_pairs(p, sh, grp, publish);
    if (!publish) return;
    const Routing& r = p.r;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        r.idx[i] = sh.pe[i];
        r.w[i] = sh.w[i];
        if (p.out_idx) p.out_idx[i] = sh.idx[i];
        if (p.out_w) p.out_w[i] = sh.w[i];
        r.slot_pair[i] = sh.slot_pair[i];
        r.pair_slot[i] = sh.pair_slot[i];
        r.slot_tok[i] = sh.slot_tok[i];
        r.slot_w[i] = sh.slot_w[i];
        r.pgrp[i] = sh.pgrp[i];
        if (i < sh.n_unique) {
            r.uexp[i] = sh.uexp[i];
            r.ucnt[i] = sh.ucnt[i];
            r.uoff[i] = sh.uoff[i];
            r.ugrp[i] = sh.ugrp[i];
        }
    }
    for (int i = threadIdx.x; i < T * G; i += blockDim.x) {
        const int t = i / G, g = i - t * G;
        uint8_t hit = 0;
        for (int k = 0; k < K; ++k) hit |= sh.pgrp[t * K + k] == g;
        r.tghit[i] = hit;
    }
    for (int g = threadIdx.x; g < G; g += blockDim.x) r.ghit[g] = sh.gcnt[g];
    if (threadIdx.x == 0) *r.n_unique = sh.n_unique;
}


}  // namespace lmoe
