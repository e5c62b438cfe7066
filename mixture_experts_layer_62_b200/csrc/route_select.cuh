// Per-token selection of the small-batch router ("Week 2 Day 2: Mixture of
// Experts" §1.3 and §4.2): the logit row as the sum of the router's partial
// logits in part order, the softmax over all experts, the selection key of
// the bias mode, k rounds of a warp arg-max in which the lowest index wins
// ties, and the rank of a pair inside its expert. Kept apart from the kernel
// so that any other kernel that has to reproduce the router's decisions bit
// for bit runs the same code.
#pragma once

#include "common.cuh"

namespace moe {
namespace small {

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// z[t][e] = sum over parts, in part order, of the partial logits [T][P][E]
// (read through L2: the producer is an earlier kernel)
__device__ __forceinline__ float sum_partials(const float* probs, int t, int P, int E, int e) {
    float pv[kSmallMaxParts];
#pragma unroll
    for (int part = 0; part < kSmallMaxParts; ++part)
        pv[part] = part < P ? __ldcg(probs + ((size_t)t * P + part) * E + e) : 0.f;
    float v = 0.f;
#pragma unroll
    for (int part = 0; part < kSmallMaxParts; ++part)
        if (part < P) v += pv[part];
    return v;
}

// One token's logits held by a warp: lane l has experts l and l + 32 (E <= 64).
struct TokenSoftmax {
    float zz[2], ex[2];   // logits, exp(z - m) (0 for e >= E)
    float m, s, inv_s;    // max, sum of ex, 1 / s
    unsigned valid;       // bit i: expert lane + 32 i exists
};

__device__ __forceinline__ TokenSoftmax token_softmax(float z0, float z1, int E, int lane) {
    TokenSoftmax r;
    r.valid = 0;
    const float zin[2] = {z0, z1};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int e = lane + 32 * i;
        r.zz[i] = e < E ? zin[i] : -INFINITY;
        if (e < E) r.valid |= 1u << i;
    }
    r.m = warp_max(fmaxf(r.zz[0], r.zz[1]));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        r.ex[i] = ((r.valid >> i) & 1u) ? expf(r.zz[i] - r.m) : 0.f;
        s += r.ex[i];
    }
    r.s = warp_sum(s);
    r.inv_s = 1.f / r.s;
    return r;
}

// Probability of expert lane + 32 i.
__device__ __forceinline__ float token_prob(const TokenSoftmax& ts, int i) { return ts.ex[i] * ts.inv_s; }

// The k selected experts, in descending key order: lane 0 writes slot j's
// expert to esel[j] and its raw logit to zsel[j].
__device__ __forceinline__ void token_topk(const TokenSoftmax& ts, const float* bias_s, int bias_mode, int E, int k,
                                           int lane, float* zsel, int* esel) {
    float key[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int e = lane + 32 * i;
        const float p = token_prob(ts, i);
        const float b = e < E ? bias_s[e] : 0.f;
        key[i] = bias_mode == MOE_BIAS_NONE ? ts.zz[i] : bias_mode == MOE_BIAS_LOGIT ? ts.zz[i] + b : p + b;
    }
    unsigned taken = 0;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        float bk = -INFINITY, bz = 0.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const bool ok = ((ts.valid >> i) & 1u) && !((taken >> i) & 1u);
            if (ok && (key[i] > bk || be == 0x7fffffff)) { bk = key[i]; be = lane + 32 * i; bz = ts.zz[i]; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ok_ = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
            const bool better = (oe != 0x7fffffff) && (be == 0x7fffffff || ok_ > bk || (ok_ == bk && oe < be));
            if (better) { bk = ok_; be = oe; bz = oz; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == 0) {
            zsel[j] = bz;
            esel[j] = be;
        }
    }
}

// Rank of pair i = t k + j among the pairs of its expert e = sidx[i]: earlier
// tokens (token order), or earlier slots of every token and then this slot of
// earlier tokens (slot priority).
__device__ __forceinline__ int pair_rank(const int* sidx, int i, int T, int k, bool drop_slot) {
    const int t = i / k, j = i % k, e = sidx[i];
    int rank = 0;
    if (drop_slot) {
        for (int q = 0; q < T * k; ++q) {
            const int tq = q / k, jq = q % k;
            rank += (sidx[q] == e) && (jq < j || (jq == j && tq < t));
        }
    } else {
        for (int q = 0; q < t * k; ++q) rank += (sidx[q] == e);
    }
    return rank;
}

}  // namespace small
}  // namespace moe
