// select.cuh -- FP32 softmax, top-k with index tie-break and renormalisation for one token
// by one warp ("27. Mixture of experts", inference.shantanugoel.com, section "The router").
#pragma once

#include "common.cuh"

namespace moe {

// Order-preserving map of an FP32 bit pattern to an unsigned key (larger float -> larger key).
__device__ __forceinline__ uint32_t float_order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_from_order_key(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Selection for one token by one warp.  The token's logits are the sum of nsplit partial
// rows (part + s*split_stride, added in split order) plus the bias when given; lane L holds
// experts L, L+32, ...  and writes them to logits_out when given.  Experts are ranked by the
// order-preserving key of their logit; among equal keys the lower index wins: each round,
// one warp-wide max over the keys, then one over the complemented indices of the lanes
// holding that key.
// L2_LOADS: the partial rows were written by other blocks of the running kernel, so they
// are read through L2 (ld.global.cg); otherwise with generic loads (shared memory, or
// global memory written by an earlier kernel).
template <int VPL, bool L2_LOADS = false>
__device__ __forceinline__ void select_token(const float* part, int nsplit, size_t split_stride,
                                             const float* bias, int E, int k, int norm,
                                             int32_t* idx_out, float* w_out, float* logits_out) {
    const int lane = threadIdx.x & 31;
    float v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? (L2_LOADS ? __ldcg(part + e) : part[e]) : 0.f;
    }
#pragma unroll
    for (int sp = 1; sp < kRouterMaxSplit; ++sp) {  // loads of all partials in flight together
        if (sp < nsplit) {
            float q[VPL];
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int e = lane + 32 * i;
                q[i] = e < E ? part[(size_t)sp * split_stride + e] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i) v[i] += q[i];  // split order
        }
    }
    uint32_t key[VPL];
    uint32_t kmax = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            if (bias) v[i] = v[i] + __ldg(bias + e);
            if (logits_out) logits_out[e] = v[i];
            v[i] = v[i] + 0.0f;  // -0.0 + 0.0 = +0.0: the two zeros compare and key equal
            key[i] = float_order_key(v[i]);
            kmax = key[i] > kmax ? key[i] : kmax;
        } else {
            key[i] = 0u;  // below every finite logit's key
        }
    }
    const float m = float_from_order_key(__reduce_max_sync(0xffffffffu, kmax));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i < E) s += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

    int my_e = 0;
    float my_l = 0.f;
    for (int j = 0; j < k; ++j) {
        uint32_t bk = 0;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            if (key[i] > bk) {  // strict: the lane's lowest index among equal keys
                bk = key[i];
                bi = i;
            }
        const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t cand = (bk == mk && bk != 0u) ? 0xFFFFFFFFu - (uint32_t)(lane + 32 * bi) : 0u;
        const int e = (int)(0xFFFFFFFFu - __reduce_max_sync(0xffffffffu, cand));
        if ((e & 31) == lane) {
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (i == (e >> 5)) key[i] = 0u;
        }
        if (lane == j) {
            my_e = e;
            my_l = float_from_order_key(mk);
        }
    }
    const float p = (lane < k) ? expf(my_l - m) / s : 0.f;  // FP32 softmax probability
    float out = p;
    if (norm) {
        float tot = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        out = p / tot;
    }
    if (lane < k) {
        idx_out[lane] = my_e;
        w_out[lane] = out;
    }
}

}  // namespace moe
