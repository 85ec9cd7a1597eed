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

// Selection for one token by one warp.  Lane L holds experts L, L+32, ...  Keys pack (logit
// order, ~index) into 64 bits so a single unsigned max picks the higher logit and, on equal
// logits, the lower index.
template <int VPL>
__device__ __forceinline__ void select_token(const float* row, int E, int k, int norm,
                                             int32_t* idx_out, float* w_out) {
    const int lane = threadIdx.x & 31;
    float v[VPL];
    uint32_t alive = 0;
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            v[i] = row[e] + 0.0f;  // -0.0 + 0.0 = +0.0: the two zeros compare and key equal
            alive |= 1u << i;
            m = fmaxf(m, v[i]);
        } else {
            v[i] = -INFINITY;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
        if (alive & (1u << i)) s += expf(v[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

    int my_e = 0;
    float my_l = 0.f;
    for (int j = 0; j < k; ++j) {
        unsigned long long best = 0ull;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            if (alive & (1u << i)) {
                const unsigned long long key =
                    ((unsigned long long)float_order_key(v[i]) << 32) |
                    (unsigned long long)(0xFFFFFFFFu - (uint32_t)(lane + 32 * i));
                best = key > best ? key : best;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        const int e = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
        if ((e & 31) == lane) alive &= ~(1u << (e >> 5));
        if (lane == j) {
            my_e = e;
            my_l = float_from_order_key((uint32_t)(best >> 32));
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
