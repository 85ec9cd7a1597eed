// router.cu -- router logits for small token counts, and the FP32 softmax / top-k / renorm.
//
// "27. Mixture of experts" (inference.shantanugoel.com), section "The router": the router is
// one linear layer x -> E scores; Qwen-family models take a softmax over all experts in
// FP32, keep the k largest probabilities with their indices (ties broken by index), and with
// norm_topk_prob divide the kept weights by their sum.
//
// Reading taken here: experts are ranked by their FP32 logit (the softmax is strictly
// increasing, so this is the same set as ranking probabilities, and ties made only by the
// rounding of exp cannot arise); equal logits rank the lower expert index first, and -0.0
// equals +0.0.  Weights are FP32.
#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------ small-T router logits
//
// One warp computes the logits of one expert for a group of up to 8 tokens: each lane walks
// the row of W_r in 16-byte pieces (8 bf16), 256 elements per step, and accumulates the
// exact bf16 products in FP32.  Used when T is small enough that the whole GEMM is a
// weight read (decode); larger T goes to the tcgen05 router GEMM.
__global__ void __launch_bounds__(256) router_small_kernel(const uint16_t* __restrict__ x,
                                                           const uint16_t* __restrict__ W_r,
                                                           const float* __restrict__ bias,
                                                           int T, int D, int E,
                                                           float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int ngroups = (T + 7) >> 3;
    const long ntask = (long)E * ngroups;
    const long nwarps = ((long)gridDim.x * blockDim.x) >> 5;
    for (long task = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; task < ntask;
         task += nwarps) {
        const int e = (int)(task / ngroups);
        const int t0 = (int)(task % ngroups) * 8;
        const int nt = min(8, T - t0);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        const uint16_t* wr = W_r + (size_t)e * D;
        for (int c = lane * 8; c < D; c += 256) {
            const uint4 w = ld_v4(wr + c);
            const float w0 = bf16_lo(w.x), w1 = bf16_hi(w.x), w2 = bf16_lo(w.y), w3 = bf16_hi(w.y);
            const float w4 = bf16_lo(w.z), w5 = bf16_hi(w.z), w6 = bf16_lo(w.w), w7 = bf16_hi(w.w);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < nt) {
                    const uint4 v = ld_v4(x + (size_t)(t0 + i) * D + c);
                    float a = acc[i];
                    a = fmaf(w0, bf16_lo(v.x), a);
                    a = fmaf(w1, bf16_hi(v.x), a);
                    a = fmaf(w2, bf16_lo(v.y), a);
                    a = fmaf(w3, bf16_hi(v.y), a);
                    a = fmaf(w4, bf16_lo(v.z), a);
                    a = fmaf(w5, bf16_hi(v.z), a);
                    a = fmaf(w6, bf16_lo(v.w), a);
                    a = fmaf(w7, bf16_hi(v.w), a);
                    acc[i] = a;
                }
            }
        }
        float mine = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float a = acc[i];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (lane == i) mine = a;
        }
        if (lane < nt) {
            float l = mine;
            if (bias) l = l + bias[e];
            logits[(size_t)(t0 + lane) * E + e] = l;
        }
    }
}

cudaError_t launch_router_small(const uint16_t* x, const uint16_t* W_r, const float* bias, int T,
                                int D, int E, float* logits, cudaStream_t s) {
    const long ntask = (long)E * ((T + 7) / 8);
    const int warps_per_block = 8;
    long blocks = (ntask + warps_per_block - 1) / warps_per_block;
    if (blocks > 148 * 16) blocks = 148 * 16;
    router_small_kernel<<<(int)blocks, warps_per_block * 32, 0, s>>>(x, W_r, bias, T, D, E, logits);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ softmax / top-k / renorm

// Order-preserving map of an FP32 bit pattern to an unsigned key (larger float -> larger key).
__device__ __forceinline__ uint32_t float_order_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_from_order_key(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// One warp per token.  Lane L holds experts L, L+32, ...  Keys pack (logit order, ~index)
// into 64 bits so a single unsigned max picks the higher logit and, on equal logits, the
// lower index.
template <int VPL>
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ logits, int T, int E,
                                                     int k, int norm, int32_t* __restrict__ idx,
                                                     float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* row = logits + (size_t)t * E;
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
            idx[(size_t)t * k + lane] = my_e;
            w[(size_t)t * k + lane] = out;
        }
    }
}

cudaError_t launch_select(const float* logits, int T, int E, int k, int norm, int32_t* idx,
                          float* w, cudaStream_t s) {
    const int threads = 256;
    int blocks = (T + 7) / 8;
    if (blocks > 148 * 32) blocks = 148 * 32;
    if (blocks < 1) blocks = 1;
    if (E <= 32)
        select_kernel<1><<<blocks, threads, 0, s>>>(logits, T, E, k, norm, idx, w);
    else if (E <= 64)
        select_kernel<2><<<blocks, threads, 0, s>>>(logits, T, E, k, norm, idx, w);
    else if (E <= 128)
        select_kernel<4><<<blocks, threads, 0, s>>>(logits, T, E, k, norm, idx, w);
    else if (E <= 256)
        select_kernel<8><<<blocks, threads, 0, s>>>(logits, T, E, k, norm, idx, w);
    else
        select_kernel<16><<<blocks, threads, 0, s>>>(logits, T, E, k, norm, idx, w);
    return cudaGetLastError();
}

}  // namespace moe
