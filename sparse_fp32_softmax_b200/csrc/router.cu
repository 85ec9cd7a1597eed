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
#include "select.cuh"

namespace moe {

// ------------------------------------------------------------------ small-T router logits
//
// One warp computes the logits of one expert for a group of up to 8 tokens: each lane walks
// the row of W_r in 16-byte pieces (8 bf16), 256 elements per step, and accumulates the
// exact bf16 products in FP32.  Used when T is small enough that the whole GEMM is a
// weight read (decode); larger T goes to the tcgen05 router GEMM.
__global__ void __launch_bounds__(256) router_small_kernel(const uint16_t* __restrict__ x,
                                                           const uint16_t* __restrict__ W_r,
                                                           int T, int D, int E,
                                                           float* __restrict__ logits) {
    pdl_wait();
    pdl_launch_dependents();
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
        if (lane < nt) logits[(size_t)(t0 + lane) * E + e] = mine;  // bias: added by the selection
    }
}

cudaError_t launch_router_small(const uint16_t* x, const uint16_t* W_r, int T, int D, int E,
                                float* logits, bool pdl, cudaStream_t s) {
    const long ntask = (long)E * ((T + 7) / 8);
    const int warps_per_block = 8;
    long blocks = (ntask + warps_per_block - 1) / warps_per_block;
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    if (blocks > sms * 16) blocks = sms * 16;
    return launch_kernel(router_small_kernel, dim3((int)blocks), dim3(warps_per_block * 32), 0, s, pdl,
                         x, W_r, T, D, E, logits);
}

// ------------------------------------------------------------------ softmax / top-k / renorm

// One warp per token over the router's partial sums in global memory.
template <int VPL>
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ part, int nsplit,
                                                     const float* __restrict__ bias, int T, int E,
                                                     int k, int norm, int32_t* __restrict__ idx,
                                                     float* __restrict__ w,
                                                     float* __restrict__ logits_out) {
    pdl_wait();
    pdl_launch_dependents();
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps)
        select_token<VPL>(part + (size_t)t * E, nsplit, (size_t)T * E, bias, E, k, norm,
                          idx + (size_t)t * k, w + (size_t)t * k,
                          logits_out ? logits_out + (size_t)t * E : nullptr);
}

cudaError_t launch_select(const float* part, int nsplit, const float* bias, int T, int E, int k,
                          int norm, int32_t* idx, float* w, float* logits_out, bool pdl,
                          cudaStream_t s) {
    const int threads = 256;
    int blocks = (T + 7) / 8;
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    if (blocks > sms * 32) blocks = sms * 32;
    if (blocks < 1) blocks = 1;
    void (*k_)(const float*, int, const float*, int, int, int, int, int32_t*, float*, float*) =
        E <= 32 ? select_kernel<1> : E <= 64 ? select_kernel<2> : E <= 128 ? select_kernel<4>
        : E <= 256 ? select_kernel<8> : select_kernel<16>;
    return launch_kernel(k_, dim3(blocks), dim3(threads), 0, s, pdl, part, nsplit, bias, T, E, k,
                         norm, idx, w, logits_out);
}

}  // namespace moe
