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
// One block of 8 warps computes the logits of one expert for a group of up to 8 tokens; the
// warps split the row of W_r into 8 consecutive slices.  In its slice, lane L takes the
// 16-byte pieces (8 bf16) L, L+32, ... and accumulates the exact bf16 products in FP32 in
// order; a butterfly adds the lanes, and warp 0 adds the 8 slices in slice order.  Every
// weight load of the block is in flight at once, and the E x ceil(T/8) blocks spread the
// router's bytes over the SMs, so at decode sizes the logits cost about one memory round
// trip.  Used for T <= 64; larger T goes to the tcgen05 router GEMM.
constexpr int kRsWarps = 8;
__global__ void __launch_bounds__(kRsWarps * 32) router_small_kernel(const uint16_t* __restrict__ x,
                                                                   const uint16_t* __restrict__ W_r,
                                                                   int T, int D, int E,
                                                                   float* __restrict__ logits) {
    __shared__ float part[kRsWarps][8];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ngroups = (T + 7) >> 3;
    const int e = blockIdx.x / ngroups;
    const int t0 = (blockIdx.x % ngroups) * 8;
    const int nt = min(8, T - t0);
    const int slice = D / kRsWarps;              // a multiple of 16 elements (D % 128 == 0)
    const int c0 = warp * slice, c1 = c0 + slice;
    const uint16_t* wr = W_r + (size_t)e * D;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int c = c0 + lane * 8; c < c1; c += 256) {
        const uint4 w = ld_v4(wr + c);
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < nt) v[i] = ld_v4(x + (size_t)(t0 + i) * D + c);
        const float w0 = bf16_lo(w.x), w1 = bf16_hi(w.x), w2 = bf16_lo(w.y), w3 = bf16_hi(w.y);
        const float w4 = bf16_lo(w.z), w5 = bf16_hi(w.z), w6 = bf16_lo(w.w), w7 = bf16_hi(w.w);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < nt) {
                float q = acc[i];
                q = fmaf(w0, bf16_lo(v[i].x), q);
                q = fmaf(w1, bf16_hi(v[i].x), q);
                q = fmaf(w2, bf16_lo(v[i].y), q);
                q = fmaf(w3, bf16_hi(v[i].y), q);
                q = fmaf(w4, bf16_lo(v[i].z), q);
                q = fmaf(w5, bf16_hi(v[i].z), q);
                q = fmaf(w6, bf16_lo(v[i].w), q);
                q = fmaf(w7, bf16_hi(v[i].w), q);
                acc[i] = q;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float q = acc[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        if (lane == 0) part[warp][i] = q;
    }
    __syncthreads();
    if (warp == 0 && lane < nt) {
        float l = part[0][lane];
#pragma unroll
        for (int w = 1; w < kRsWarps; ++w) l += part[w][lane];   // slice order
        logits[(size_t)(t0 + lane) * E + e] = l;                  // bias: added by the selection
    }
}

cudaError_t launch_router_small(const uint16_t* x, const uint16_t* W_r, int T, int D, int E,
                                float* logits, bool pdl, cudaStream_t s) {
    if (D % (kRsWarps * 16) != 0) return cudaErrorInvalidValue;
    const long blocks = (long)E * ((T + 7) / 8);
    return launch_kernel(router_small_kernel, dim3((unsigned)blocks), dim3(kRsWarps * 32), 0, s, pdl,
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
