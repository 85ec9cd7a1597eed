// route_fused.cu -- routing of small batches in few launches.
//
// "27. Mixture of experts" (inference.shantanugoel.com): section "The router" (logits,
// FP32 softmax over all experts, top-k with ties to the lower index, renormalisation) and
// section "Dispatch" (stable grouping of the assignments by expert).  At decode sizes each
// of these steps is a few microseconds of work, so launching them separately costs more
// than running them: for T <= 32 one kernel does all of them; above, while T*k fits one
// permutation block, one kernel selects and permutes after the router GEMM.
#include "permute_block.cuh"
#include "select.cuh"

namespace moe {

// ------------------------------------------------------------------ fused small-T routing
//
// Blocks split the experts: block b computes the FP32 logits of its experts for every token
// (T <= 32), one warp per (expert, token) pair, with the same exact-product FP32
// accumulation as the small-T router.  Logits go to global memory; each block then takes an
// atomic ticket after a fence, and the block that draws the last ticket sees every block's
// logits (read through L2): it selects all tokens (one warp per token) and performs the whole
// permutation.
// One launch replaces the router, the selection and the permutation kernels.
template <int VPL>
__global__ void __launch_bounds__(1024) route_fused_kernel(RouteArgs a) {
    extern __shared__ int route_smem[];
    int* wb = route_smem;                                               // [32][E] (last block)
    __shared__ int s_ticket;
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E, D = a.D, T = a.T;
    const int per_block = (E + gridDim.x - 1) / gridDim.x;
    const int e0 = blockIdx.x * per_block;
    const int e1 = min(E, e0 + per_block);
    const int npairs = max(0, e1 - e0) * T;
    for (int q = warp; q < npairs; q += 32) {
        const int e = e0 + q / T, t = q % T;
        const uint16_t* wr = a.W_r + (size_t)e * D;
        const uint16_t* xr = a.x + (size_t)t * D;
        float acc = 0.f;
#pragma unroll 8
        for (int c = lane * 8; c < D; c += 256) {
            const uint4 wv = ld_v4(wr + c);
            const uint4 v = ld_v4(xr + c);
            acc = fmaf(bf16_lo(wv.x), bf16_lo(v.x), acc);
            acc = fmaf(bf16_hi(wv.x), bf16_hi(v.x), acc);
            acc = fmaf(bf16_lo(wv.y), bf16_lo(v.y), acc);
            acc = fmaf(bf16_hi(wv.y), bf16_hi(v.y), acc);
            acc = fmaf(bf16_lo(wv.z), bf16_lo(v.z), acc);
            acc = fmaf(bf16_hi(wv.z), bf16_hi(v.z), acc);
            acc = fmaf(bf16_lo(wv.w), bf16_lo(v.w), acc);
            acc = fmaf(bf16_hi(wv.w), bf16_hi(v.w), acc);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            float l = acc;
            if (a.bias) l = l + a.bias[e];
            a.logits_out[(size_t)t * E + e] = l;
        }
    }
    // publish this block's logits; the last block routes and permutes everything
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(a.ticket, 1);
    __syncthreads();
    if (s_ticket != (int)gridDim.x - 1) return;
    __threadfence();
    for (int t = warp; t < T; t += 32)
        select_token<VPL, true>(a.logits_out + (size_t)t * E, 1, 0, nullptr, E, a.k, a.norm,
                                a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k, nullptr);
    __syncthreads();
    permute_one_block(a.perm, wb);
}

cudaError_t launch_route_fused(const RouteArgs& a, bool pdl, cudaStream_t s) {
    if (a.T > kFusedRouteMaxT) return cudaErrorInvalidValue;
    const int smem = 32 * a.E * 4;
    void (*k_)(RouteArgs) = a.E <= 32 ? route_fused_kernel<1> : a.E <= 64 ? route_fused_kernel<2>
                          : a.E <= 128 ? route_fused_kernel<4> : a.E <= 256 ? route_fused_kernel<8>
                          : route_fused_kernel<16>;
    cudaError_t err = ensure_smem_attr((const void*)k_, 32 * kMaxE * 4);
    if (err != cudaSuccess) return err;
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const int blocks = a.E < sms ? a.E : sms;
    return launch_kernel(k_, dim3(blocks), dim3(1024), smem, s, pdl, a);
}

// ------------------------------------------------------------------ selection + permutation
//
// For T*k <= 4096 above the fused-routing sizes: the router GEMM has left partial logit sums;
// each block selects 32 tokens (one warp per token: sum of the partials in split order, bias,
// FP32 softmax, top-k, renormalisation), then takes an atomic ticket after a fence, and the
// block that draws the last ticket performs the whole permutation.
template <int VPL>
__global__ void __launch_bounds__(1024) select_permute_kernel(RouteArgs a) {
    extern __shared__ int sp_smem[];   // [32][E] (last block)
    __shared__ int s_ticket;
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * 32 + warp;
    const int E = a.E;
    if (t < a.T)
        select_token<VPL>(a.part + (size_t)t * E, a.nsplit, (size_t)a.T * E, a.bias, E, a.k, a.norm,
                          a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k,
                          a.logits_out ? a.logits_out + (size_t)t * E : nullptr);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(a.ticket, 1);
    __syncthreads();
    if (s_ticket != (int)gridDim.x - 1) return;
    __threadfence();
    permute_one_block(a.perm, sp_smem);
}

cudaError_t launch_select_permute(const RouteArgs& a, bool pdl, cudaStream_t s) {
    if ((long long)a.T * a.k > kPermChunk) return cudaErrorInvalidValue;
    const int smem = 32 * a.E * 4;
    void (*k_)(RouteArgs) = a.E <= 32 ? select_permute_kernel<1> : a.E <= 64 ? select_permute_kernel<2>
                          : a.E <= 128 ? select_permute_kernel<4> : a.E <= 256 ? select_permute_kernel<8>
                          : select_permute_kernel<16>;
    cudaError_t err = ensure_smem_attr((const void*)k_, 32 * kMaxE * 4);
    if (err != cudaSuccess) return err;
    return launch_kernel(k_, dim3((a.T + 31) / 32), dim3(1024), smem, s, pdl, a);
}

}  // namespace moe
