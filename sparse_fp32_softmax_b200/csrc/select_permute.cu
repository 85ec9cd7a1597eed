// select_permute.cu -- selection and permutation of small batches in one launch.
//
// "27. Mixture of experts" (inference.shantanugoel.com): section "The router" (FP32 softmax
// over all experts, top-k with ties to the lower index, renormalisation) and section
// "Dispatch" (stable grouping of the assignments by expert).  At decode sizes each of these
// steps is a few microseconds of work, so launching them separately costs more than running
// them: while T*k fits one permutation block, one kernel selects and permutes after the
// router logits.
#include "permute_block.cuh"
#include "select.cuh"

namespace moe {

// ------------------------------------------------------------------ selection + permutation
//
// For T*k <= 4096: the router has left its partial logit sums;
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
    permute_one_block(a.perm, sp_smem, load_warp_slice<false>(a.perm, 0));
}

// T <= 32: one block selects every token into shared memory, writes the routing outputs and
// permutes at once (no ticket, and no round trip of the selection through global memory).
template <int VPL>
__global__ void __launch_bounds__(1024) select_permute_one_kernel(RouteArgs a) {
    extern __shared__ int sp_smem[];   // [32][E]
    __shared__ int s_idx[32 * kMaxK];
    __shared__ float s_w[32 * kMaxK];
    pdl_wait();
    pdl_launch_dependents();
    const int t = threadIdx.x >> 5;
    const int E = a.E;
    if (t < a.T)
        select_token<VPL>(a.part + (size_t)t * E, a.nsplit, (size_t)a.T * E, a.bias, E, a.k, a.norm,
                          s_idx + t * a.k, s_w + t * a.k,
                          a.logits_out ? a.logits_out + (size_t)t * E : nullptr);
    __syncthreads();
    for (int i = threadIdx.x; i < a.T * a.k; i += blockDim.x) {
        a.topk_idx[i] = s_idx[i];
        a.topk_w[i] = s_w[i];
    }
    permute_one_block(a.perm, sp_smem, load_warp_slice<true>(a.perm, 0, s_idx, s_w));
}

cudaError_t launch_select_permute(const RouteArgs& a, bool pdl, cudaStream_t s) {
    if ((long long)a.T * a.k > kPermChunk) return cudaErrorInvalidValue;
    const int smem = 32 * a.E * 4;
    void (*k_)(RouteArgs);
    if (a.T <= 32)
        k_ = a.E <= 32 ? select_permute_one_kernel<1> : a.E <= 64 ? select_permute_one_kernel<2>
           : a.E <= 128 ? select_permute_one_kernel<4> : a.E <= 256 ? select_permute_one_kernel<8>
           : select_permute_one_kernel<16>;
    else
        k_ = a.E <= 32 ? select_permute_kernel<1> : a.E <= 64 ? select_permute_kernel<2>
           : a.E <= 128 ? select_permute_kernel<4> : a.E <= 256 ? select_permute_kernel<8>
           : select_permute_kernel<16>;
    cudaError_t err = ensure_smem_attr((const void*)k_, 32 * kMaxE * 4);
    if (err != cudaSuccess) return err;
    return launch_kernel(k_, dim3((a.T + 31) / 32), dim3(1024), smem, s, pdl, a);
}

}  // namespace moe
