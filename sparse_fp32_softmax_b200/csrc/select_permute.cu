// select_permute.cu -- selection and permutation of mid-sized batches in one launch.
//
// "27. Mixture of experts" (inference.shantanugoel.com): section "The router" (FP32
// softmax over all experts, top-k with ties to the lower index, renormalisation) and
// section "Dispatch" (stable grouping of the assignments by expert).  While T*k fits one
// permutation block each of these steps is a few microseconds of work, so one kernel
// selects every token and permutes after the router GEMM instead of two launches.
#include "permute_block.cuh"
#include "select.cuh"

namespace moe {

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
    if (t < a.T) {
        select_token<VPL>(a.part + (size_t)t * E, a.nsplit, (size_t)a.T * E, a.bias, E, a.k, a.norm,
                          a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k,
                          a.logits_out ? a.logits_out + (size_t)t * E : nullptr);
        if (a.gates) {
            const float g = shared_gate_value(a.x + (size_t)t * a.D, a.shared_gate, a.D);
            if ((threadIdx.x & 31) == 0) a.gates[t] = g;
        }
    }
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
