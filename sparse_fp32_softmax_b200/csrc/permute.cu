// permute.cu -- expert-contiguous layout of the T*k routing assignments.
//
// "27. Mixture of experts" (inference.shantanugoel.com), section "Dispatch", grouped
// dispatch: flatten the N*k assignments, sort them by expert with a stable sort so each
// expert's rows are contiguous, count them per expert (bincount), and permute the token rows
// into that order.  Here the stable sort is a counting sort on the GPU:
//   1. per-chunk histograms (shared-memory atomics: counts do not depend on order);
//   2. per-expert totals, tile-padded offsets and, for every (chunk, expert), the first row
//      that chunk may write; also the work tables the expert kernels schedule from;
//   3. each chunk ranks its assignments stably (warp match + popcount, warps in order) and
//      writes row_token / row_weight / row_dest / slot_row;
//   4. (when the expert kernels read a permuted copy) a gather copies x rows into order.
// When all assignments fit one chunk (T*k <= 4096, the decode sizes) steps 1-3 run as one
// single-block kernel.  Within an expert, rows keep increasing assignment order
// a = t*k + j (the stable argsort).
#include "permute_block.cuh"

namespace moe {

__global__ void __launch_bounds__(kPermThreads) perm_fused_kernel(PermuteArgs a) {
    extern __shared__ int wb[];  // [32][E]
    pdl_wait();
    pdl_launch_dependents();
    permute_one_block(a, wb, load_warp_slice(a, 0));
}

// ------------------------------------------------------------------ multi-block path

// 1. histogram of one chunk of assignments
__global__ void __launch_bounds__(kPermThreads) perm_hist_kernel(PermuteArgs a) {
    extern __shared__ int cnt[];
    pdl_wait();
    pdl_launch_dependents();
    const int E = a.E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const long n = (long)a.T * a.k;
    const long a0 = (long)blockIdx.x * kPermChunk;
    const long a1 = min(n, a0 + kPermChunk);
    for (long as = a0 + threadIdx.x; as < a1; as += blockDim.x) {
        const int e = a.topk_idx[as];
        if (e < 0 || e >= E)
            set_error(a.err, kErrBadIndex);
        else
            atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) a.chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// 2. totals, offsets, chunk bases and work tables (one block of 1024 threads)
__global__ void __launch_bounds__(kPermThreads) perm_scan_kernel(PermuteArgs a) {
    __shared__ int s_cnt[kMaxSegments];
    __shared__ int s_off[kMaxSegments + 1];
    pdl_wait();
    pdl_launch_dependents();
    const int E = a.E;
    // per-expert totals; chunk_counts becomes the exclusive prefix over chunks (relative)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int c = 0; c < a.nchunks; ++c) {
            const int v = a.chunk_counts[(size_t)c * E + e];
            a.chunk_counts[(size_t)c * E + e] = run;
            run += v;
        }
        s_cnt[e] = run;
    }
    __syncthreads();
    finish_offsets(a, s_cnt, s_off);
    for (int q = threadIdx.x; q < a.nchunks * E; q += blockDim.x)
        a.chunk_counts[q] += s_off[q % E];
}

// 3. stable scatter of one chunk per block
__global__ void __launch_bounds__(kPermThreads, 1) perm_scatter_kernel(PermuteArgs a) {
    extern __shared__ int wb[];  // [32][E]: per-warp counts, then per-warp running row bases
    pdl_wait();
    pdl_launch_dependents();
    const int E = a.E;
    if (blockIdx.x < a.nchunks) {
        const WarpSlice ws = load_warp_slice(a, (long)blockIdx.x * kPermChunk);
        for (int q = threadIdx.x; q < 32 * E; q += blockDim.x) wb[q] = 0;
        __syncthreads();
        count_warp_slices(a, ws, wb);
        __syncthreads();
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            int run = a.chunk_counts[(size_t)blockIdx.x * E + e];
            for (int w = 0; w < 32; ++w) {
                const int v = wb[w * E + e];
                wb[w * E + e] = run;
                run += v;
            }
        }
        __syncthreads();
        scatter_warp_slices(a, ws, wb);
    }
    write_fixed_rows(a, __ldg(a.offsets + E), a.offsets, a.counts, blockIdx.x, gridDim.x);
}

cudaError_t launch_permute(const PermuteArgs& a, bool pdl, cudaStream_t s) {
    const size_t wb_bytes = 32 * (size_t)a.E * sizeof(int);
    if (a.nchunks == 1) {
        cudaError_t err = ensure_smem_attr((const void*)perm_fused_kernel,
                                           32 * kMaxSegments * (int)sizeof(int));
        if (err != cudaSuccess) return err;
        return launch_kernel(perm_fused_kernel, dim3(1), dim3(kPermThreads), wb_bytes, s, pdl, a);
    }
    cudaError_t err = ensure_smem_attr((const void*)perm_scatter_kernel,
                                       32 * kMaxSegments * (int)sizeof(int));
    if (err != cudaSuccess) return err;
    err = launch_kernel(perm_hist_kernel, dim3(a.nchunks), dim3(kPermThreads), a.E * sizeof(int), s,
                        pdl, a);
    if (err != cudaSuccess) return err;
    err = launch_kernel(perm_scan_kernel, dim3(1), dim3(kPermThreads), 0, s, true, a);
    if (err != cudaSuccess) return err;
    int blocks = a.nchunks;
    if (a.has_shared && blocks < (a.T + kPermThreads - 1) / kPermThreads)
        blocks = (a.T + kPermThreads - 1) / kPermThreads;
    return launch_kernel(perm_scatter_kernel, dim3(blocks), dim3(kPermThreads), wb_bytes, s, true, a);
}

// 4. x rows into permuted order: one warp per row, 16-byte pieces.  Rows with
// row_token < 0 (padding) are zero-filled.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ row_token,
                                                          int rows, int D,
                                                          uint16_t* __restrict__ x_perm) {
    // gate_up (next) may launch now: it issues its speculative weight prefetch while the
    // routing finishes, and waits for this kernel itself
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int vec = D >> 3;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nw) {
        const int t = __ldg(row_token + r);
        uint4* dst = reinterpret_cast<uint4*>(x_perm + (size_t)r * D);
        if (t >= 0) {
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * D);
            for (int i = lane; i < vec; i += 32) dst[i] = __ldg(src + i);
        } else {
            for (int i = lane; i < vec; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* row_token, int rows, int D,
                               uint16_t* x_perm, bool pdl, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    int blocks = (rows + 7) / 8;
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    if (blocks > sms * 8) blocks = sms * 8;
    return launch_kernel(gather_rows_kernel, dim3(blocks), dim3(256), 0, s, pdl, x, row_token, rows,
                         D, x_perm);
}

}  // namespace moe
