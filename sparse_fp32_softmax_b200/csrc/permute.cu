// permute.cu -- expert-contiguous layout of the T*k routing assignments.
//
// "27. Mixture of experts" (inference.shantanugoel.com), section "Dispatch", grouped
// dispatch: flatten the N*k assignments, sort them by expert with a stable sort so each
// expert's rows are contiguous, count them per expert (bincount), and permute the token rows
// into that order.  Here the stable sort is a counting sort on the GPU:
//   1. per-chunk histograms (shared-memory atomics: counts do not depend on order);
//   2. one block turns them into per-expert totals, tile-padded offsets and, for every
//      (chunk, expert), the first row that chunk may write; it also writes the work tables
//      the expert kernels schedule from;
//   3. each chunk ranks its assignments stably (warp match + popcount, warps in order) and
//      writes row_token / row_weight / row_dest / slot_row;
//   4. (grouped path only) a gather copies x rows into the permuted buffer.
// Within an expert, rows keep increasing assignment order a = t*k + j (the stable argsort).
#include "common.cuh"

namespace moe {

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024, multiple of 32).
// Returns the exclusive prefix; *total receives the sum.  Contains __syncthreads.
__device__ int block_exclusive_scan(int v, int* total) {
    __shared__ int warp_sums[32];
    __shared__ int s_total;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? warp_sums[lane] : 0;
        int winc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, winc, o);
            if (lane >= o) winc += y;
        }
        if (lane < nwarps) warp_sums[lane] = winc - w;  // exclusive warp offsets
        if (lane == 31) s_total = winc;                 // grand total
    }
    __syncthreads();
    const int res = warp_sums[warp] + inc - v;
    const int tot = s_total;
    __syncthreads();
    if (total) *total = tot;
    return res;
}

// 1. histogram of one chunk of assignments
__global__ void __launch_bounds__(kPermThreads) perm_hist_kernel(const int32_t* __restrict__ idx,
                                                                 long n, int E,
                                                                 int* __restrict__ chunk_counts,
                                                                 int* err) {
    extern __shared__ int cnt[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const long a0 = (long)blockIdx.x * kPermChunk;
    const long a1 = min(n, a0 + kPermChunk);
    for (long a = a0 + threadIdx.x; a < a1; a += blockDim.x) {
        const int e = idx[a];
        if (e < 0 || e >= E)
            set_error(err, kErrBadIndex);
        else
            atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// 2. totals, tile-padded offsets, chunk bases and work tables (one block of 1024 threads)
__global__ void __launch_bounds__(kPermThreads) perm_scan_kernel(PermuteArgs a) {
    const int E = a.E;
    const int nseg = E + (a.has_shared ? 1 : 0);
    __shared__ int s_cnt[kMaxSegments];
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
    if (a.has_shared && threadIdx.x == 0) s_cnt[E] = a.T;
    __syncthreads();
    // offsets: exclusive scan of the padded counts (E <= kMaxSegments - 1 < 1024 * 1)
    int total = 0;
    const int e = threadIdx.x;
    const int padded = (e < E) ? (s_cnt[e] + a.tile_m - 1) / a.tile_m * a.tile_m : 0;
    const int off = block_exclusive_scan(padded, &total);
    if (e < E) {
        a.counts[e] = s_cnt[e];
        a.offsets[e] = off;
        if (a.tables.seg_count) {
            a.tables.seg_count[e] = s_cnt[e];
            a.tables.seg_start[e] = off;
        }
    }
    if (threadIdx.x == 0) {
        a.offsets[E] = total;
        if (a.has_shared && a.tables.seg_count) {
            a.tables.seg_count[E] = a.T;
            a.tables.seg_start[E] = total;
        }
    }
    __syncthreads();
    __shared__ int s_off[kMaxSegments];
    if (e < E) s_off[e] = off;
    __syncthreads();
    for (int q = threadIdx.x; q < a.nchunks * E; q += blockDim.x)
        a.chunk_counts[q] += s_off[q % E];
    // work tables of the expert kernels
    if (a.tables.gu_items) {
        const int s = threadIdx.x;
        int gi = 0, di = 0, gt = 0, dt = 0;
        if (s < nseg) {
            const int c = s_cnt[s];
            const int Iseg = (s == E) ? a.I_s : a.I;
            if (c > 0) {
                gi = (c + kGuBN - 1) / kGuBN * (Iseg / kTcM);
                di = (c + kDnBN - 1) / kDnBN * (a.D / kTcM);
                gt = Iseg / 8;      // streaming gate_up: one warp per 8 features
                dt = a.D / 16;      // streaming down: one warp per 16 output rows
            }
        }
        int tot;
        const int pgi = block_exclusive_scan(gi, &tot);
        if (s < nseg) a.tables.gu_items[s] = pgi;
        if (s == 0) a.tables.gu_items[nseg] = tot;
        const int pdi = block_exclusive_scan(di, &tot);
        if (s < nseg) a.tables.dn_items[s] = pdi;
        if (s == 0) a.tables.dn_items[nseg] = tot;
        const int pgt = block_exclusive_scan(gt, &tot);
        if (s < nseg) a.tables.gu_tasks[s] = pgt;
        if (s == 0) a.tables.gu_tasks[nseg] = tot;
        const int pdt = block_exclusive_scan(dt, &tot);
        if (s < nseg) a.tables.dn_tasks[s] = pdt;
        if (s == 0) a.tables.dn_tasks[nseg] = tot;
    }
}

// 3. stable scatter of one chunk: 32 warps, warp w owns assignments [w*128, w*128+128) of
// the chunk, four rounds of 32 in increasing order.
__global__ void __launch_bounds__(kPermThreads) perm_scatter_kernel(PermuteArgs a) {
    extern __shared__ int wb[];  // [32][E]: per-warp counts, then per-warp running row bases
    const int E = a.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long n = (long)a.T * a.k;
    const long a0 = (long)blockIdx.x * kPermChunk + warp * (kPermChunk / 32);
    const uint32_t lt_mask = (1u << lane) - 1u;
    if (blockIdx.x < a.nchunks) {
        for (int q = threadIdx.x; q < 32 * E; q += blockDim.x) wb[q] = 0;
        __syncthreads();
#pragma unroll 1
        for (int r = 0; r < kPermChunk / 32 / 32; ++r) {
            const long as = a0 + r * 32 + lane;
            int e = (as < n) ? a.topk_idx[as] : -1;
            if (e >= E) e = -1;
            const uint32_t m = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && (m & lt_mask) == 0) wb[warp * E + e] += __popc(m);
        }
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
#pragma unroll 1
        for (int r = 0; r < kPermChunk / 32 / 32; ++r) {
            const long as = a0 + r * 32 + lane;
            int e = (as < n) ? a.topk_idx[as] : -1;
            if (e >= E) e = -1;
            const uint32_t m = __match_any_sync(0xffffffffu, e);
            int base = 0;
            if (e >= 0) base = wb[warp * E + e];
            __syncwarp();
            if (e >= 0 && (m & lt_mask) == 0) wb[warp * E + e] = base + __popc(m);
            __syncwarp();
            if (e >= 0) {
                const int row = base + __popc(m & lt_mask);
                const int t = (int)(as / a.k), j = (int)(as % a.k);
                a.slot_row[as] = row;
                if (row < a.cap) {
                    a.row_token[row] = t;
                    if (a.row_weight) a.row_weight[row] = a.topk_w ? a.topk_w[as] : 1.0f;
                    if (a.row_dest) a.row_dest[row] = t * a.slots_per_token + j;
                }
            }
        }
    }
    // rows of the shared expert: segment E, all tokens in order after the routed rows
    if (a.has_shared) {
        const int rows0 = __ldg(a.offsets + E);
        for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < a.T; t += gridDim.x * blockDim.x) {
            const int row = rows0 + t;
            if (row < a.cap) {
                a.row_token[row] = t;
                if (a.row_weight) a.row_weight[row] = 1.0f;
                if (a.row_dest) a.row_dest[row] = t * a.slots_per_token + a.k;
            }
        }
    }
    // padding rows of each expert segment (tile_m > 1)
    if (a.tile_m > 1) {
        for (int e = blockIdx.x; e < E; e += gridDim.x) {
            const int r0 = __ldg(a.offsets + e) + __ldg(a.counts + e), r1 = __ldg(a.offsets + e + 1);
            for (int row = r0 + threadIdx.x; row < r1 && row < a.cap; row += blockDim.x) {
                a.row_token[row] = -1;
                if (a.row_weight) a.row_weight[row] = 0.0f;
                if (a.row_dest) a.row_dest[row] = -1;
            }
        }
    }
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
    cudaError_t err = ensure_smem_attr((const void*)perm_scatter_kernel,
                                       32 * kMaxSegments * (int)sizeof(int), 0);
    if (err != cudaSuccess) return err;
    const long n = (long)a.T * a.k;
    perm_hist_kernel<<<a.nchunks, kPermThreads, a.E * sizeof(int), s>>>(a.topk_idx, n, a.E,
                                                                         a.chunk_counts, a.err);
    perm_scan_kernel<<<1, kPermThreads, 0, s>>>(a);
    int blocks = a.nchunks;
    if (a.has_shared && blocks < (a.T + kPermThreads - 1) / kPermThreads)
        blocks = (a.T + kPermThreads - 1) / kPermThreads;
    perm_scatter_kernel<<<blocks, kPermThreads, 32 * a.E * sizeof(int), s>>>(a);
    return cudaGetLastError();
}

// 4. x rows into permuted order: one warp per row, 16-byte pieces.  Rows with
// row_token < 0 (padding) are zero-filled.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ row_token,
                                                          int rows, int D,
                                                          uint16_t* __restrict__ x_perm) {
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
                               uint16_t* x_perm, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    int blocks = (rows + 7) / 8;
    if (blocks > 148 * 8) blocks = 148 * 8;
    gather_rows_kernel<<<blocks, 256, 0, s>>>(x, row_token, rows, D, x_perm);
    return cudaGetLastError();
}

}  // namespace moe
