// permute_block.cuh -- block-level pieces of the expert counting sort (see permute.cu):
// block scan, offsets and work tables, stable per-warp ranking and scattering, and the
// whole permutation by one block.  Included by the translation units that use them.
#pragma once

#include "common.cuh"

namespace moe {

// Block-wide exclusive scan of three ints per thread at once (blockDim.x <= 1024, a multiple
// of 32): v[j] becomes its exclusive prefix over the block, tot[j] the block's sum.  Two
// __syncthreads.
static __device__ void block_exclusive_scan3(int (&v)[3], int (&tot)[3]) {
    __shared__ int wsum[32][3];
    __shared__ int wtot[3];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int inc[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        inc[j] = v[j];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc[j], o);
            if (lane >= o) inc[j] += y;
        }
        if (lane == 31) wsum[warp][j] = inc[j];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int w = lane < nwarps ? wsum[lane][j] : 0;
            int winc = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, winc, o);
                if (lane >= o) winc += y;
            }
            if (lane < nwarps) wsum[lane][j] = winc - w;  // exclusive warp offsets
            if (lane == 31) wtot[j] = winc;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        v[j] = wsum[warp][j] + inc[j] - v[j];
        tot[j] = wtot[j];
    }
}

// From per-expert totals s_cnt[0..E) (block-visible shared memory), by the whole block (one
// thread per segment, nseg <= blockDim.x): write counts, the tile-padded offsets (also into
// s_off[0..E]), the segment tables and the work-item prefix sums of the expert kernels.
// Ends with the block synchronised.
static __device__ void finish_offsets(const PermuteArgs& a, const int* s_cnt, int* s_off) {
    const int E = a.E;
    const int nseg = E + (a.has_shared ? 1 : 0);
    const int s = threadIdx.x;
    int v[3] = {0, 0, 0};   // padded rows, gate_up items, down items
    int c = 0;
    if (s < nseg) {
        c = (s == E) ? a.T : s_cnt[s];
        if (s < E) v[0] = (c + a.tile_m - 1) / a.tile_m * a.tile_m;
        if (c > 0) {
            const int Iseg = (s == E) ? a.I_s : a.I;
            v[1] = (c + a.gu_bn - 1) / a.gu_bn * (Iseg / a.gu_features);
            v[2] = (c + a.dn_bn - 1) / a.dn_bn * (a.D / a.dn_rows);
        }
    }
    int tot[3];
    block_exclusive_scan3(v, tot);
    if (s < E) {
        a.counts[s] = c;
        a.offsets[s] = v[0];
        s_off[s] = v[0];
        if (a.tables.seg_count) {
            a.tables.seg_count[s] = c;
            a.tables.seg_start[s] = v[0];
        }
    } else if (s == E) {
        a.offsets[E] = tot[0];
        s_off[E] = tot[0];
        if (a.has_shared && a.tables.seg_count) {   // the shared expert: after the routed rows
            a.tables.seg_count[E] = a.T;
            a.tables.seg_start[E] = tot[0];
        }
    }
    if (a.tables.gu_items && s <= nseg) {
        a.tables.gu_items[s] = s < nseg ? v[1] : tot[1];
        a.tables.dn_items[s] = s < nseg ? v[2] : tot[2];
    }
    __syncthreads();
}

// Warp w of a block of W warps owns assignments [a0 + w*L, a0 + w*L + L) of the chunk's n_c
// assignments (n_c <= 4096), L = ceil(n_c / W) rounded up to a multiple of 32 (at most 256 =
// 8 rounds of 32), in rounds of 32 in increasing order: every warp gets a share, so the
// serial rounds per warp are as few as the chunk allows.  A lane's experts (and weights) of
// all rounds are loaded once, up front, so the passes below cost one memory round trip
// instead of one per round.
constexpr int kMaxRounds = 8;
struct WarpSlice {
    int e[kMaxRounds];      // expert of the lane's assignment in each round (-1: none)
    float w[kMaxRounds];    // its routing weight
    int rounds;
    long w0;                // first assignment of the warp's slice
};

// (FROM_SMEM: the assignments' experts and weights are in shared memory at idx_s / w_s,
// the block having just selected them itself; otherwise they are read from a.topk_idx /
// a.topk_w)
template <bool FROM_SMEM = false>
static __device__ __forceinline__ WarpSlice load_warp_slice(const PermuteArgs& a, long a0,
                                                            const int* idx_s = nullptr,
                                                            const float* w_s = nullptr) {
    WarpSlice ws;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long n = (long)a.T * a.k;
    const long n_c = n - a0 < kPermChunk ? n - a0 : kPermChunk;   // this chunk's assignments
    const int nwarps = blockDim.x >> 5;
    const int slice = (int)((n_c + nwarps - 1) / nwarps + 31) / 32 * 32;
    ws.rounds = slice / 32;
    ws.w0 = a0 + (long)warp * slice;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        const long as = ws.w0 + r * 32 + lane;
        const bool in = r < ws.rounds && as < n;
        int e;
        if (FROM_SMEM) {
            e = in ? idx_s[as] : -1;
            ws.w[r] = in ? w_s[as] : 1.0f;
        } else {
            e = in ? __ldcg(a.topk_idx + as) : -1;
            ws.w[r] = (in && a.topk_w) ? __ldcg(a.topk_w + as) : 1.0f;
        }
        if (in && (e >= a.E || e < 0)) {
            set_error(a.err, kErrBadIndex);
            e = -1;
        }
        ws.e[r] = e;
    }
    return ws;
}

// Lanes of the warp holding the same value as this lane (e in [-1, 1023]; -1 matches -1):
// one ballot per bit of the 10-bit value.
static __device__ __forceinline__ uint32_t match_expert(int e) {
    const uint32_t v = (uint32_t)e & 0x3FFu;
    uint32_t m = 0xffffffffu;
#pragma unroll
    for (int b = 0; b < 10; ++b) {
        const uint32_t bit = (v >> b) & 1u;
        const uint32_t bb = __ballot_sync(0xffffffffu, bit);
        m &= bit ? bb : ~bb;
    }
    return m;
}

// Counting pass: wb[w*E + e] += assignments of e in the warp's slice.
static __device__ void count_warp_slices(const PermuteArgs& a, const WarpSlice& ws, int* wb) {
    const int E = a.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        if (r >= ws.rounds) break;
        const int e = ws.e[r];
        const uint32_t m = match_expert(e);
        if (e >= 0 && (m & lt_mask) == 0) wb[warp * E + e] += __popc(m);
    }
}

// Scatter pass: wb[w*E + e] holds the first row warp w may give to expert e; each
// assignment takes the next row of its expert (stable: lanes in order, rounds in order).
static __device__ void scatter_warp_slices(const PermuteArgs& a, const WarpSlice& ws, int* wb) {
    const int E = a.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        if (r >= ws.rounds) break;
        const int e = ws.e[r];
        const long as = ws.w0 + r * 32 + lane;
        const uint32_t m = match_expert(e);
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
                if (a.row_weight) a.row_weight[row] = ws.w[r];
                if (a.row_dest) a.row_dest[row] = t * a.slots_per_token + j;
            }
        }
    }
}

// The same pass for a single block whose routed rows fit kInvRows: rows are recorded in a
// shared-memory inverse (row -> assignment, and its weight) instead of written to global
// memory in assignment order; write_rows_from_inverse then writes them in row order.
constexpr int kInvRows = 4096;
static __device__ void scatter_warp_slices_inv(const PermuteArgs& a, const WarpSlice& ws, int* wb,
                                               int* inv, float* winv) {
    const int E = a.E;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        if (r >= ws.rounds) break;
        const int e = ws.e[r];
        const long as = ws.w0 + r * 32 + lane;
        const uint32_t m = match_expert(e);
        int base = 0;
        if (e >= 0) base = wb[warp * E + e];
        __syncwarp();
        if (e >= 0 && (m & lt_mask) == 0) wb[warp * E + e] = base + __popc(m);
        __syncwarp();
        if (e >= 0) {
            const int row = base + __popc(m & lt_mask);
            a.slot_row[as] = row;
            inv[row] = (int)as;
            winv[row] = ws.w[r];
        }
    }
}

// Row metadata of routed rows [0, rows) in row order (coalesced): padding rows (inv < 0) get
// token -1, weight 0, destination -1.
static __device__ void write_rows_from_inverse(const PermuteArgs& a, const int* inv,
                                               const float* winv, int rows) {
    for (int r = threadIdx.x; r < rows && r < a.cap; r += blockDim.x) {
        const int as = inv[r];
        const int t = as >= 0 ? as / a.k : -1;
        a.row_token[r] = t;
        if (a.row_weight) a.row_weight[r] = as >= 0 ? winv[r] : 0.0f;
        if (a.row_dest) a.row_dest[r] = as >= 0 ? t * a.slots_per_token + (as - t * a.k) : -1;
    }
}

// Rows of the shared expert (segment E: all tokens in order after the routed rows) and
// padding rows of each expert segment (tile_m > 1), spread over blocks b0 of nb.
static __device__ void write_fixed_rows(const PermuteArgs& a, int rows0, const int* offsets,
                                 const int* counts, int b0, int nb) {
    if (a.has_shared) {
        for (int t = b0 * blockDim.x + threadIdx.x; t < a.T; t += nb * blockDim.x) {
            const int row = rows0 + t;
            if (row < a.cap) {
                a.row_token[row] = t;
                if (a.row_weight) a.row_weight[row] = 1.0f;
                if (a.row_dest) a.row_dest[row] = t * a.slots_per_token + a.k;
            }
        }
    }
    if (a.tile_m > 1) {
        for (int e = b0; e < a.E; e += nb) {
            const int r0 = offsets[e] + counts[e], r1 = offsets[e + 1];
            for (int row = r0 + threadIdx.x; row < r1 && row < a.cap; row += blockDim.x) {
                a.row_token[row] = -1;
                if (a.row_weight) a.row_weight[row] = 0.0f;
                if (a.row_dest) a.row_dest[row] = -1;
            }
        }
    }
}

// ------------------------------------------------------------------ single-block path

// The whole permutation by one block of 1024 threads (T*k <= 4096), from the block's warp
// slices (load_warp_slice with a0 = 0).  wb: [32][E] ints of shared memory.
static __device__ void permute_one_block(const PermuteArgs& a, int* wb, const WarpSlice& ws) {
    __shared__ int s_cnt[kMaxSegments];
    __shared__ int s_off[kMaxSegments + 1];
    const int E = a.E;
    for (int q = threadIdx.x; q < 32 * E; q += blockDim.x) wb[q] = 0;
    __syncthreads();
    count_warp_slices(a, ws, wb);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {   // per-warp exclusive prefix
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int v = wb[w * E + e];
            wb[w * E + e] = run;
            run += v;
        }
        s_cnt[e] = run;
    }
    __syncthreads();
    finish_offsets(a, s_cnt, s_off);
    for (int q = threadIdx.x; q < 32 * E; q += blockDim.x) wb[q] += s_off[q % E];
    const int rows = s_off[E];
    if (rows <= kInvRows) {
        __shared__ int inv[kInvRows];
        __shared__ float winv[kInvRows];
        for (int r = threadIdx.x; r < rows; r += blockDim.x) inv[r] = -1;   // padding rows
        __syncthreads();
        scatter_warp_slices_inv(a, ws, wb, inv, winv);
        __syncthreads();
        write_rows_from_inverse(a, inv, winv, rows);
        if (a.has_shared) write_fixed_rows(a, rows, s_off, s_cnt, 0, 1);   // shared rows only
    } else {
        __syncthreads();
        scatter_warp_slices(a, ws, wb);
        write_fixed_rows(a, rows, s_off, s_cnt, 0, 1);
    }
}

}  // namespace moe
