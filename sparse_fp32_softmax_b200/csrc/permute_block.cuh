// permute_block.cuh -- block-level pieces of the expert counting sort (see permute.cu):
// block scan, offsets and work tables, stable per-warp ranking and scattering, and the
// whole permutation by one block.  Included by the translation units that use them.
#pragma once

#include "common.cuh"

namespace moe {

// Warp-wide exclusive scan; *total receives the warp's sum.
static __device__ __forceinline__ int warp_exclusive_scan(int v, int* total) {
    const int lane = threadIdx.x & 31;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    *total = __shfl_sync(0xffffffffu, inc, 31);
    return inc - v;
}

// From per-expert totals s_cnt[0..E) (block-visible shared memory), by one whole warp: write
// counts, the tile-padded offsets (also into s_off[0..E]), the segment tables and the
// work-item prefix sums of the expert kernels.  Lane L owns a contiguous run of segments;
// a pass for the lane totals, five warp scans, and a pass that writes.  The caller
// synchronises the block afterwards.
static __device__ void finish_offsets_warp(const PermuteArgs& a, const int* s_cnt, int* s_off) {
    const int lane = threadIdx.x & 31;
    const int E = a.E;
    const int nseg = E + (a.has_shared ? 1 : 0);
    const int per = (nseg + 31) >> 5;
    const int s0 = min(nseg, lane * per), s1 = min(nseg, s0 + per);
    const bool items = a.tables.gu_items != nullptr;
    struct Seg { int c, pad, gi, di, gt, dt; };
    auto seg = [&](int s) {
        Seg g;
        g.c = (s == E) ? a.T : s_cnt[s];
        g.pad = (s < E) ? (g.c + a.tile_m - 1) / a.tile_m * a.tile_m : 0;
        const int Iseg = (s == E) ? a.I_s : a.I;
        g.gi = g.di = g.gt = g.dt = 0;
        if (g.c > 0) {
            g.gi = (g.c + a.gu_bn - 1) / a.gu_bn * (Iseg / a.gu_features);
            g.di = (g.c + a.dn_bn - 1) / a.dn_bn * (a.D / kTcM);
            g.gt = Iseg / 8;    // streaming gate_up: one warp per 8 features
            g.dt = a.D / 16;    // streaming down: one warp per 16 output rows
        }
        return g;
    };
    int tp = 0, tgi = 0, tdi = 0, tgt = 0, tdt = 0;
    for (int s = s0; s < s1; ++s) {
        const Seg g = seg(s);
        tp += g.pad; tgi += g.gi; tdi += g.di; tgt += g.gt; tdt += g.dt;
    }
    int Tp, Tgi, Tdi, Tgt, Tdt;
    int rp = warp_exclusive_scan(tp, &Tp);
    int rgi = warp_exclusive_scan(tgi, &Tgi);
    int rdi = warp_exclusive_scan(tdi, &Tdi);
    int rgt = warp_exclusive_scan(tgt, &Tgt);
    int rdt = warp_exclusive_scan(tdt, &Tdt);
    for (int s = s0; s < s1; ++s) {
        const Seg g = seg(s);
        if (s < E) {
            a.counts[s] = g.c;
            a.offsets[s] = rp;
            s_off[s] = rp;
            if (a.tables.seg_count) {
                a.tables.seg_count[s] = g.c;
                a.tables.seg_start[s] = rp;
            }
            rp += g.pad;
        } else if (a.tables.seg_count) {  // the shared expert: all T rows after the routed ones
            a.tables.seg_count[E] = a.T;
            a.tables.seg_start[E] = Tp;
        }
        if (items) {
            a.tables.gu_items[s] = rgi; rgi += g.gi;
            a.tables.dn_items[s] = rdi; rdi += g.di;
            a.tables.gu_tasks[s] = rgt; rgt += g.gt;
            a.tables.dn_tasks[s] = rdt; rdt += g.dt;
        }
    }
    if (lane == 0) {
        a.offsets[E] = Tp;
        s_off[E] = Tp;
        if (items) {
            a.tables.gu_items[nseg] = Tgi;
            a.tables.dn_items[nseg] = Tdi;
            a.tables.gu_tasks[nseg] = Tgt;
            a.tables.dn_tasks[nseg] = Tdt;
        }
    }
}

// Warp w of a block of W warps owns assignments [a0 + w*L, a0 + w*L + L), L = 4096 / W
// (at most 256 = 8 rounds of 32), in rounds of 32 in increasing order.  A lane's experts
// (and weights) of all rounds are loaded once, up front, so the passes below cost one memory
// round trip instead of one per round.
constexpr int kMaxRounds = 8;
struct WarpSlice {
    int e[kMaxRounds];      // expert of the lane's assignment in each round (-1: none)
    float w[kMaxRounds];    // its routing weight
    int rounds;
    long w0;                // first assignment of the warp's slice
};

static __device__ __forceinline__ WarpSlice load_warp_slice(const PermuteArgs& a, long a0) {
    WarpSlice ws;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int slice = kPermChunk / (blockDim.x >> 5);
    const long n = (long)a.T * a.k;
    ws.rounds = slice / 32;
    ws.w0 = a0 + (long)warp * slice;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
        const long as = ws.w0 + r * 32 + lane;
        const bool in = r < ws.rounds && as < n;
        int e = in ? __ldcg(a.topk_idx + as) : -1;
        ws.w[r] = (in && a.topk_w) ? __ldcg(a.topk_w + as) : 1.0f;
        if (in && (e >= a.E || e < 0)) {
            set_error(a.err, kErrBadIndex);
            e = -1;
        }
        ws.e[r] = e;
    }
    return ws;
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
        const uint32_t m = __match_any_sync(0xffffffffu, e);
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
                if (a.row_weight) a.row_weight[row] = ws.w[r];
                if (a.row_dest) a.row_dest[row] = t * a.slots_per_token + j;
            }
        }
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

// The whole permutation by one block of 1024 threads (T*k <= 4096).  wb: [32][E] ints of
// shared memory.  Also called by the fused routing kernel's last block.
static __device__ void permute_one_block(const PermuteArgs& a, int* wb) {
    __shared__ int s_cnt[kMaxSegments];
    __shared__ int s_off[kMaxSegments + 1];
    const int E = a.E;
    const WarpSlice ws = load_warp_slice(a, 0);
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
    if (threadIdx.x < 32) finish_offsets_warp(a, s_cnt, s_off);
    __syncthreads();
    for (int q = threadIdx.x; q < 32 * E; q += blockDim.x) wb[q] += s_off[q % E];
    __syncthreads();
    scatter_warp_slices(a, ws, wb);
    write_fixed_rows(a, s_off[E], s_off, s_cnt, 0, 1);
}

}  // namespace moe
