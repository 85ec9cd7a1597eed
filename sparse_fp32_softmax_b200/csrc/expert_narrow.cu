// expert_narrow.cu -- the expert stage of decode-sized batches in one persistent kernel.
//
// "27. Mixture of experts" (inference.shantanugoel.com): section "Dispatch" (experts stacked
// as gate_up [E, 2I, D], gate rows first, and down [E, D, I]; expert(x) =
// down(silu(gate x) * up x); the grouped dispatch sorts the assignments by expert), section
// "The router" (y = sum_j w_j expert_j(x)), section "The shared expert" (+ sigmoid(w_s . x)
// shared(x)), and section "The economics of MoE inference": a decode step reads only the
// experts its tokens use, so at these sizes the stage is bound by streaming those weights.
//
// With few rows per expert (T*k <= 32*E) an expert is one or a few 64-token tiles and the
// time goes to streaming weights, not to the MMAs.  One persistent kernel runs the whole
// stage, so no kernel boundary interrupts the weight stream:
//   gate_up units: 128 features of one expert (its gate rows and the matching up rows, two
//                  accumulators) x up to 64 of its token rows; the epilogue writes
//                  h = silu(g) * u in bf16 and counts the unit as done for its expert;
//   down units:    128 output rows of one expert x up to 64 of its token rows; the producer
//                  loads the unit's weight tiles at once but its h tiles only after every
//                  gate_up unit of that expert is done (bounded wait on the expert's count);
//                  the epilogue scales each token's 128-row piece by the routing weight and
//                  stores it in the token's slot j;
//   combine units: 128 output rows of 4 tokens (one warp each); once every down unit is
//                  done (bounded wait on a count), a token's slots are added in slot order
//                  j = 0..k-1, then
//                  the gated shared expert and the residual, and the output is rounded once
//                  to bf16 (the arithmetic, and its order, of a separate combine pass).
// Work units are handed out in order by an atomic counter -- gate_up units, then down
// units, then combine units -- so a unit only waits for units that running CTAs have
// already taken: every wait ends, whatever the residency of the grid.  Per CTA: warp 0 takes units and issues the TMA loads,
// warp 1 allocates TMEM and one of its threads issues tcgen05.mma, warps 2..9 run the
// epilogues; unit indices reach warps 1..9 through a small shared-memory queue.  Items of a
// phase (gate_up or down) that fill whole waves of the grid run one per unit; when the
// remaining tail is at most half a wave, each tail item is split along K into slices whose
// FP32 partial sums the last slice to finish (atomic ticket) adds in slice order.
//
// route = 1 (T <= 32): after the router logits, every CTA selects the k experts of every
// token itself (FP32 softmax, top-k with ties to the lower index, renormalisation: section
// "The router") and sorts the assignments by expert with a stable counting sort run by one
// warp, into its shared memory -- cheaper than a separate kernel writing the same tables.
// CTA 0 writes the routing outputs the caller asked for.
//
// Every wait is bounded (a.wait_ns): on expiry the kernel records it in the device error
// word and winds down with no copy in flight and its TMEM released.
#include "select.cuh"

namespace moe {

namespace {

constexpr int kNwBN = kNarrowBN;                               // token columns per tile
constexpr int kNwStages = 5;
constexpr int kNwATile = kTcM * kTcK * 2;                      // 16 KB of weights
// A stage holds the gate and up tiles plus up to 64 token rows of a gate_up step; a down
// unit with at most 32 token rows puts two K steps in a stage (two weight tiles, two token
// tiles of <= 4 KB at 32 KB and 36 KB), so down keeps as many weight bytes in flight as
// gate_up does.
constexpr int kNwSB = 2 * kNwATile + kNwBN * kTcK * 2;         // 40 KB per stage
constexpr int kNwHalfB = 32 * kTcK * 2;                        // token tile of <= 32 rows
// Two threads (in warps 1 and 10) issue the MMAs: one takes the even pipeline stages of a
// unit, the other the odd ones, each into its own accumulators (the issuing thread, not the
// tensor core, bounds these narrow MMAs); the epilogue adds the two.  An accumulator set is
// gate | up (64 columns each) for gate_up, or 64 columns for down, per issuer.
constexpr int kNwHalfAcc = 2 * kNwBN;                          // one issuer's columns
constexpr int kNwAcc = 2 * kNwHalfAcc;                         // TMEM columns per buffer
constexpr int kNwBufs = 2;                                     // one buffer per epilogue group
constexpr int kNwTmem = kNwBufs * kNwAcc;                      // all of TMEM
constexpr int kNwQD = 8;                                       // unit queue depth
constexpr int kNwEpiWarps = 8;
constexpr int kNwGroupWarps = 4;                               // epilogue warps per group
constexpr int kNwMmaWarpB = 2 + kNwEpiWarps;                   // the second MMA issuer's warp
constexpr int kNwThreads = (3 + kNwEpiWarps) * 32;
constexpr int kNwCombTok = 4;                                  // tokens per combine unit
constexpr int kNwMaxAssign = kGatherMaxT * kMaxK;

struct NwTables {
    int gu_prefix[kMaxSegments + 1];   // work-item prefix sums per segment
    int dn_prefix[kMaxSegments + 1];
    int count[kMaxSegments];           // rows of each segment
    int start[kMaxSegments];           // first permuted row of each segment
};

struct NwRoute {                       // route = 1 only
    int idx[kNwMaxAssign];             // selected experts, [T, k]
    float w[kNwMaxAssign];             // routing weights, [T, k]
    float gate[kGatherMaxT];           // shared-expert gate of each token
    int rows[kNwEpiWarps + 1][kGatherMaxT];   // per warp: the assignments of one expert
};

struct NwBars {
    uint64_t full[kNwStages], empty[kNwStages], tfull[kNwBufs], tempty[kNwBufs], drain;
    uint64_t qfull[kNwQD], qempty[kNwQD];
    int q[kNwQD];
    uint32_t tmem;
    uint32_t seg_ok[(kMaxSegments + 31) / 32];   // experts this CTA has seen gate_up finish
};

constexpr int kNwSmem = kNwStages * kNwSB + 1024 + (int)sizeof(NwBars) + (int)sizeof(NwTables) +
                        (int)sizeof(NwRoute);
static_assert(kNwSmem <= 232448, "shared memory per block");
static_assert(kNwTmem <= 512, "TMEM");

struct NwPhase {
    int n;       // items
    int full;    // items in whole waves
    int S;       // slices per tail item
    int units;
};

__device__ __forceinline__ NwPhase nw_phase(int n, int G, int kstages, int slots) {
    NwPhase p;
    p.n = n;
    p.full = n / G * G;
    p.S = 1;
    const int tail = n - p.full;
    if (tail > 0 && 2 * tail <= G) {
        int S = min(G / tail, kMaxKSplit);
        S = min(S, kstages);
        S = min(S, slots / tail);
        if (S >= 2) p.S = S;
    }
    p.units = p.full + tail * p.S;
    return p;
}

struct NwTile {
    int comb;      // combine unit (rows m0 .. m0+127 of tokens b_row .. b_row + n_valid - 1)
    int gu;        // gate_up unit (else down or combine)
    int seg;       // segment: expert, or E = the shared expert
    int shared;
    int a_row0;    // gate rows (gate_up) or down rows
    int a_row1;    // up rows (gate_up)
    int b_row;     // first permuted row
    int n_valid;   // token rows, 1..64
    int bi;        // token box: 16 << bi rows
    int k0, nk;    // K steps (64 elements each) of this unit
    int dbl;       // down unit with <= 32 token rows: two K steps per pipeline stage
    int steps;     // pipeline stages of this unit
    int m0;        // first feature (gate_up) or output row (down) within the segment
    int split, nsplit, tail;
};

__device__ __forceinline__ NwTile nw_decode(const NarrowArgs& a, const NwTables* tb, const NwPhase& pg,
                                            const NwPhase& pd, int u) {
    NwTile t;
    t.comb = u >= pg.units + pd.units;
    if (t.comb) {
        const int ndt = a.D / kTcM;
        const int v = u - pg.units - pd.units;
        t.gu = 0;
        t.m0 = (v % ndt) * kTcM;
        t.b_row = (v / ndt) * kNwCombTok;
        t.n_valid = min(kNwCombTok, a.T - t.b_row);
        return t;
    }
    t.gu = u < pg.units;
    const NwPhase& ph = t.gu ? pg : pd;
    const int v = t.gu ? u : u - pg.units;
    int item = v;
    t.split = 0;
    t.nsplit = 1;
    t.tail = 0;
    if (ph.S > 1 && v >= ph.full) {
        t.tail = (v - ph.full) / ph.S;
        t.split = (v - ph.full) % ph.S;
        item = ph.full + t.tail;
        t.nsplit = ph.S;
    }
    const int* prefix = t.gu ? tb->gu_prefix : tb->dn_prefix;
    const int s = find_segment_smem(prefix, a.nseg, item);
    const int local = item - prefix[s];
    const int sh = s == a.E;
    const int Iseg = sh ? a.I_s : a.I;
    const int mtc = t.gu ? Iseg / kTcM : a.D / kTcM;
    const int tt = local / mtc, mt = local % mtc;
    t.seg = s;
    t.shared = sh;
    t.m0 = mt * kTcM;
    t.b_row = tb->start[s] + tt * kNwBN;
    t.n_valid = min(kNwBN, tb->count[s] - tt * kNwBN);
    if (t.gu) {
        const int base = sh ? 0 : s * 2 * a.I;
        t.a_row0 = base + t.m0;
        t.a_row1 = base + Iseg + t.m0;
    } else {
        t.a_row0 = (sh ? 0 : s * a.D) + t.m0;
        t.a_row1 = 0;
    }
    const int nkt = (t.gu ? a.D : Iseg) / kTcK;
    t.k0 = t.split * nkt / t.nsplit;
    t.nk = (t.split + 1) * nkt / t.nsplit - t.k0;
    t.bi = t.n_valid <= 16 ? 0 : (t.n_valid <= 32 ? 1 : 2);
    t.dbl = !t.gu && t.bi < 2;
    t.steps = t.dbl ? (t.nk + 1) / 2 : t.nk;
    return t;
}

// ------------------------------------------------------------------ routing (route = 1)

// The expert-sorted layout of the T*k assignments (T <= 32, so an expert has at most 32
// rows: one token tile): per-expert counts by shared-memory atomics of the whole block,
// then the segment tables by warp 0 (tile-padded row starts with tile_m = 1, work-item
// prefix sums).  The rows of an expert are its assignments in increasing order a = t*k + j
// (the stable sort); a unit finds them itself with nw_expert_rows, so no scatter is needed.
__device__ void nw_layout(const NarrowArgs& a, NwTables* tb, const NwRoute* rt) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = a.E, n = a.T * a.k, nseg = a.nseg;
    for (int e = threadIdx.x; e < E; e += blockDim.x) tb->count[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) atomicAdd(&tb->count[rt->idx[i]], 1);
    __syncthreads();
    if (warp != 0) return;
    // segment tables: lane owns segments [s0, s1); exclusive scans over the lanes
    const int per = (nseg + 31) / 32;
    const int s0 = min(nseg, lane * per), s1 = min(nseg, s0 + per);
    int r = 0, gi = 0, di = 0;
    for (int s = s0; s < s1; ++s) {
        const int c = s == E ? a.T : tb->count[s];
        if (s < E) r += c;
        if (c > 0) {
            const int Iseg = s == E ? a.I_s : a.I;
            gi += (c + kNwBN - 1) / kNwBN * (Iseg / kTcM);
            di += (c + kNwBN - 1) / kNwBN * (a.D / kTcM);
        }
    }
    int ir = r, ig = gi, id = di;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yg = __shfl_up_sync(0xffffffffu, ig, o);
        const int yd = __shfl_up_sync(0xffffffffu, id, o);
        if (lane >= o) {
            ir += yr;
            ig += yg;
            id += yd;
        }
    }
    int pr = ir - r, pg = ig - gi, pd = id - di;
    for (int s = s0; s < s1; ++s) {
        const int c = s == E ? a.T : tb->count[s];
        if (s == E) {
            tb->count[E] = a.T;
            tb->start[E] = n;          // the shared expert's rows follow the routed rows
        } else {
            tb->start[s] = pr;
            pr += c;
        }
        tb->gu_prefix[s] = pg;
        tb->dn_prefix[s] = pd;
        if (c > 0) {
            const int Iseg = s == E ? a.I_s : a.I;
            pg += (c + kNwBN - 1) / kNwBN * (Iseg / kTcM);
            pd += (c + kNwBN - 1) / kNwBN * (a.D / kTcM);
        }
    }
    if (lane == 31) {
        tb->gu_prefix[nseg] = ig;
        tb->dn_prefix[nseg] = id;
    }
}

// The assignments of expert e in increasing order, into list[0 .. count) (warp-collective;
// T <= 32 so an expert has at most 32 of them).
__device__ __forceinline__ void nw_expert_rows(const NarrowArgs& a, const NwRoute* rt, int e, int* list) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const int n = a.T * a.k;
    int base = 0;
    for (int a0 = 0; a0 < n; a0 += 32) {
        const int as = a0 + lane;
        const bool hit = as < n && rt->idx[as] == e;
        const uint32_t m = __ballot_sync(0xffffffffu, hit);
        if (hit) list[base + __popc(m & lt)] = as;
        base += __popc(m);
    }
    __syncwarp();
}

// The routing outputs the caller asked for, by CTA 0 (the row of assignment a is its
// expert's start plus the number of earlier assignments to the same expert).
__device__ void nw_route_outputs(const NarrowArgs& a, const NwTables* tb, const NwRoute* rt) {
    const int n = a.T * a.k;
    if (a.counts_out)
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.counts_out[e] = tb->count[e];
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        if (a.topk_idx_out) a.topk_idx_out[i] = rt->idx[i];
        if (a.topk_w_out) a.topk_w_out[i] = rt->w[i];
        if (a.slot_row_out) {
            const int e = rt->idx[i];
            int r = 0;
            for (int q = 0; q < i; ++q) r += rt->idx[q] == e;
            a.slot_row_out[i] = tb->start[e] + r;
        }
    }
}

// Selection of every token (warp w takes tokens w, w + 10, ...; the logits of all of them
// are loaded first, so the warp waits for memory once) and the shared-expert gates, then
// the permutation by warp 0.  Ends with the block synchronised.
constexpr int kNwTokPerWarp = (kGatherMaxT + 9) / 10;
template <int VPL>
__device__ void nw_select_all(const NarrowArgs& a, NwRoute* rt) {
    const int warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    const bool cta0 = blockIdx.x == 0;
    float v[kNwTokPerWarp][VPL];
#pragma unroll
    for (int j = 0; j < kNwTokPerWarp; ++j) {
        const int t = warp + j * nw;
        if (t < a.T) load_logits<VPL, true>(a.logits + (size_t)t * a.E, 1, 0, a.E, v[j]);
    }
#pragma unroll
    for (int j = 0; j < kNwTokPerWarp; ++j) {
        const int t = warp + j * nw;
        if (t < a.T)
            select_values<VPL>(v[j], a.bias, a.E, a.k, a.norm, rt->idx + t * a.k, rt->w + t * a.k,
                               (cta0 && a.logits_out) ? a.logits_out + (size_t)t * a.E : nullptr);
    }
}

__device__ void nw_route(const NarrowArgs& a, NwTables* tb, NwRoute* rt) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const bool cta0 = blockIdx.x == 0;
    if (a.E <= 32)
        nw_select_all<1>(a, rt);
    else if (a.E <= 64)
        nw_select_all<2>(a, rt);
    else if (a.E <= 128)
        nw_select_all<4>(a, rt);
    else if (a.E <= 256)
        nw_select_all<8>(a, rt);
    else
        nw_select_all<16>(a, rt);
    if (a.nseg > a.E)
        for (int t = warp; t < a.T; t += nw) {
            float g = 1.0f;
            if (a.shared_gate) g = shared_gate_value(a.x + (size_t)t * a.D, a.shared_gate, a.D);
            if (lane == 0) rt->gate[t] = g;
        }
    __syncthreads();
    nw_layout(a, tb, rt);
    __syncthreads();
    if (cta0) nw_route_outputs(a, tb, rt);
}

// ------------------------------------------------------------------ hand-off and combine

// gate_up -> down hand-off: every lane of the finishing warps releases its own h stores
// (ordinary stores that down reads with TMA, the async proxy, hence the proxy fence) with a
// non-returning add to its expert's count.
__device__ __forceinline__ void nw_signal_done(const NarrowArgs& a, int seg) {
    asm volatile("fence.proxy.async.global;" ::: "memory");
    red_release_add(a.seg_done + seg, 1);
}

// Bounded wait (one lane) until gate_up has finished segment seg: one signal per item from
// each lane of the 4 warps of the epilogue group that finished it.  A segment seen finished is
// remembered in shared memory (seg_ok), so later units of the same expert do not ask again.
__device__ bool nw_wait_done(const NarrowArgs& a, const NwTables* tb, uint32_t* seg_ok, int seg) {
    const uint32_t bit = 1u << (seg & 31);
    if (seg_ok[seg >> 5] & bit) return true;
    const int target = kNwGroupWarps * 32 * (tb->gu_prefix[seg + 1] - tb->gu_prefix[seg]);
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(a.seg_wait + seg) < target) {
        __nanosleep(64);
        if (globaltimer_ns() - t0 > a.wait_ns) {
            set_error(a.err, kErrWaitProducer);
            return false;
        }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    seg_ok[seg >> 5] |= bit;
    return true;
}

__device__ __forceinline__ float nw_gate(const NarrowArgs& a, const NwRoute* rt, int t) {
    if (a.route) return rt->gate[t];
    return a.gates ? __ldcg(a.gates + t) : 1.0f;
}

// Rows m0 .. m0+127 of token t from its S slots (lane L: rows m0 + 4L .. m0 + 4L + 3, one
// float4 per slot, every slot load in flight at once): sum j = 0..k-1 in order, then the
// gated shared expert, then the residual; one rounding to bf16.
__device__ __forceinline__ void nw_combine(const NarrowArgs& a, const NwRoute* rt, int t, int m0) {
    const int lane = threadIdx.x & 31;
    const int d = m0 + 4 * lane;
    const float* base = a.slots + (size_t)t * a.S * a.D + d;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < a.k; j0 += 8) {   // groups of 8 slots: their loads overlap
        float4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (j0 + q < a.k) v[q] = __ldcg(reinterpret_cast<const float4*>(base + (size_t)(j0 + q) * a.D));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (j0 + q >= a.k) break;
            if (j0 + q == 0) {
                acc = v[q];
            } else {
                acc.x += v[q].x; acc.y += v[q].y; acc.z += v[q].z; acc.w += v[q].w;
            }
        }
    }
    if (a.S > a.k) {
        const float4 sv = __ldcg(reinterpret_cast<const float4*>(base + (size_t)a.k * a.D));
        const float g = nw_gate(a, rt, t);
        acc.x = fmaf(g, sv.x, acc.x); acc.y = fmaf(g, sv.y, acc.y);
        acc.z = fmaf(g, sv.z, acc.z); acc.w = fmaf(g, sv.w, acc.w);
    }
    const size_t o = (size_t)t * a.D + d;
    if (a.residual) {
        const uint2 r = __ldcg(reinterpret_cast<const uint2*>(a.residual + o));
        acc.x += bf16_lo(r.x); acc.y += bf16_hi(r.x); acc.z += bf16_lo(r.y); acc.w += bf16_hi(r.y);
    }
    if (a.out_f32) *reinterpret_cast<float4*>(a.out_f32 + o) = acc;
    *reinterpret_cast<uint2*>(a.out + o) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

// Bounded wait (one lane) until every lane of every down item's four quarter warps has
// stored (and released) its slots.
__device__ bool nw_wait_down(const NarrowArgs& a, int target) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(a.dn_done) < target) {
        __nanosleep(64);
        if (globaltimer_ns() - t0 > a.wait_ns) {
            set_error(a.err, kErrWaitEpilogue);
            return false;
        }
    }
    return true;
}

}  // namespace

template <bool ROUTE>
__global__ void __launch_bounds__(kNwThreads, 1)
    narrow_expert_kernel(const __grid_constant__ NarrowMaps maps, const NarrowArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    NwBars* bars = reinterpret_cast<NwBars*>(smem + kNwStages * kNwSB);
    NwTables* tb = reinterpret_cast<NwTables*>(bars + 1);
    NwRoute* rt = reinterpret_cast<NwRoute*>(tb + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // prologue: independent of earlier kernels, overlaps them under launch chaining
    if (threadIdx.x == 0) {
        for (int s = 0; s < kNwStages; ++s) {
            mbar_init(bars->full + s, 1);
            mbar_init(bars->empty + s, 1);
        }
        for (int b = 0; b < kNwBufs; ++b) {
            mbar_init(bars->tfull + b, 2);                     // both MMA issuers
            mbar_init(bars->tempty + b, kNwGroupWarps * 32);   // the epilogue group of the buffer
        }
        mbar_init(&bars->drain, 2);
        for (int i = 0; i < (kMaxSegments + 31) / 32; ++i) bars->seg_ok[i] = 0;
        for (int q = 0; q < kNwQD; ++q) {
            mbar_init(bars->qfull + q, 1);
            mbar_init(bars->qempty + q, 2 + kNwEpiWarps);   // both MMA threads and each epilogue warp
        }
        mbar_fence_init();
    }
    if (warp == 0 && lane < 10) tma_prefetch_desc(&maps.gu_A + lane);
    if (warp == 1) tmem_alloc(&bars->tmem, kNwTmem);
    pdl_wait();
    pdl_launch_dependents();
    if (ROUTE) {
        nw_route(a, tb, rt);
    } else {
        for (int i = threadIdx.x; i <= a.nseg; i += blockDim.x) {
            tb->gu_prefix[i] = __ldcg(a.tables.gu_items + i);
            tb->dn_prefix[i] = __ldcg(a.tables.dn_items + i);
        }
        for (int i = threadIdx.x; i < a.nseg; i += blockDim.x) {
            tb->count[i] = __ldcg(a.tables.seg_count + i);
            tb->start[i] = __ldcg(a.tables.seg_start + i);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem;
    const int G = gridDim.x;
    const NwPhase pg = nw_phase(tb->gu_prefix[a.nseg], G, a.D / kTcK, a.partial_slots);
    const NwPhase pd = nw_phase(tb->dn_prefix[a.nseg], G, (a.I_s > 0 ? min(a.I, a.I_s) : a.I) / kTcK,
                                a.partial_slots);
    const int n_comb = (a.D / kTcM) * ((a.T + kNwCombTok - 1) / kNwCombTok);
    const int total = pg.units + pd.units + n_comb;

    if (warp == 0) {
        // ------------------------------------------------------------ units + TMA producer
        int it = 0;
        bool ok = true, dep_dead = false;
        int last_round[kNwStages];
#pragma unroll
        for (int s = 0; s < kNwStages; ++s) last_round[s] = -1;
        // the next unit is taken once the current one has posted its first stage, so that at
        // the start every CTA takes one unit before any takes a second
        int next = 0;
        if (lane == 0) next = atomicAdd(a.queue, 1);
        bool grabbed = false;
        auto grab_next = [&]() {
            if (!grabbed && lane == 0) next = atomicAdd(a.queue, 1);
            grabbed = true;
        };
        auto stage_begin = [&](uint32_t bytes) -> int {   // wait for a free stage, post its bytes
            const int s = it % kNwStages;
            const int round = it / kNwStages;
            const bool got = mbar_wait(bars->empty + s, (round & 1) ^ 1, a.err, kErrWaitProducer, a.wait_ns);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                return -1;
            }
            if (lane == 0) mbar_arrive_expect_tx(bars->full + s, bytes);
#pragma unroll
            for (int q = 0; q < kNwStages; ++q)
                if (q == s) last_round[q] = round;
            ++it;
            grab_next();
            return s;
        };
        for (int qi = 0; ok; ++qi) {
            const int u = __shfl_sync(0xffffffffu, next, 0);
            grabbed = u >= total;
            const int qs = qi % kNwQD;
            const bool gotq = mbar_wait(bars->qempty + qs, ((qi / kNwQD) & 1) ^ 1, a.err, kErrWaitProducer,
                                        a.wait_ns);
            if (!__all_sync(0xffffffffu, gotq)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                bars->q[qs] = u < total ? u : -1;
                mbar_arrive(bars->qfull + qs);
            }
            if (u >= total) break;
            const NwTile t = nw_decode(a, tb, pg, pd, u);
            if (t.comb) {   // no operands: the epilogue adds the slots
                grab_next();
                continue;
            }
            const int brows = 16 << t.bi;
            if (t.gu) {
                const CUtensorMap* mA = t.shared ? &maps.gu_A_shared : &maps.gu_A;
                int g0 = 0, g1 = 0, g2 = 0, g3 = 0;
                if (ROUTE) {   // token rows gathered from x: lane i takes rows 4i..4i+3
                    const int last = t.n_valid - 1;
                    if (t.shared) {
                        g0 = min(4 * lane, last);
                        g1 = min(4 * lane + 1, last);
                        g2 = min(4 * lane + 2, last);
                        g3 = min(4 * lane + 3, last);
                    } else {
                        int* list = rt->rows[kNwEpiWarps];
                        nw_expert_rows(a, rt, t.seg, list);
                        g0 = list[min(4 * lane, last)] / a.k;
                        g1 = list[min(4 * lane + 1, last)] / a.k;
                        g2 = list[min(4 * lane + 2, last)] / a.k;
                        g3 = list[min(4 * lane + 3, last)] / a.k;
                    }
                }
                const uint32_t bytes = 2 * kNwATile + (uint32_t)brows * kTcK * 2;
                for (int kb = 0; kb < t.nk; ++kb) {
                    const int s = stage_begin(bytes);
                    if (s < 0) break;
                    uint8_t* st = smem + s * kNwSB;
                    const int kx = (t.k0 + kb) * kTcK;
                    if (lane == 0) {
                        tma_load(st, mA, bars->full + s, kx, t.a_row0);
                        tma_load(st + kNwATile, mA, bars->full + s, kx, t.a_row1);
                        if (!ROUTE) tma_load(st + 2 * kNwATile, &maps.gu_B[t.bi], bars->full + s, kx, t.b_row);
                    }
                    if (ROUTE) {
                        __syncwarp();   // expect_tx is posted before any gather can complete
                        if (4 * lane < brows)
                            tma_gather4(st + 2 * kNwATile + lane * 4 * kTcK * 2, &maps.gu_B[0], bars->full + s,
                                        kx, g0, g1, g2, g3);
                    }
                }
            } else {
                const CUtensorMap* mA = t.shared ? &maps.dn_A_shared : &maps.dn_A;
                const CUtensorMap* mB = &maps.dn_B[t.bi];
                const uint32_t step_bytes = kNwATile + (uint32_t)brows * kTcK * 2;
                // K steps of stage j: 2j, 2j+1 (dbl) or j
                auto nsteps = [&](int j) { return t.dbl ? min(2, t.nk - 2 * j) : 1; };
                auto first = [&](int j) { return t.dbl ? 2 * j : j; };
                auto load_a = [&](int s, int j) {
                    for (int q = 0; q < nsteps(j); ++q)
                        tma_load(smem + s * kNwSB + q * kNwATile, mA, bars->full + s,
                                 (t.k0 + first(j) + q) * kTcK, t.a_row0);
                };
                auto load_b = [&](int s, int j) {
                    for (int q = 0; q < nsteps(j); ++q)
                        tma_load(smem + s * kNwSB + (t.dbl ? 2 * kNwATile + q * kNwHalfB : kNwATile), mB,
                                 bars->full + s, (t.k0 + first(j) + q) * kTcK, t.b_row);
                };
                // weight tiles of the first stages do not depend on gate_up: issue them now
                const int pre = min(t.steps, kNwStages);
                const int it0 = it;
                for (int j = 0; j < pre; ++j) {
                    const int s = stage_begin(step_bytes * nsteps(j));
                    if (s < 0) break;
                    if (lane == 0) load_a(s, j);
                }
                if (!ok) break;
                // the unit's later weight tiles start their way into L2 too
                if (lane == 0)
                    for (int kb = first(pre); kb < t.nk; ++kb) tma_prefetch_l2(mA, (t.k0 + kb) * kTcK, t.a_row0);
                // h tiles once gate_up has finished this expert (after a timed-out wait the
                // loads still run, so every posted stage completes; the error is recorded)
                if (!dep_dead) {
                    bool got = true;
                    if (lane == 0) got = nw_wait_done(a, tb, bars->seg_ok, t.seg);
                    if (!__shfl_sync(0xffffffffu, got, 0)) dep_dead = true;
                }
                if (lane == 0)
                    for (int j = 0; j < pre; ++j) load_b((it0 + j) % kNwStages, j);
                for (int j = pre; j < t.steps; ++j) {
                    const int s = stage_begin(step_bytes * nsteps(j));
                    if (s < 0) break;
                    if (lane == 0) {
                        load_a(s, j);
                        load_b(s, j);
                    }
                }
            }
        }
        // wait until the MMA issuer has released every stage, then until every issued load
        // has landed, so no copy is in flight when the CTA exits
        if (ok) {
            for (int i = 0; i < kNwStages; ++i, ++it) {
                const int s = it % kNwStages;
                const int round = it / kNwStages;
                const bool got = mbar_wait(bars->empty + s, (round & 1) ^ 1, a.err, kErrWaitTail, a.wait_ns);
                if (!__all_sync(0xffffffffu, got)) break;
            }
        }
#pragma unroll
        for (int s = 0; s < kNwStages; ++s)
            if (last_round[s] >= 0) mbar_wait(bars->full + s, last_round[s] & 1, a.err, kErrWaitTail, a.wait_ns);
    } else if (warp == 1 || warp == kNwMmaWarpB) {
        // ------------------------------------------------------------ MMA issuers
        // Issuer X (0: warp 1, 1: warp 10) takes the stages j of each unit with j % 2 == X,
        // into accumulators at column offset X * kNwHalfAcc of the unit's buffer; both follow
        // the ring position of every stage (a running count over all units).
        const int X = warp == 1 ? 0 : 1;
        if (lane == 0) {
            const uint32_t idesc0 = umma_idesc_bf16_f32(kTcM, 16) & ~(0x3Fu << 17);
            const uint64_t dA0 = umma_desc_sw128(smem);
            const uint64_t dA1 = umma_desc_sw128(smem + kNwATile);
            const uint64_t dBg = umma_desc_sw128(smem + 2 * kNwATile);   // gate_up token tile
            const uint64_t dBd = umma_desc_sw128(smem + kNwATile);       // down h tile
            const uint64_t dBd0 = umma_desc_sw128(smem + 2 * kNwATile);  // two-step down stages
            const uint64_t dBd1 = umma_desc_sw128(smem + 2 * kNwATile + kNwHalfB);
            int pos = 0, tc = 0;   // ring position of the next unit's first stage
            for (int qi = 0;; ++qi) {
                const int qs = qi % kNwQD;
                if (!mbar_wait(bars->qfull + qs, (qi / kNwQD) & 1, a.err, kErrWaitMma, a.wait_ns)) break;
                const int u = bars->q[qs];
                mbar_arrive(bars->qempty + qs);
                if (u < 0) break;
                const NwTile t = nw_decode(a, tb, pg, pd, u);
                if (t.comb) continue;
                const int b = tc & 1, use = tc >> 1;
                ++tc;
                const int base = pos;
                pos += t.steps;
                if (!mbar_wait(bars->tempty + b, (use & 1) ^ 1, a.err, kErrWaitMma, a.wait_ns)) break;
                tc_fence_after();
                int n = (t.n_valid + 15) & ~15;
                n = n < 16 ? 16 : n;
                const uint32_t idesc = idesc0 | ((uint32_t)(n >> 3) << 17);
                const uint32_t d0 = tmem + (uint32_t)(b * kNwAcc + X * kNwHalfAcc);
                bool ok = true;
                for (int j = X; j < t.steps; j += 2) {
                    const int P = base + j;
                    const int s = P % kNwStages;
                    const int round = P / kNwStages;
                    // The other issuer may still hold this slot's previous stage (P - STAGES),
                    // so its full barrier may not have reached P's phase yet, and a parity wait
                    // cannot tell two phases apart: first wait until that stage is released
                    // (the producer's own condition for loading P), then for P's data.
                    if (round > 0 &&
                        !mbar_wait(bars->empty + s, (round & 1) ^ 1, a.err, kErrWaitMma, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(bars->full + s, round & 1, a.err, kErrWaitMma, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t off = (uint64_t)(s * (kNwSB >> 4));
                    const uint32_t acc = j > X ? 1u : 0u;   // this issuer's first stage overwrites
                    if (t.gu) {
                        umma_bf16(d0, dA0 + off, dBg + off, idesc, acc);
                        umma_bf16(d0 + kNwBN, dA1 + off, dBg + off, idesc, acc);
#pragma unroll
                        for (int kk = 1; kk < kTcK / 16; ++kk) {
                            umma_bf16_acc(d0, dA0 + off + 2 * kk, dBg + off + 2 * kk, idesc);
                            umma_bf16_acc(d0 + kNwBN, dA1 + off + 2 * kk, dBg + off + 2 * kk, idesc);
                        }
                    } else if (t.dbl) {
                        umma_bf16(d0, dA0 + off, dBd0 + off, idesc, acc);
#pragma unroll
                        for (int kk = 1; kk < kTcK / 16; ++kk)
                            umma_bf16_acc(d0, dA0 + off + 2 * kk, dBd0 + off + 2 * kk, idesc);
                        if (2 * j + 1 < t.nk) {
#pragma unroll
                            for (int kk = 0; kk < kTcK / 16; ++kk)
                                umma_bf16_acc(d0, dA1 + off + 2 * kk, dBd1 + off + 2 * kk, idesc);
                        }
                    } else {
                        umma_bf16(d0, dA0 + off, dBd + off, idesc, acc);
#pragma unroll
                        for (int kk = 1; kk < kTcK / 16; ++kk)
                            umma_bf16_acc(d0, dA0 + off + 2 * kk, dBd + off + 2 * kk, idesc);
                    }
                    umma_commit(bars->empty + s);
                }
                if (!ok) break;
                umma_commit(bars->tfull + b);   // (with no stages of this issuer: arrives at once)
            }
            // every issued MMA must be complete before TMEM is released
            umma_commit(&bars->drain);
            mbar_wait(&bars->drain, 0, a.err, kErrWaitMma, a.wait_ns);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps 2..9
        // Two groups of four warps take alternate units (group g: units tc with tc % 2 == g,
        // in TMEM buffer g), so one group's stores and fences overlap the other's; within a
        // group warp w reads its TMEM lane quarter w % 4 and finishes both 32-column chunks of
        // the unit.  A unit's value is the first issuer's accumulator plus the second's (when
        // the unit has a second stage).
        const int quarter = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int row = quarter * 32 + lane;
        int tc = 0, cc = 0;
        bool down_done = false;
        for (int qi = 0;; ++qi) {
            const int qs = qi % kNwQD;
            const bool gotq = mbar_wait(bars->qfull + qs, (qi / kNwQD) & 1, a.err, kErrWaitEpilogue, a.wait_ns);
            if (!__all_sync(0xffffffffu, gotq)) break;
            const int u = bars->q[qs];
            __syncwarp();
            if (lane == 0) mbar_arrive(bars->qempty + qs);
            if (u < 0) break;
            const NwTile t = nw_decode(a, tb, pg, pd, u);
            if (t.comb) {
                // combine units alternate between the groups too
                const bool mine_c = (cc & 1) == grp;
                ++cc;
                if (!mine_c) continue;
                if (!down_done) {
                    bool ok = true;
                    if (lane == 0) ok = nw_wait_down(a, kNwGroupWarps * 32 * pd.n);
                    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
                    down_done = true;
                }
                // the group's warp of lane quarter q takes token b_row + q of the unit
                if (quarter < t.n_valid) nw_combine(a, rt, t.b_row + quarter, t.m0);
                continue;
            }
            const int b = tc % kNwBufs, use = tc / kNwBufs;
            const bool mine = (tc & 1) == grp;
            ++tc;
            if (!mine) continue;
            const bool got = mbar_wait(bars->tfull + b, use & 1, a.err, kErrWaitEpilogue, a.wait_ns);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t tb_addr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * kNwAcc);
            const int nch = (t.n_valid + 31) >> 5;   // 1 or 2 chunks
            const bool two = t.steps >= 2;           // the second issuer wrote its accumulators
            // 32 columns of the first issuer's accumulator plus the second's, into dst
            auto ld_sum = [&](uint32_t addr, float (&dst)[32]) {
                tmem_ld32(addr, dst);
                tmem_ld_wait();
                if (two) {
                    float tmp[16];
                    tmem_ld16(addr + kNwHalfAcc, tmp);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) dst[i] += tmp[i];
                    tmem_ld16(addr + kNwHalfAcc + 16, tmp);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) dst[16 + i] += tmp[i];
                }
            };
            // down: the slot and the weight of column c*32 + lane of each chunk
            int dl[2] = {0, 0};
            float wl[2] = {0.f, 0.f};
            if (!t.gu && ROUTE) {
                // one chunk (an expert has at most 32 rows when the kernel routes)
                if (t.shared) {
                    dl[0] = lane * a.S + a.k;
                    wl[0] = 1.0f;
                } else {
                    int* list = rt->rows[warp - 2];
                    nw_expert_rows(a, rt, t.seg, list);
                    if (lane < t.n_valid) {
                        const int as = list[lane];
                        const int tok = as / a.k;
                        dl[0] = tok * a.S + (as - tok * a.k);
                        wl[0] = rt->w[as];
                    }
                }
            } else if (!t.gu) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int col = c * 32 + lane;
                    if (col < t.n_valid) {
                        const int r = t.b_row + col;
                        dl[c] = __ldg(a.row_dest + r);
                        wl[c] = __ldg(a.row_weight + r);
                    }
                }
            }
            float v[32], uu[32];
            const int NA = t.gu ? 2 : 1;
            if (t.nsplit > 1) {
                // 1. this slice's partial accumulators: [NA][128 rows][64 columns] FP32
                float* ps = (t.gu ? a.partial_gu : a.partial_dn) +
                            (size_t)(t.tail * t.nsplit + t.split) * (NA * kTcM * kNwBN);
                for (int c = 0; c < nch; ++c) {
                    ld_sum(tb_addr + c * 32, v);
                    if (t.gu) ld_sum(tb_addr + kNwBN + c * 32, uu);
                    float4* d0 = reinterpret_cast<float4*>(ps + (size_t)row * kNwBN + c * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q) d0[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    if (t.gu) {
                        float4* d1 = reinterpret_cast<float4*>(ps + (size_t)(kTcM + row) * kNwBN + c * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            d1[q] = make_float4(uu[4 * q], uu[4 * q + 1], uu[4 * q + 2], uu[4 * q + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(bars->tempty + b);
                // 2. publish; the warp that completes this (item, quarter) portion reduces it
                __threadfence();
                __syncwarp();
                int old = 0;
                int* ticket = (t.gu ? a.tickets_gu : a.tickets_dn) + t.tail * 4 + quarter;
                if (lane == 0) old = atomicAdd(ticket, 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old != t.nsplit - 1) continue;
                __threadfence();
                if (lane == 0) *ticket = 0;   // ready for the next launch
            }
            for (int c = 0; c < nch; ++c) {
                const int nv = min(32, t.n_valid - c * 32);
                if (t.nsplit > 1) {
                    const float* p0 = (t.gu ? a.partial_gu : a.partial_dn) +
                                      (size_t)(t.tail * t.nsplit) * (NA * kTcM * kNwBN) + c * 32;
                    // the slices are added in slice order (their loads overlap as far as the
                    // registers allow)
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        if (4 * g >= nv) break;
                        const float* pp = p0 + 4 * g;
                        float4 sv = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)row * kNwBN));
                        float4 su = t.gu ? __ldcg(reinterpret_cast<const float4*>(pp + (size_t)(kTcM + row) * kNwBN)) : sv;
                        for (int sp = 1; sp < t.nsplit; ++sp) {
                            const float* q = pp + (size_t)sp * (NA * kTcM * kNwBN);
                            const float4 lv = __ldcg(reinterpret_cast<const float4*>(q + (size_t)row * kNwBN));
                            sv.x += lv.x; sv.y += lv.y; sv.z += lv.z; sv.w += lv.w;
                            if (t.gu) {
                                const float4 lu = __ldcg(reinterpret_cast<const float4*>(q + (size_t)(kTcM + row) * kNwBN));
                                su.x += lu.x; su.y += lu.y; su.z += lu.z; su.w += lu.w;
                            }
                        }
                        v[4 * g] = sv.x; v[4 * g + 1] = sv.y; v[4 * g + 2] = sv.z; v[4 * g + 3] = sv.w;
                        uu[4 * g] = su.x; uu[4 * g + 1] = su.y; uu[4 * g + 2] = su.z; uu[4 * g + 3] = su.w;
                    }
                } else {
                    ld_sum(tb_addr + c * 32, v);
                    if (t.gu) ld_sum(tb_addr + kNwBN + c * 32, uu);
                    if (c == nch - 1) {
                        tc_fence_before();
                        mbar_arrive(bars->tempty + b);   // all values are in registers or stored
                    }
                }
                // v (and uu) hold row `row` of the chunk's columns
                if (t.gu) {
                    uint16_t* hp = a.h + (size_t)(t.b_row + c * 32) * a.ld_h + t.m0 + row;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (j < nv) hp[(size_t)j * a.ld_h] = to_bf16_bits(silu(v[j]) * uu[j]);
                } else {
                    const int d = t.m0 + row;
                    const int dlc = c ? dl[1] : dl[0];
                    const float wlc = c ? wl[1] : wl[0];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int dj = __shfl_sync(0xffffffffu, dlc, j);
                        const float wj = __shfl_sync(0xffffffffu, wlc, j);
                        if (j < nv) a.slots[(size_t)dj * a.D + d] = wj * v[j];
                    }
                }
            }
            if (t.gu)
                nw_signal_done(a, t.seg);
            else
                red_release_add(a.dn_done, 1);   // this lane's slots of the item are stored
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kNwTmem);
    }
}

cudaError_t launch_narrow(const NarrowMaps& maps, const NarrowArgs& a, int grid, bool pdl, cudaStream_t s) {
    if (a.route && (a.T > kGatherMaxT || a.T * a.k > kNwMaxAssign)) return cudaErrorInvalidValue;
    auto kernel = a.route ? narrow_expert_kernel<true> : narrow_expert_kernel<false>;
    cudaError_t err = ensure_smem_attr((const void*)kernel, kNwSmem);
    if (err != cudaSuccess) return err;
    if (grid < 1) grid = 1;
    return launch_kernel(kernel, dim3(grid), dim3(kNwThreads), kNwSmem, s, pdl, maps, a);
}

}  // namespace moe
