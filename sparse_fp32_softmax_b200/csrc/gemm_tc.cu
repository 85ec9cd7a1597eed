// gemm_tc.cu -- persistent grouped GEMMs on the 5th-generation tensor core (tcgen05).
//
// "27. Mixture of experts" (inference.shantanugoel.com), section "Dispatch": after the
// assignments are sorted by expert, each expert runs on its contiguous slice of rows, and a
// grouped GEMM does all of these independent matmuls of different sizes in one launch.
// The expert is down(silu(gate x) * up x) with gate_up [E, 2I, D] (gate rows first) and
// down [E, D, I].  The router logits x W_r^T are a plain dense GEMM of the same shape class.
//
// Layout of the work (swap-AB): a tile is 128 weight rows (the MMA's M) by up to BN tokens
// (its N), so an expert with few tokens costs a narrow N instead of a padded 128-row M.
//   gate_up, narrow tiles (BN = 64, decode): two accumulators per tile, gate rows
//            [f0, f0+128) and the matching up rows [I+f0, ...), against the same token tile;
//            TMEM lane f holds gate and up of feature f, and the epilogue writes
//            h = silu(g) * u in bf16.
//   gate_up, wide tiles (BN = 256): one accumulator whose 128 rows interleave gate and up
//            of 64 features in groups of 16 (fetched by one 5-D TMA load); lane l and lane
//            l+16 of a lane quarter hold gate and up of one feature and swap halves with a
//            shuffle.  A tcgen05.mma costs its issuing thread roughly the same whatever N,
//            so N = 256 halves the instructions of the two-accumulator layout at N = 128.
//   down:    one accumulator, down rows [d0, d0+128) against a tile of h rows; the epilogue
//            scales by the routing weight and stores FP32 into the token's slot (a bf16 slot
//            would add a third bf16 rounding on top of h and the output).
//   router:  one accumulator, router rows [e0, e0+128) against a tile of x rows over one
//            of ksplit slices of K; FP32 partial sums out (added in slice order, with the
//            bias, by the selection), so that a handful of token tiles still fills the SMs.
//
// Per CTA (one per SM, persistent over a device-side item list):
//   warp 0      TMA producer: ring of STAGES stages {A tile(s) 128x64, B tile BNx64} of bf16
//               in the 128-byte swizzle layout, completion counted on an mbarrier;
//   warp 1      allocates TMEM, and one thread issues tcgen05.mma (M=128, N=tile width,
//               K=16 x 4 per stage) with FP32 accumulation in TMEM; tcgen05.commit frees a
//               stage when its MMAs are done and publishes an accumulator when a tile is;
//   warps 2..9  epilogue: two warps per TMEM lane quarter (a warp may only read the quarter
//               warp % 4), taking alternate 32-column chunks of the tile: tcgen05.ld, apply
//               the epilogue, store; accumulators are double-buffered so the next tile's
//               MMAs overlap this epilogue.
// All mbarrier waits are bounded (common.cuh); on expiry the kernel records the fact in the
// device error word and winds down without leaving TMEM allocated.
#include <cstdlib>
#include <mutex>

#include "common.cuh"

namespace moe {

enum { kModeGateUp = 0, kModeDown = 1, kModeRouter = 2 };

constexpr int kEpiWarps = 8;
constexpr int kConvWarps = 4;      // F8: warps that widen FP8 weight tiles to bf16
constexpr int kQD = 4;             // entries of the claimed-unit ring (narrow tiles)
constexpr int kBarRegion = 512;    // bytes of mbarriers and small shared state

// One kernel configuration: mode, token columns per tile, pipeline depth, CTA pairs, and
// whether the weights arrive as FP8 E4M3 with a scale per weight row (F8).
template <int MODE, int BN_, int STAGES_, bool PAIR_ = false, bool F8_ = false>
struct TcCfg {
    static constexpr int BN = BN_, STAGES = STAGES_;
    // PAIR: two CTAs of a cluster share M = 256 MMAs; each holds 128 weight rows and half of
    // the tile's BN token rows (BNC), and its TMEM holds its 128 rows over all BN columns
    static constexpr bool PAIR = PAIR_;
    static constexpr int BNC = PAIR ? BN / 2 : BN;
    // gate_up: narrow tiles keep gate and up in two accumulators (two A tiles per stage);
    // wide tiles interleave them in one A tile and one accumulator
    static constexpr bool IL = MODE == kModeGateUp && BN > kNarrowBN;
    static constexpr int NA = (MODE == kModeGateUp && !IL) ? 2 : 1;   // A tiles per stage
    static constexpr int ACC = NA * BN;                       // TMEM columns per accumulator set
    // two accumulator sets, rounded up to the power-of-two allocation unit (>= 32 columns)
    static constexpr int TMEM = 2 * ACC <= 32 ? 32 : 2 * ACC <= 64 ? 64 : 2 * ACC <= 128 ? 128
                              : 2 * ACC <= 256 ? 256 : 512;
    static_assert(2 * ACC <= 512, "accumulators exceed TMEM");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "token tile");
    // F8: the weight tiles of a stage arrive as FP8 bytes (64 per row per K step, no swizzle)
    // in the load ring; converter warps widen them (exactly) to bf16 into a ring of CONV
    // 128-byte-swizzled stages, copy the stage's bf16 token tile next to them and release the
    // load stage at once, so the loads in flight do not wait for the MMAs; the MMAs read the
    // bf16 ring.
    static constexpr bool F8 = F8_;
    static_assert(!F8 || (!PAIR && !IL && MODE != kModeRouter), "FP8 weights: narrow tiles only");
    static constexpr int CONV = F8 ? (NA == 2 ? 2 : 3) : 0;
    static constexpr int A_BYTES = NA * kTcM * kTcK * (F8 ? 1 : 2);   // weight bytes per load stage
    static constexpr int SB = A_BYTES + BNC * kTcK * 2;              // bytes per load stage
    static constexpr int CSB = NA * kTcM * kTcK * 2 + BNC * kTcK * 2;   // bf16 stage (F8)
    static constexpr int CONVB = CONV * CSB;                           // bf16 ring (F8)
    static constexpr int THREADS = (2 + kEpiWarps + (F8 ? kConvWarps : 0)) * 32;
    static constexpr int SMEM = STAGES * SB + CONVB + 1024 + kBarRegion + (int)sizeof(SmemTables) +
                                (MODE == kModeDown ? 8 * 2 * 4 * BN : 0);
    static_assert(SB % 1024 == 0, "stages keep the 1024-byte alignment of swizzled tiles");
    static_assert((2 * STAGES + 6) * 8 + kQD * 20 + 2 * CONV * 8 <= kBarRegion, "barrier region");
    static_assert(SMEM <= 232448, "shared memory per block");
};

constexpr int kATileBytes = kTcM * kTcK * 2;  // 16 KB
constexpr int kA8TileBytes = kTcM * kTcK;     // 8 KB (FP8)

struct TileInfo {
    int bi;       // token-operand box: 16 << bi rows
    int shared;   // A comes from the shared-expert tensor map
    int a_row0;   // first A row (gate rows for gate_up; interleaved: 16-feature group)
    int a_row1;   // first up row (gate_up; interleaved: expert)
    int b_row;    // first B (token) row
    int n_valid;  // valid token columns, 1..BN
    int nk;       // K stages
    int k0;       // first K stage of this unit
    int split;    // K slice index (router slices, or a split tail item's slice)
    int nsplit;   // > 1: tail item split over K, partial sums reduced by the last slice
    int tail;     // index of a split item among the tail items
    int seg;      // segment (expert; E = the shared expert)
    int m0;       // first output feature of this tile within its segment
};

// Work schedule of one launch (identical in every CTA): the first `full` items -- whole
// waves of G = gridDim.x -- run one item per unit; when the remaining tail is at most half a
// wave, each tail item is split along K into S slices so that no CTA ends a whole item
// after the others.  The slices come last (at most one per CTA): their reduction then reads
// L2 while the SM's TMA engine is idle -- mid-stream, those loads would queue behind the
// weight traffic.  A slice writes FP32 partial accumulators; the last slice of an item to
// finish (atomic ticket) adds them in slice order and runs the epilogue, so the sums do not
// depend on timing.
struct Sched {
    int n;      // items
    int full;   // items in whole waves
    int S;      // slices per tail item (1: no split)
    int units;  // work units
};

template <int MODE, int BN>
__device__ __forceinline__ int tc_total_items(const TcArgs& a, const SmemTables* st) {
    if (MODE == kModeRouter) return ((a.T + BN - 1) / BN) * ((a.E + kTcM - 1) / kTcM) * a.ksplit;
    return st->prefix[a.nseg];
}

template <int MODE, int BN, bool SPLIT>
__device__ __forceinline__ Sched tc_schedule(const TcArgs& a, const SmemTables* st, int G) {
    Sched sc;
    sc.n = tc_total_items<MODE, BN>(a, st);
    sc.full = sc.n / G * G;
    sc.S = 1;
    const int tail = sc.n - sc.full;
    if (SPLIT && tail > 0 && 2 * tail <= G) {
        const int kmin = MODE == kModeGateUp ? a.D : (a.I_s > 0 ? min(a.I, a.I_s) : a.I);
        int S = min(G / tail, kMaxKSplit);
        S = min(S, kmin / kTcK);
        S = min(S, a.partial_slots / tail);
        if (S >= 2) sc.S = S;
    }
    sc.units = sc.full + tail * sc.S;
    return sc;
}

// Smallest token box (16 << bi rows, bi <= log2(BN/16)) that covers n valid rows.
template <int BN>
__device__ __forceinline__ int box_index(int n) {
    int bi = 0;
    while ((16 << bi) < n && (16 << bi) < BN) ++bi;
    return bi;
}

// Work item -> tile.  PAIR: the pair's tile covers 128 features (gate_up) or 256 down rows
// and up to BN tokens; `rank` selects this CTA's half of the weight rows (its m0 and A rows);
// b_row and n_valid describe the whole tile, bi the per-CTA token box (half the tile's rows).
template <int MODE, int BN, bool PAIR = false>
__device__ __forceinline__ TileInfo tc_decode_item(const TcArgs& a, const SmemTables* st, int item,
                                                   int rank = 0) {
    TileInfo ti;
    ti.k0 = 0;
    ti.split = 0;
    ti.nsplit = 1;
    ti.tail = 0;
    ti.seg = 0;
    if (MODE == kModeRouter) {
        // consecutive items are the K splits of one tile
        const int mtc = (a.E + kTcM - 1) / kTcM;
        ti.split = item % a.ksplit;
        item /= a.ksplit;
        const int tt = item / mtc, mt = item % mtc;
        ti.shared = 0;
        ti.a_row0 = mt * kTcM;
        ti.a_row1 = 0;
        ti.b_row = tt * BN;
        ti.n_valid = min(BN, a.T - tt * BN);
        const int nkt = a.D / kTcK;
        ti.k0 = ti.split * nkt / a.ksplit;
        ti.nk = (ti.split + 1) * nkt / a.ksplit - ti.k0;
        ti.m0 = mt * kTcM;
        ti.bi = box_index<BN>(ti.n_valid);
        return ti;
    }
    const int s = find_segment_smem(st->prefix, a.nseg, item);
    const int local = item - st->prefix[s];
    ti.seg = s;
    const int sh = (s == a.E);
    const int Iseg = sh ? a.I_s : a.I;
    // weight rows per tile: features (gate_up) or down rows; the pair's tile is twice a CTA's
    const int fpt = (MODE == kModeGateUp && BN > kNarrowBN) ? kGuILFeatures : kTcM;
    const int mtc = (MODE == kModeGateUp) ? Iseg / (fpt * (PAIR ? 2 : 1)) : a.D / (kTcM * (PAIR ? 2 : 1));
    const int tt = local / mtc, mt = local % mtc;
    const int cnt = st->count[s];
    const int start = st->start[s];
    ti.shared = sh;
    ti.b_row = start + tt * BN;
    ti.n_valid = min(BN, cnt - tt * BN);
    ti.m0 = (MODE == kModeGateUp) ? (mt * (PAIR ? 2 : 1) + rank) * fpt : (mt * (PAIR ? 2 : 1) + rank) * kTcM;
    if (MODE == kModeGateUp && BN > kNarrowBN) {
        // interleaved: 64 features [m0, m0+64) of expert s, as four 16-feature groups
        ti.a_row0 = ti.m0 / 16;
        ti.a_row1 = sh ? 0 : s;
        ti.nk = a.D / kTcK;
    } else if (MODE == kModeGateUp) {
        const int base = sh ? 0 : s * 2 * a.I;
        ti.a_row0 = base + mt * kTcM;
        ti.a_row1 = base + Iseg + mt * kTcM;
        ti.nk = a.D / kTcK;
    } else {
        const int base = sh ? 0 : s * a.D;
        ti.a_row0 = base + ti.m0;
        ti.a_row1 = 0;
        ti.nk = Iseg / kTcK;
    }
    ti.bi = PAIR ? box_index<BN / 2>((ti.n_valid + 1) / 2) : box_index<BN>(ti.n_valid);
    return ti;
}

template <int MODE, int BN, bool PAIR = false>
__device__ __forceinline__ TileInfo tc_decode_unit(const TcArgs& a, const SmemTables* st,
                                                   const Sched& sc, int u, int rank = 0) {
    if (sc.S == 1 || u < sc.full) return tc_decode_item<MODE, BN, PAIR>(a, st, u, rank);
    const int tail = (u - sc.full) / sc.S, split = (u - sc.full) % sc.S;
    TileInfo ti = tc_decode_item<MODE, BN, PAIR>(a, st, sc.full + tail, rank);
    const int nkt = ti.nk;
    ti.k0 = split * nkt / sc.S;
    ti.nk = (split + 1) * nkt / sc.S - ti.k0;
    ti.split = split;
    ti.nsplit = sc.S;
    ti.tail = tail;
    return ti;
}

// gate_up -> down hand-off per expert (narrow tiles).  The signalling warp has written h
// with ordinary stores; the down kernel reads h with TMA (the async proxy), hence the proxy
// fence on both sides.
__device__ __forceinline__ void signal_segment_done(const TcArgs& a, int seg, int lane) {
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __threadfence();
    __syncwarp();
    if (lane == 0) {
        atomicAdd(a.seg_done + seg, 1);
        atomicAdd(a.seg_done + a.nseg, 1);
    }
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait of the down producer (one lane) until gate_up has finished segment seg.
__device__ __forceinline__ bool wait_segment_done(const TcArgs& a, int seg, bool& all_done) {
    if (all_done) return true;
    const int all_target = 8 * __ldg(a.gu_prefix + a.nseg);
    const int target = 8 * (__ldg(a.gu_prefix + seg + 1) - __ldg(a.gu_prefix + seg));
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (ld_acquire(a.seg_done + a.nseg) >= all_target) {
            all_done = true;
            break;
        }
        if (ld_acquire(a.seg_done + seg) >= target) break;
        __nanosleep(128);
        if (globaltimer_ns() - t0 > a.wait_ns) {
            set_error(a.err, kErrWaitProducer);
            return false;
        }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

// Plain 2-D TMA load without an L2 hint.
__device__ __forceinline__ void tma_load(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                         int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

template <int MODE, int BN, int STAGES, bool PAIR = false, bool F8 = false>
__global__ void __launch_bounds__((TcCfg<MODE, BN, STAGES, PAIR, F8>::THREADS), 1)
    tc_gemm_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    using Tr = TcCfg<MODE, BN, STAGES, PAIR, F8>;
    constexpr int NA = Tr::NA, ACC = Tr::ACC;
    constexpr bool SPLIT = MODE != kModeRouter && BN <= kNarrowBN;
    // DYN (narrow tiles): CTA b starts with unit b; each further unit is claimed from a
    // counter in global memory (units grid, grid + 1, ... in claiming order), one ahead, by
    // the producer, which hands each to the MMA issuer and the epilogue warps through a ring
    // of kQD entries; CTAs that run faster (or draw lighter units) take more of them.
    // Otherwise CTA (pair) b takes units b, b + grid, ...
    constexpr bool DYN = SPLIT;
    constexpr int SB = Tr::SB;
    constexpr int CONVD = Tr::CONV > 0 ? Tr::CONV : 1;   // the bf16 ring's size as a divisor
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* convs = smem + STAGES * SB;   // F8: CONV bf16 stages (NA weight tiles, token tile)
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SB + Tr::CONVB);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;  // [2]
    uint64_t* tempty = tfull + 2;       // [2]
    uint64_t* drain = tempty + 2;       // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    // narrow tiles: ring of claimed units (see DYN below), after the TMEM slot
    uint64_t* qfull = drain + 2;                            // [kQD]
    uint64_t* qempty = qfull + kQD;                         // [kQD]
    int* qitem = reinterpret_cast<int*>(qempty + kQD);      // [kQD]
    uint64_t* conv = reinterpret_cast<uint64_t*>(qitem + kQD);   // [CONV] (F8)
    uint64_t* cempty = conv + Tr::CONV;                          // [CONV] (F8)
    SmemTables* tabs = reinterpret_cast<SmemTables*>(smem + STAGES * SB + Tr::CONVB + kBarRegion);
    // down: per epilogue warp, the current tile's row destinations and weights
    int* ep_dest_all = reinterpret_cast<int*>(tabs + 1);                       // [8][BN]
    float* ep_wt_all = reinterpret_cast<float*>(ep_dest_all + kEpiWarps * BN);  // [8][BN]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // work units are handed to CTAs, or (PAIR) to the clusters of two CTAs, round-robin
    const int rank = PAIR ? (int)cluster_ctarank() : 0;
    const int ublk = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int ugrid = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    // prologue: independent of earlier kernels, overlaps them under launch chaining
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, F8 ? kConvWarps : 1);   // F8: released by the converter warps
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, (PAIR ? 2 : 1) * kEpiWarps * 32);  // PAIR: both CTAs' epilogues
        }
        mbar_init(drain, 1);
        for (int q = 0; q < kQD; ++q) {
            mbar_init(qfull + q, 1);
            // the MMA thread, each epilogue warp and (F8) each converter warp
            mbar_init(qempty + q, 1 + kEpiWarps + (F8 ? kConvWarps : 0));
        }
        for (int c = 0; c < Tr::CONV; ++c) {
            mbar_init(conv + c, kConvWarps);   // a converted tile: one arrival per converter warp
            mbar_init(cempty + c, 1);          // its MMAs are complete (commit)
        }
        mbar_fence_init();
    }
    if (warp == 0 && lane < 2 + kNumBBoxes) {
        const CUtensorMap* m = lane == 0 ? (F8 ? &maps.A8 : &maps.A)
                                         : (lane == 1 ? &maps.A_shared : &maps.B[lane - 2]);
        tma_prefetch_desc(m);
    }
    if (warp == 1) {
        if (PAIR)
            tmem_alloc_pair(tmem_slot, Tr::TMEM);
        else
            tmem_alloc(tmem_slot, Tr::TMEM);
    }
    if (MODE == kModeDown) {
        // The work tables come from the permutation, two kernels back: it completed before
        // the gate_up kernel (this kernel's predecessor) passed its own dependency wait,
        // which precedes the moment this kernel can start.  So they are read (through L2)
        // before this kernel's wait, and this CTA's first tile of weights -- which does not
        // depend on gate_up -- is requested into L2 while gate_up finishes.
        load_tables(tabs, a.tables.dn_items, a.tables.seg_count, a.tables.seg_start, a.nseg);
        __syncthreads();
        if (warp == 0 && lane == 0 && ublk < tabs->prefix[a.nseg]) {
            const TileInfo t0 = tc_decode_item<MODE, BN, PAIR>(a, tabs, ublk, rank);
            const CUtensorMap* mA = t0.shared ? &maps.A_shared : (F8 ? &maps.A8 : &maps.A);
            for (int kb = 0; kb < t0.nk; ++kb) tma_prefetch_l2(mA, kb * kTcK, t0.a_row0);
        }
    }
    // (down with per-expert hand-off: no wait for the whole gate_up grid; everything read
    // below besides h was complete before this kernel could start -- see above)
    if (MODE == kModeGateUp && DYN && a.spec_steps > 0 && warp == 0 && lane == 0) {
        const int mt = a.I / kTcM;
        const int e = (int)blockIdx.x / mt;
        if (e < a.E) {
            const int r0 = e * 2 * a.I + ((int)blockIdx.x % mt) * kTcM;
            for (int kb = 0; kb < a.spec_steps; ++kb) {
                tma_prefetch_l2(F8 ? &maps.A8 : &maps.A, kb * kTcK, r0);
                tma_prefetch_l2(F8 ? &maps.A8 : &maps.A, kb * kTcK, r0 + a.I);
            }
        }
    }
    // (gate_up lets down start only after its own wait, which down's early reads of the work
    // tables rely on -- see above)
    if (!(MODE == kModeDown && a.dep_wait)) pdl_wait();
    pdl_launch_dependents();
    if (MODE == kModeGateUp)
        load_tables(tabs, a.tables.gu_items, a.tables.seg_count, a.tables.seg_start, a.nseg);
    tc_fence_before();
    if (PAIR)
        cluster_sync_all();   // both CTAs' barriers exist before any cross-CTA arrive or load
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const Sched sc = tc_schedule<MODE, BN, SPLIT>(a, tabs, ugrid);
    const int total = sc.units;

    if (!DYN && ublk >= total) {
        // no work for this CTA: nothing was issued; fall through to the TMEM release
    } else if (warp == 0) {
        // ------------------------------------------------------------ TMA producer warp
        // Weight tiles are issued by lane 0.  Token tiles: in gather mode gate_up fetches its
        // rows from x by row_token, lane i taking rows 4i..4i+3 of the tile (rows past the
        // segment repeat its last row; their columns are never used); otherwise lane 0 loads
        // a tile of the permuted rows.
        const int first = ublk, step = ugrid;   // this CTA's (pair's) units
        bool dep_all_done = false;
        int it = 0;
        bool ok = true;
        int last_round[STAGES];
#pragma unroll
        for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
        const bool gather = MODE == kModeGateUp && a.gather;
        // the next unit's gather rows are loaded while the current unit's stages are issued
        auto gather_rows = [&](const TileInfo& t, int (&g)[4]) {
            const int base = t.b_row + 4 * lane;
            const int last = t.b_row + t.n_valid - 1;
#pragma unroll
            for (int q = 0; q < 4; ++q) g[q] = __ldg(a.row_token + min(base + q, last));
        };
        TileInfo tn{};
        int gn[4] = {0, 0, 0, 0};
        if (!DYN && first < total) {
            tn = tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, first, rank);
            if (gather) gather_rows(tn, gn);
        }
        // DYN: the unit claimed for after the current one; the first is the CTA's own index
        // (no claim), later ones come from the counter, numbered from the grid size on
        int next = (int)blockIdx.x;
        for (int item = first, qi = 0; ok; item += DYN ? 0 : step, ++qi) {
            if (DYN) {
                // publish the claimed unit (or the end, -1) to the MMA and epilogue warps
                item = __shfl_sync(0xffffffffu, next, 0);
                const int qs = qi % kQD;
                const bool gq = mbar_wait(qempty + qs, ((qi / kQD) & 1) ^ 1, a.err, kErrWaitProducer, a.wait_ns);
                if (!__all_sync(0xffffffffu, gq)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    qitem[qs] = item < total ? item : -1;
                    mbar_arrive(qfull + qs);
                }
                if (item >= total) break;
                tn = tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, item, rank);
                if (gather) gather_rows(tn, gn);
            } else if (item >= total) {
                break;
            }
            const TileInfo ti = tn;
            const int g0 = gn[0], g1 = gn[1], g2 = gn[2], g3 = gn[3];
            if (!DYN && item + step < total) {
                tn = tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, item + step, rank);
                if (gather) gather_rows(tn, gn);
            }
            if (MODE == kModeDown && a.dep_wait) {
                bool got = true;
                if (lane == 0) got = wait_segment_done(a, ti.seg, dep_all_done);
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
            }
            const CUtensorMap* mA = ti.shared ? &maps.A_shared : (F8 ? &maps.A8 : &maps.A);
            const CUtensorMap* mB = &maps.B[ti.bi];
            const int brows = 16 << ti.bi;
            // PAIR: the leader's barrier counts both CTAs' bytes (same geometry in each)
            const uint32_t bytes = (PAIR ? 2u : 1u) * (Tr::A_BYTES + (uint32_t)brows * kTcK * 2);
            for (int kb = 0; kb < ti.nk; ++kb, ++it) {
                const int s = it % STAGES;
                const int round = it / STAGES;
                const bool got = mbar_wait(empty + s, (round & 1) ^ 1, a.err, kErrWaitProducer, a.wait_ns);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + s * SB;
                if (PAIR && lane == 0) {
                    // both CTAs load their halves; completion is counted by the leader
                    if (rank == 0) mbar_arrive_expect_tx(full + s, bytes);
                    const uint32_t fb = mapa_shared(full + s, 0);
                    const int kx = (ti.k0 + kb) * kTcK;
                    if (Tr::IL)
                        tma_load_5d_pair(st, mA, fb, kx, 0, 0, ti.a_row0, ti.a_row1);
                    else
                        tma_load_2d_pair(st, mA, fb, kx, ti.a_row0);
                    tma_load_2d_pair(st + Tr::A_BYTES, mB, fb, kx, ti.b_row + rank * brows);
                } else if (!PAIR && lane == 0) {
                    mbar_arrive_expect_tx(full + s, bytes);
                    const int kx = (ti.k0 + kb) * kTcK;
                    if (Tr::IL)
                        tma_load_5d(st, mA, full + s, kx, 0, 0, ti.a_row0, ti.a_row1);
                    else
                        tma_load(st, mA, full + s, kx, ti.a_row0);
                    if (NA == 2) tma_load(st + Tr::A_BYTES / 2, mA, full + s, kx, ti.a_row1);
                    if (!gather) tma_load(st + Tr::A_BYTES, mB, full + s, kx, ti.b_row);
                }
                if (gather) {
                    __syncwarp();  // expect_tx is posted before any gather can complete
                    if (4 * lane < brows)
                        tma_gather4(st + Tr::A_BYTES + lane * 4 * kTcK * 2, mB, full + s,
                                    (ti.k0 + kb) * kTcK, g0, g1, g2, g3);
                }
#pragma unroll
                for (int q = 0; q < STAGES; ++q)
                    if (q == s) last_round[q] = round;
                // DYN: the next unit is claimed once this one's first stage is on its way, so
                // that at the start every CTA holds one unit before any holds two
                if (DYN && kb == 0 && lane == 0)
                    next = total <= (int)gridDim.x ? total : (int)gridDim.x + atomicAdd(a.sched, 1);
            }
        }
        // wait until the MMA issuer has released every stage, then until every issued
        // load has landed, so no copy is in flight when the CTA exits
        if (ok) {
            for (int i = 0; i < STAGES; ++i, ++it) {
                const int s = it % STAGES;
                const int round = it / STAGES;
                const bool got = mbar_wait(empty + s, (round & 1) ^ 1, a.err, kErrWaitTail, a.wait_ns);
                if (!__all_sync(0xffffffffu, got)) break;
            }
        }
        // (PAIR: a released stage implies its loads landed; the full barriers are the leader's)
        if (!PAIR) {
#pragma unroll
            for (int s = 0; s < STAGES; ++s)
                if (last_round[s] >= 0) mbar_wait(full + s, last_round[s] & 1, a.err, kErrWaitTail, a.wait_ns);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (PAIR: the leader CTA's thread issues the pair's M = 256 MMAs)
        if (lane == 0 && rank == 0) {
            const uint32_t idesc0 = umma_idesc_bf16_f32(PAIR ? 2 * kTcM : kTcM, 16) & ~(0x3Fu << 17);
            // shared-memory descriptors of stage 0; stage s adds s * SB / 16 to the address
            // field (stages stay below 256 KB, so the 14-bit field does not carry)
            // (F8: both operands are read from the bf16 ring, slot c adds c * CSB / 16)
            const uint64_t dA0 = umma_desc_sw128(F8 ? convs : smem);
            const uint64_t dA1 = umma_desc_sw128((F8 ? convs : smem) + kATileBytes);
            const uint64_t dB = umma_desc_sw128(F8 ? convs + NA * kATileBytes : smem + Tr::A_BYTES);
            int s = 0, phase = 0;   // ring position of the next stage
            int pos = 0;            // F8: stages consumed so far (the bf16 ring follows them)
            int tc = 0;
            bool ok = true;
            for (int item = ublk, qi = 0; ok; item += DYN ? 0 : ugrid, ++tc, ++qi) {
                if (DYN) {
                    const int qs = qi % kQD;
                    if (!mbar_wait(qfull + qs, (qi / kQD) & 1, a.err, kErrWaitMma, a.wait_ns)) break;
                    item = qitem[qs];
                    mbar_arrive(qempty + qs);
                    if (item < 0) break;
                } else if (item >= total) {
                    break;
                }
                const TileInfo ti = tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, item, rank);
                const int b = tc & 1;
                const int use = tc >> 1;
                if (!mbar_wait(tempty + b, (use & 1) ^ 1, a.err, kErrWaitMma, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                int n = (ti.n_valid + 15) & ~15;
                n = n < 16 ? 16 : (n > BN ? BN : n);
                if (PAIR) n = 2 * (16 << ti.bi);   // both CTAs' token boxes
                const uint32_t idesc = idesc0 | ((uint32_t)(n >> 3) << 17);
                const uint32_t d0 = tmem_base + (uint32_t)(b * ACC);
                for (int kb = 0; kb < ti.nk; ++kb) {
                    // (F8: the converted stage holds both operands; the load stage may already
                    // hold a later stage, so its barrier is not looked at)
                    const int cs = F8 ? pos % CONVD : 0;
                    if (!(F8 ? mbar_wait(conv + cs, (pos / CONVD) & 1, a.err, kErrWaitMma, a.wait_ns)
                             : mbar_wait(full + s, phase, a.err, kErrWaitMma, a.wait_ns))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t off = F8 ? (uint64_t)(cs * (Tr::CSB >> 4)) : (uint64_t)(s * (SB >> 4));
                    const uint64_t da0 = dA0 + off, da1 = dA1 + off, db = dB + off;
                    if (PAIR) {
                        umma_bf16_pair(d0, da0, db, idesc, kb);
#pragma unroll
                        for (int kk = 1; kk < kTcK / 16; ++kk)
                            umma_bf16_pair_acc(d0, da0 + 2 * kk, db + 2 * kk, idesc);
                        umma_commit_pair_both(empty + s);   // frees the stage in both CTAs
                    } else {
                        umma_bf16(d0, da0, db, idesc, kb);  // the tile's first MMA overwrites D
                        if (NA == 2) umma_bf16(d0 + BN, da1, db, idesc, kb);
#pragma unroll
                        for (int kk = 1; kk < kTcK / 16; ++kk) {
                            umma_bf16_acc(d0, da0 + 2 * kk, db + 2 * kk, idesc);
                            if (NA == 2) umma_bf16_acc(d0 + BN, da1 + 2 * kk, db + 2 * kk, idesc);
                        }
                        if (F8)
                            umma_commit(cempty + cs);   // the bf16 stage is free again
                        else
                            umma_commit(empty + s);
                    }
                    if (F8) ++pos;
                    if (++s == STAGES) {
                        s = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                if (PAIR)
                    umma_commit_pair_both(tfull + b);
                else
                    umma_commit(tfull + b);
            }
            // every issued MMA must be complete before TMEM is released
            if (PAIR)
                umma_commit_pair_local(drain);
            else
                umma_commit(drain);
            mbar_wait(drain, 0, a.err, kErrWaitMma, a.wait_ns);
        }
    } else if (F8 && warp >= 2 + kEpiWarps) {
        // ------------------------------------------------------------ converter warps (F8)
        // Each stage's FP8 weight tiles (NA x 128 rows x 64 bytes, row-major) become bf16
        // tiles in the 128-byte-swizzled K-major layout the MMAs read (the layout a TMA load
        // with 128-byte swizzle writes: 16-byte chunk c of row r at r * 128 + ((c ^ (r % 8))
        // * 16)).  Converter thread t takes the 16-byte pieces t, t + 32 * kConvWarps, ... of the stage
        // (piece = row * 4 + j within a tile), widens its 16 values and stores them as the
        // row's chunks 2j and 2j + 1.  Units come from the ring like the epilogue's.
        static_assert(512 % (kConvWarps * 32) == 0, "converter threads divide a tile's pieces");
        const int ct = (warp - 2 - kEpiWarps) * 32 + lane;   // 0 .. kConvWarps * 32 - 1
        int pos = 0;
        bool ok = true;
        for (int qi = 0; ok; ++qi) {
            const int qs = qi % kQD;
            const bool gq = mbar_wait(qfull + qs, (qi / kQD) & 1, a.err, kErrWaitEpilogue, a.wait_ns);
            if (!__all_sync(0xffffffffu, gq)) break;
            const int item = qitem[qs];
            __syncwarp();
            if (lane == 0) mbar_arrive(qempty + qs);
            if (item < 0) break;
            const TileInfo ti = tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, item, rank);
            for (int kb = 0; kb < ti.nk; ++kb, ++pos) {
                const int s = pos % STAGES, cs = pos % CONVD;
                bool got = mbar_wait(full + s, (pos / STAGES) & 1, a.err, kErrWaitEpilogue, a.wait_ns);
                if (got)
                    got = mbar_wait(cempty + cs, ((pos / CONVD) & 1) ^ 1, a.err, kErrWaitEpilogue, a.wait_ns);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const uint8_t* src = smem + s * SB;
                uint8_t* dst = convs + cs * Tr::CSB;
#pragma unroll
                for (int q = 0; q < NA * 512 / (kConvWarps * 32); ++q) {
                    const int piece = q * (kConvWarps * 32) + ct;
                    const int at = piece >> 9, pr = piece & 511;
                    const int row = pr >> 2, j = pr & 3;
                    const uint4 v = *reinterpret_cast<const uint4*>(src + at * kA8TileBytes + row * 64 + j * 16);
                    uint4 lo, hi;
                    widen_e4m3x16(v, lo, hi);
                    uint8_t* drow = dst + at * kATileBytes + row * 128;
                    *reinterpret_cast<uint4*>(drow + (((2 * j) ^ (row & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4*>(drow + (((2 * j + 1) ^ (row & 7)) << 4)) = hi;
                }
                // the token tile (bf16, already in its swizzled layout, which depends only on
                // the 1024-byte-aligned position) is copied next to the widened weights
                {
                    const uint4* bsrc = reinterpret_cast<const uint4*>(src + Tr::A_BYTES);
                    uint4* bdst = reinterpret_cast<uint4*>(dst + NA * kATileBytes);
                    constexpr int kBChunks = BN * kTcK * 2 / 16;
#pragma unroll
                    for (int i = ct; i < kBChunks; i += kConvWarps * 32) bdst[i] = bsrc[i];
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(empty + s);   // the load stage has been read
                    mbar_arrive(conv + cs);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue warps 2..9
        const int quarter = warp & 3;
        const int ew = warp - 2;               // epilogue warp 0..7
        const int half = ew >> 2;              // which alternate chunks this warp takes
        const int row = quarter * 32 + lane;  // TMEM lane = weight row within the tile
        int* ep_dest = ep_dest_all + ew * BN;
        float* ep_wt = ep_wt_all + ew * BN;
        // down, wide tiles: the slot destinations and routing weights of the token columns
        // this warp stores (its chunks half, half + 2, ...) are loaded one tile ahead into
        // registers (nd, nw), so their memory latency overlaps the previous tile's epilogue
        // (measured: it helps the long-K wide tiles and costs the short narrow ones); the
        // current tile's copy (cd, cw) stays in registers and reaches the lanes by shuffles,
        // keeping the per-element work off shared memory, which the MMAs read their
        // operands from
        constexpr bool kAhead = MODE == kModeDown && BN > kNarrowBN;
        constexpr int kCPW = (BN + 63) / 64;   // chunks per epilogue warp
        int nd[kCPW] = {}, cd[kCPW] = {};
        float nw[kCPW] = {}, cw[kCPW] = {};
        // The epilogue of one 32-column chunk: v (and u, the up accumulator) hold row `row`.
        auto finish_chunk = [&](const TileInfo& ti, int c, const float* v, const float* u) {
            if (Tr::IL) {
                // lanes 0-15 of the quarter hold gate rows of features m0 + 16*quarter + l,
                // lanes 16-31 the up rows of the same features: lane l takes the chunk's tokens
                // 0-15, lane l+16 tokens 16-31, swapping the other half with its partner
                const bool is_gate = (lane & 16) == 0;
                const int f = ti.m0 + 16 * quarter + (lane & 15);
                const int t0 = c * 32 + (is_gate ? 0 : 16);
                uint16_t* hp = a.h + (size_t)(ti.b_row + t0) * a.ld_h + f;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float send = is_gate ? v[16 + t] : v[t];
                    const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
                    const float g = is_gate ? v[t] : recv;
                    const float uu = is_gate ? recv : v[16 + t];
                    if (t0 + t < ti.n_valid) hp[(size_t)t * a.ld_h] = to_bf16_bits(silu(g) * uu);
                }
            } else if (MODE == kModeGateUp) {
                const int f = ti.m0 + row;
                uint16_t* hp = a.h + (size_t)(ti.b_row + c * 32) * a.ld_h + f;
                // F8: the accumulators hold sums of q * x; the row scales make them g and u
                const float sg = F8 ? __ldg(a.a_scale + ti.a_row0 + row) : 1.0f;
                const float su = F8 ? __ldg(a.a_scale + ti.a_row1 + row) : 1.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (c * 32 + j < ti.n_valid)
                        hp[(size_t)j * a.ld_h] = F8 ? to_bf16_bits(silu(v[j] * sg) * (u[j] * su))
                                                    : to_bf16_bits(silu(v[j]) * u[j]);
            } else if (MODE == kModeDown) {
                const int d = ti.m0 + row;
                if (kAhead) {
                    // lane j holds column c*32 + j of this warp's chunk (c - half) / 2
                    const int i = (c - half) >> 1;
                    int dsel = cd[0];
                    float wsel = cw[0];
#pragma unroll
                    for (int q = 1; q < kCPW; ++q)
                        if (q == i) {
                            dsel = cd[q];
                            wsel = cw[q];
                        }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int dj = __shfl_sync(0xffffffffu, dsel, j);
                        const float wj = __shfl_sync(0xffffffffu, wsel, j);
                        if (c * 32 + j < ti.n_valid) a.slots[(size_t)dj * a.D + d] = wj * v[j];
                    }
                } else {
                    const float sd = F8 ? __ldg(a.a_scale + ti.a_row0 + row) : 1.0f;   // F8 row scale
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c * 32 + j;
                        if (col < ti.n_valid)
                            a.slots[(size_t)ep_dest[col] * a.D + d] = ep_wt[col] * (F8 ? v[j] * sd : v[j]);
                    }
                }
            } else {
                const int e = ti.m0 + row;
                if (e < a.E) {
                    float* part = a.logits + (size_t)ti.split * a.T * a.E;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int t = ti.b_row + c * 32 + j;
                        if (c * 32 + j < ti.n_valid) part[(size_t)t * a.E + e] = v[j];
                    }
                }
            }
        };
        // The same for four columns 4g..4g+3 of chunk c (the split-tail reduction).
        auto finish_quad = [&](const TileInfo& ti, int c, int g, const float4& v4, const float4& u4) {
            const float v[4] = {v4.x, v4.y, v4.z, v4.w};
            const float u[4] = {u4.x, u4.y, u4.z, u4.w};
            const int col0 = c * 32 + 4 * g;
            if (MODE == kModeGateUp) {
                uint16_t* hp = a.h + (size_t)(ti.b_row + col0) * a.ld_h + ti.m0 + row;
                const float sg = F8 ? __ldg(a.a_scale + ti.a_row0 + row) : 1.0f;
                const float su = F8 ? __ldg(a.a_scale + ti.a_row1 + row) : 1.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (col0 + j < ti.n_valid)
                        hp[(size_t)j * a.ld_h] = F8 ? to_bf16_bits(silu(v[j] * sg) * (u[j] * su))
                                                    : to_bf16_bits(silu(v[j]) * u[j]);
            } else if (MODE == kModeDown) {
                const int d = ti.m0 + row;
                const float sd = F8 ? __ldg(a.a_scale + ti.a_row0 + row) : 1.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (col0 + j < ti.n_valid)
                        a.slots[(size_t)ep_dest[col0 + j] * a.D + d] = ep_wt[col0 + j] * (F8 ? v[j] * sd : v[j]);
            }
        };
        auto fetch_dest = [&](const TileInfo& t) {
#pragma unroll
            for (int i = 0; i < kCPW; ++i) {
                const int col = (half + 2 * i) * 32 + lane;
                const bool in = col < t.n_valid;
                nd[i] = in ? __ldg(a.row_dest + t.b_row + col) : 0;
                nw[i] = in ? __ldg(a.row_weight + t.b_row + col) : 0.f;
            }
        };
        if (kAhead && ublk < total)
            fetch_dest(tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, ublk, rank));
        int tc = 0;
        // PAIR: the accumulator is released on the leader's barrier by both CTAs
        const uint32_t tempty_leader0 = PAIR ? mapa_shared(tempty, 0) : 0u;
        for (int item = ublk, qi = 0;; item += DYN ? 0 : ugrid, ++tc, ++qi) {
            if (DYN) {
                const int qs = qi % kQD;
                const bool gq = mbar_wait(qfull + qs, (qi / kQD) & 1, a.err, kErrWaitEpilogue, a.wait_ns);
                if (!__all_sync(0xffffffffu, gq)) break;
                item = qitem[qs];
                __syncwarp();
                if (lane == 0) mbar_arrive(qempty + qs);
                if (item < 0) break;
            } else if (item >= total) {
                break;
            }
            const TileInfo ti = tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, item, rank);
            const int b = tc & 1;
            const int use = tc >> 1;
            const bool got = mbar_wait(tfull + b, use & 1, a.err, kErrWaitEpilogue, a.wait_ns);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * ACC);
            const int nchunks = (ti.n_valid + 31) >> 5;
            if (kAhead) {
#pragma unroll
                for (int i = 0; i < kCPW; ++i) {
                    cd[i] = nd[i];
                    cw[i] = nw[i];
                }
                if (item + ugrid < total)
                    fetch_dest(tc_decode_unit<MODE, BN, PAIR>(a, tabs, sc, item + ugrid, rank));
            } else if (MODE == kModeDown) {
                __syncwarp();
                for (int c = lane; c < ti.n_valid; c += 32) {
                    ep_dest[c] = __ldg(a.row_dest + ti.b_row + c);
                    ep_wt[c] = __ldg(a.row_weight + ti.b_row + c);
                }
                __syncwarp();
            }
            if (SPLIT && ti.nsplit > 1) {
                // 1. this slice's partial accumulators (rows x BN per accumulator, FP32)
                float* ps = a.partial + (size_t)(ti.tail * ti.nsplit + ti.split) * (NA * kTcM * BN);
                for (int c = half; c < nchunks; c += 2) {
                    float v[32];
                    tmem_ld32(tb + c * 32, v);
                    float u[32];
                    if (NA == 2) tmem_ld32(tb + BN + c * 32, u);
                    tmem_ld_wait();
                    float4* d0 = reinterpret_cast<float4*>(ps + (size_t)row * BN + c * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        d0[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    if (NA == 2) {
                        float4* d1 = reinterpret_cast<float4*>(ps + (size_t)(kTcM + row) * BN + c * 32);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            d1[q] = make_float4(u[4 * q], u[4 * q + 1], u[4 * q + 2], u[4 * q + 3]);
                    }
                }
                tc_fence_before();
                mbar_arrive_relaxed(tempty + b);  // the accumulator is free for the next tile
                // 2. publish; the warp that completes this (item, warp) portion reduces it
                __threadfence();
                __syncwarp();
                int old = 0;
                int* ticket = a.tickets + ti.tail * kEpiWarps + ew;
                if (lane == 0) old = atomicAdd(ticket, 1);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old != ti.nsplit - 1) continue;
                __threadfence();
                if (lane == 0) *ticket = 0;  // ready for the next launch
                const float* p0 = a.partial + (size_t)(ti.tail * ti.nsplit) * (NA * kTcM * BN);
                for (int c = half; c < nchunks; c += 2) {
                    // valid columns only, four at a time; the loads of all slices of a group
                    // are in flight together and are added in slice order
                    const int ng = (min(32, ti.n_valid - c * 32) + 3) >> 2;
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        if (g >= ng) break;
                        float4 lv[kMaxKSplit], lu[kMaxKSplit] = {};
#pragma unroll
                        for (int sp = 0; sp < kMaxKSplit; ++sp) {
                            if (sp < ti.nsplit) {
                                const float* pp = p0 + (size_t)sp * (NA * kTcM * BN) + c * 32 + 4 * g;
                                lv[sp] = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)row * BN));
                                if (NA == 2)
                                    lu[sp] = __ldcg(reinterpret_cast<const float4*>(pp + (size_t)(kTcM + row) * BN));
                            }
                        }
                        float4 sv = lv[0], su = lu[0];
#pragma unroll
                        for (int sp = 1; sp < kMaxKSplit; ++sp) {
                            if (sp < ti.nsplit) {
                                sv.x += lv[sp].x; sv.y += lv[sp].y; sv.z += lv[sp].z; sv.w += lv[sp].w;
                                if (NA == 2) {
                                    su.x += lu[sp].x; su.y += lu[sp].y; su.z += lu[sp].z; su.w += lu[sp].w;
                                }
                            }
                        }
                        finish_quad(ti, c, g, sv, su);
                    }
                }
                if (MODE == kModeGateUp && a.seg_done) signal_segment_done(a, ti.seg, lane);
                continue;
            }
            if (NA == 1) {
                // one accumulator: the TMEM load of the warp's next chunk is in flight while
                // this chunk is finished (two register buffers, used alternately)
                float va[32], vb[32];
                int c = half;
                if (c < nchunks) tmem_ld32(tb + c * 32, va);
                while (c < nchunks) {
                    tmem_ld_wait();
                    if (c + 2 < nchunks) tmem_ld32(tb + (c + 2) * 32, vb);
                    finish_chunk(ti, c, va, va);
                    c += 2;
                    if (c >= nchunks) break;
                    tmem_ld_wait();
                    if (c + 2 < nchunks) tmem_ld32(tb + (c + 2) * 32, va);
                    finish_chunk(ti, c, vb, vb);
                    c += 2;
                }
            } else {
                for (int c = half; c < nchunks; c += 2) {
                    float v[32], u[32];
                    tmem_ld32(tb + c * 32, v);
                    tmem_ld32(tb + BN + c * 32, u);
                    tmem_ld_wait();
                    finish_chunk(ti, c, v, u);
                }
            }
            // the accumulator's values are in registers or stored: hand it back to the MMA
            // (no release: the slot and h stores need not be ordered before the MMA)
            tc_fence_before();
            if (PAIR)
                mbar_arrive_cluster_relaxed(tempty_leader0 + 8u * b);
            else
                mbar_arrive_relaxed(tempty + b);
            if (MODE == kModeGateUp && !PAIR && a.seg_done) signal_segment_done(a, ti.seg, lane);
        }
    }
    tc_fence_before();
    if (PAIR)
        cluster_sync_all();   // the leader's MMAs into the peer's TMEM are complete
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem_base, Tr::TMEM);
        else
            tmem_dealloc(tmem_base, Tr::TMEM);
    }
}

template <int MODE, int BN, int STAGES, bool PAIR = false, bool F8 = false>
static cudaError_t launch_tc(const TcMaps& maps, const TcArgs& a, int grid, bool pdl,
                             cudaStream_t s) {
    constexpr int smem = TcCfg<MODE, BN, STAGES, PAIR, F8>::SMEM;
    constexpr int kTcThreads = TcCfg<MODE, BN, STAGES, PAIR, F8>::THREADS;
    auto kernel = tc_gemm_kernel<MODE, BN, STAGES, PAIR, F8>;
    cudaError_t err = ensure_smem_attr((const void*)kernel, smem);
    if (err != cudaSuccess) return err;
    if (grid < 1) grid = 1;
    if (!PAIR) return launch_kernel(kernel, dim3(grid), dim3(kTcThreads), smem, s, pdl, maps, a);
    // pairs: as many clusters of two as can be resident at once (persistent kernel), queried
    // once per device
    static std::mutex mu;
    static int clusters[64] = {0};
    int dev = 0;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidValue;
    std::unique_lock<std::mutex> lock(mu);
    if (clusters[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid & ~1);
        cfg.blockDim = dim3(kTcThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if ((err = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg)) != cudaSuccess) return err;
        if (n < 1) return cudaErrorInvalidConfiguration;
        clusters[dev] = n;
    }
    int pairs = grid / 2 < clusters[dev] ? grid / 2 : clusters[dev];
    lock.unlock();
    if (pairs < 1) pairs = 1;
    return launch_kernel_cluster(kernel, dim3(2 * pairs), dim3(kTcThreads), smem, s, pdl, 2, maps, a);
}

// Whether clusters of two CTAs of the pair kernels can be resident on this device (queried
// once per device); without them the forward uses the one-CTA wide tiles.  The environment
// variable MOE_B200_NO_PAIRS (any value) selects the wide tiles regardless.
bool pair_tiles_available() {
    if (getenv("MOE_B200_NO_PAIRS")) return false;
    static std::mutex mu;
    static int state[64] = {0};   // 0 unknown, 1 yes, -1 no
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (state[dev] == 0) {
        bool ok = true;
        auto probe = [&](const void* kernel, int smem) {
            if (ensure_smem_attr(kernel, smem) != cudaSuccess) return false;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(2);
            cfg.blockDim = dim3(TcCfg<kModeGateUp, kGuBN, kPairStages, true>::THREADS);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
            if (e != cudaSuccess) (void)cudaGetLastError();   // not sticky; clear it
            return e == cudaSuccess && n > 0;
        };
        ok = probe((const void*)tc_gemm_kernel<kModeGateUp, kGuBN, kPairStages, true>,
                   TcCfg<kModeGateUp, kGuBN, kPairStages, true>::SMEM) &&
             probe((const void*)tc_gemm_kernel<kModeDown, kDnBN, kPairStages, true>,
                   TcCfg<kModeDown, kDnBN, kPairStages, true>::SMEM);
        state[dev] = ok ? 1 : -1;
    }
    return state[dev] == 1;
}

cudaError_t launch_tc_router(const TcMaps& maps, const TcArgs& a, int num_sms, bool pdl,
                             cudaStream_t s) {
    const int items = ((a.T + kRtBN - 1) / kRtBN) * ((a.E + kTcM - 1) / kTcM) * a.ksplit;
    return launch_tc<kModeRouter, kRtBN, kStages>(maps, a, items < num_sms ? items : num_sms, pdl, s);
}

cudaError_t launch_tc_gate_up(const TcMaps& maps, const TcArgs& a, int num_sms, int tiles, bool f8,
                              bool pdl, cudaStream_t s) {
    if (tiles == kTilesNarrow && f8)
        return launch_tc<kModeGateUp, kNarrowBN, kGuNarrowStagesF8, false, true>(maps, a, num_sms, pdl, s);
    if (f8) return cudaErrorInvalidValue;
    if (tiles == kTilesNarrow)
        return launch_tc<kModeGateUp, kNarrowBN, kGuNarrowStages>(maps, a, num_sms, pdl, s);
    if (tiles == kTilesPair)
        return launch_tc<kModeGateUp, kGuBN, kPairStages, true>(maps, a, num_sms, pdl, s);
    return launch_tc<kModeGateUp, kGuBN, kStages>(maps, a, num_sms, pdl, s);
}

cudaError_t launch_tc_down(const TcMaps& maps, const TcArgs& a, int num_sms, int tiles, bool f8,
                           bool pdl, cudaStream_t s) {
    if (tiles == kTilesNarrow && f8)
        return launch_tc<kModeDown, kNarrowBN, kDnNarrowStagesF8, false, true>(maps, a, num_sms, pdl, s);
    if (f8) return cudaErrorInvalidValue;
    if (tiles == kTilesNarrow)
        return launch_tc<kModeDown, kNarrowBN, kDnNarrowStages>(maps, a, num_sms, pdl, s);
    if (tiles == kTilesPair)
        return launch_tc<kModeDown, kDnBN, kPairStages, true>(maps, a, num_sms, pdl, s);
    return launch_tc<kModeDown, kDnBN, kStages>(maps, a, num_sms, pdl, s);
}

}  // namespace moe
