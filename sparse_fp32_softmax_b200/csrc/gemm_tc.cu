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
//   gate_up: two accumulators per tile, gate rows [f0, f0+128) and the matching up rows
//            [I+f0, ...), against the same token tile; TMEM lane f holds gate and up of
//            feature f for every token, and the epilogue writes h = silu(g) * u in bf16.
//   down:    one accumulator, down rows [d0, d0+128) against a tile of h rows; the epilogue
//            scales by the routing weight and stores FP32 into the token's slot (a bf16 slot
//            would add a third bf16 rounding on top of h and the output).
//   router:  one accumulator, router rows [e0, e0+128) against a tile of x rows; FP32 out.
//
// Per CTA (one per SM, persistent over a device-side item list):
//   warp 0      TMA producer: 4-stage ring of {A tile(s) 128x64, B tile BNx64} bf16 tiles in
//               the 128-byte swizzle layout, completion counted on an mbarrier;
//   warp 1      allocates TMEM, and one thread issues tcgen05.mma (M=128, N=tile width,
//               K=16 x 4 per stage) with FP32 accumulation in TMEM; tcgen05.commit frees a
//               stage when its MMAs are done and publishes an accumulator when a tile is;
//   warps 2..9  epilogue: two warps per TMEM lane quarter (a warp may only read the quarter
//               warp % 4), taking alternate 32-column chunks of the tile: tcgen05.ld, apply
//               the epilogue, store; accumulators are double-buffered so the next tile's
//               MMAs overlap this epilogue.
// All mbarrier waits are bounded (common.cuh); on expiry the kernel records the fact in the
// device error word and winds down without leaving TMEM allocated.
#include "common.cuh"

namespace moe {

enum { kModeGateUp = 0, kModeDown = 1, kModeRouter = 2 };

template <int MODE>
struct TcTraits;
template <>
struct TcTraits<kModeGateUp> {
    static constexpr int BN = kGuBN, NA = 2, ACC = 2 * kGuBN, TMEM = 512;
};
template <>
struct TcTraits<kModeDown> {
    static constexpr int BN = kDnBN, NA = 1, ACC = kDnBN, TMEM = 512;
};
template <>
struct TcTraits<kModeRouter> {
    static constexpr int BN = kRtBN, NA = 1, ACC = kRtBN, TMEM = 256;
};

constexpr int kATileBytes = kTcM * kTcK * 2;  // 16 KB
constexpr int kEpiWarps = 8;
constexpr int kTcThreads = (2 + kEpiWarps) * 32;

template <int MODE>
constexpr int tc_stage_bytes() {
    return TcTraits<MODE>::NA * kATileBytes + TcTraits<MODE>::BN * kTcK * 2;
}
template <int MODE>
constexpr int tc_smem_bytes() {
    return kStages * tc_stage_bytes<MODE>() + 1024 + 256 + (int)sizeof(SmemTables) +
           (MODE == kModeDown ? kEpiWarps * 2 * 4 * kDnBN : 0);
}

struct TileInfo {
    int bi;       // token-operand box: 16 << bi rows
    int shared;   // A comes from the shared-expert tensor map
    int a_row0;   // first A row (gate rows for gate_up)
    int a_row1;   // first up row (gate_up only)
    int b_row;    // first B (token) row
    int n_valid;  // valid token columns, 1..BN
    int nk;       // K stages
    int m0;       // first output feature of this tile within its segment
};

template <int MODE>
__device__ __forceinline__ int tc_total_items(const TcArgs& a) {
    constexpr int BN = TcTraits<MODE>::BN;
    if (MODE == kModeRouter) return ((a.T + BN - 1) / BN) * ((a.E + kTcM - 1) / kTcM);
    const int* prefix = (MODE == kModeGateUp) ? a.tables.gu_items : a.tables.dn_items;
    return __ldg(prefix + a.nseg);
}

// Smallest token box (16 << bi rows, bi <= log2(BN/16)) that covers n valid rows.
template <int BN>
__device__ __forceinline__ int box_index(int n) {
    int bi = 0;
    while ((16 << bi) < n && (16 << bi) < BN) ++bi;
    return bi;
}

template <int MODE>
__device__ __forceinline__ TileInfo tc_decode_item(const TcArgs& a, const SmemTables* st, int item) {
    constexpr int BN = TcTraits<MODE>::BN;
    TileInfo ti;
    if (MODE == kModeRouter) {
        const int mtc = (a.E + kTcM - 1) / kTcM;
        const int tt = item / mtc, mt = item % mtc;
        ti.shared = 0;
        ti.a_row0 = mt * kTcM;
        ti.a_row1 = 0;
        ti.b_row = tt * BN;
        ti.n_valid = min(BN, a.T - tt * BN);
        ti.nk = a.D / kTcK;
        ti.m0 = mt * kTcM;
        ti.bi = box_index<BN>(ti.n_valid);
        return ti;
    }
    const int s = find_segment_smem(st->prefix, a.nseg, item);
    const int local = item - st->prefix[s];
    const int sh = (s == a.E);
    const int Iseg = sh ? a.I_s : a.I;
    const int mtc = (MODE == kModeGateUp) ? Iseg / kTcM : a.D / kTcM;
    const int tt = local / mtc, mt = local % mtc;
    const int cnt = st->count[s];
    const int start = st->start[s];
    ti.shared = sh;
    ti.b_row = start + tt * BN;
    ti.n_valid = min(BN, cnt - tt * BN);
    ti.m0 = mt * kTcM;
    if (MODE == kModeGateUp) {
        const int base = sh ? 0 : s * 2 * a.I;
        ti.a_row0 = base + mt * kTcM;
        ti.a_row1 = base + Iseg + mt * kTcM;
        ti.nk = a.D / kTcK;
    } else {
        const int base = sh ? 0 : s * a.D;
        ti.a_row0 = base + mt * kTcM;
        ti.a_row1 = 0;
        ti.nk = Iseg / kTcK;
    }
    ti.bi = box_index<BN>(ti.n_valid);
    return ti;
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

template <int MODE>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
    using Tr = TcTraits<MODE>;
    constexpr int BN = Tr::BN, NA = Tr::NA, ACC = Tr::ACC;
    constexpr int SB = tc_stage_bytes<MODE>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * SB);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;  // [2]
    uint64_t* tempty = tfull + 2;       // [2]
    uint64_t* drain = tempty + 2;       // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    SmemTables* tabs = reinterpret_cast<SmemTables*>(smem + kStages * SB + 256);
    // down: per epilogue warp, the current tile's row destinations and weights
    int* ep_dest_all = reinterpret_cast<int*>(tabs + 1);                       // [8][BN]
    float* ep_wt_all = reinterpret_cast<float*>(ep_dest_all + kEpiWarps * BN);  // [8][BN]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // prologue: independent of earlier kernels, overlaps them under launch chaining
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull + b, 1);
            mbar_init(tempty + b, kEpiWarps * 32);
        }
        mbar_init(drain, 1);
        mbar_fence_init();
    }
    if (warp == 0 && lane < 2 + kNumBBoxes) {
        const CUtensorMap* m = lane == 0 ? &maps.A : (lane == 1 ? &maps.A_shared : &maps.B[lane - 2]);
        tma_prefetch_desc(m);
    }
    if (warp == 1) tmem_alloc(tmem_slot, Tr::TMEM);
    pdl_wait();
    pdl_launch_dependents();
    const int total = tc_total_items<MODE>(a);
    if (MODE != kModeRouter) {
        const int* prefix = (MODE == kModeGateUp) ? a.tables.gu_items : a.tables.dn_items;
        load_tables(tabs, prefix, a.tables.seg_count, a.tables.seg_start, a.nseg);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if ((int)blockIdx.x >= total) {
        // no work for this CTA: nothing was issued; fall through to the TMEM release
    } else if (warp == 0) {
        // ------------------------------------------------------------ TMA producer warp
        // Weight tiles are issued by lane 0.  Token tiles: in gather mode gate_up fetches its
        // rows from x by row_token, lane i taking rows 4i..4i+3 of the tile (rows past the
        // segment repeat its last row; their columns are never used); otherwise lane 0 loads
        // a tile of the permuted rows.
        int it = 0;
        bool ok = true;
        int last_round[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) last_round[s] = -1;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const TileInfo ti = tc_decode_item<MODE>(a, tabs, item);
            const CUtensorMap* mA = ti.shared ? &maps.A_shared : &maps.A;
            const CUtensorMap* mB = &maps.B[ti.bi];
            const int brows = 16 << ti.bi;
            const uint32_t bytes = NA * kATileBytes + (uint32_t)brows * kTcK * 2;
            const bool gather = MODE == kModeGateUp && a.gather;
            int g0 = 0, g1 = 0, g2 = 0, g3 = 0;
            if (gather) {
                const int base = ti.b_row + 4 * lane;
                const int last = ti.b_row + ti.n_valid - 1;
                g0 = __ldg(a.row_token + min(base + 0, last));
                g1 = __ldg(a.row_token + min(base + 1, last));
                g2 = __ldg(a.row_token + min(base + 2, last));
                g3 = __ldg(a.row_token + min(base + 3, last));
            }
            for (int kb = 0; kb < ti.nk; ++kb, ++it) {
                const int s = it % kStages;
                const int round = it / kStages;
                const bool got = mbar_wait(empty + s, (round & 1) ^ 1, a.err, kErrWaitProducer);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                uint8_t* st = smem + s * SB;
                if (lane == 0) {
                    mbar_arrive_expect_tx(full + s, bytes);
                    tma_load(st, mA, full + s, kb * kTcK, ti.a_row0);
                    if (NA == 2) tma_load(st + kATileBytes, mA, full + s, kb * kTcK, ti.a_row1);
                    if (!gather) tma_load(st + NA * kATileBytes, mB, full + s, kb * kTcK, ti.b_row);
                }
                if (gather) {
                    __syncwarp();  // expect_tx is posted before any gather can complete
                    if (4 * lane < brows)
                        tma_gather4(st + NA * kATileBytes + lane * 4 * kTcK * 2, mB, full + s,
                                    kb * kTcK, g0, g1, g2, g3);
                }
#pragma unroll
                for (int q = 0; q < kStages; ++q)
                    if (q == s) last_round[q] = round;
            }
        }
        // wait until the MMA issuer has released every stage, then until every issued
        // load has landed, so no copy is in flight when the CTA exits
        if (ok) {
            for (int i = 0; i < kStages; ++i, ++it) {
                const int s = it % kStages;
                const int round = it / kStages;
                const bool got = mbar_wait(empty + s, (round & 1) ^ 1, a.err, kErrWaitTail);
                if (!__all_sync(0xffffffffu, got)) break;
            }
        }
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            if (last_round[s] >= 0) mbar_wait(full + s, last_round[s] & 1, a.err, kErrWaitTail);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc0 = umma_idesc_bf16_f32(kTcM, 16) & ~(0x3Fu << 17);
            int it = 0, tc = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++tc) {
                const TileInfo ti = tc_decode_item<MODE>(a, tabs, item);
                const int b = tc & 1;
                const int use = tc >> 1;
                if (!mbar_wait(tempty + b, (use & 1) ^ 1, a.err, kErrWaitMma)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                int n = (ti.n_valid + 15) & ~15;
                n = n < 16 ? 16 : (n > BN ? BN : n);
                const uint32_t idesc = idesc0 | ((uint32_t)(n >> 3) << 17);
                const uint32_t d0 = tmem_base + (uint32_t)(b * ACC);
                for (int kb = 0; kb < ti.nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const int round = it / kStages;
                    if (!mbar_wait(full + s, round & 1, a.err, kErrWaitMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* st = smem + s * SB;
                    const uint64_t da0 = umma_desc_sw128(st);
                    const uint64_t da1 = umma_desc_sw128(st + kATileBytes);
                    const uint64_t db = umma_desc_sw128(st + NA * kATileBytes);
#pragma unroll
                    for (int kk = 0; kk < kTcK / 16; ++kk) {
                        const uint32_t accum = (kb | kk) != 0;
                        umma_bf16(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
                        if (NA == 2) umma_bf16(d0 + BN, da1 + 2 * kk, db + 2 * kk, idesc, accum);
                    }
                    umma_commit(empty + s);
                }
                if (!ok) break;
                umma_commit(tfull + b);
            }
            // every issued MMA must be complete before TMEM is released
            umma_commit(drain);
            mbar_wait(drain, 0, a.err, kErrWaitMma);
        }
    } else {
        // ------------------------------------------------------------ epilogue warps 2..9
        const int quarter = warp & 3;
        const int ew = warp - 2;               // epilogue warp 0..7
        const int half = ew >> 2;              // which alternate chunks this warp takes
        const int row = quarter * 32 + lane;  // TMEM lane = weight row within the tile
        int tc = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++tc) {
            const TileInfo ti = tc_decode_item<MODE>(a, tabs, item);
            const int b = tc & 1;
            const int use = tc >> 1;
            const bool got = mbar_wait(tfull + b, use & 1, a.err, kErrWaitEpilogue);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * ACC);
            const int nchunks = (ti.n_valid + 31) >> 5;
            int* ep_dest = ep_dest_all + ew * BN;
            float* ep_wt = ep_wt_all + ew * BN;
            if (MODE == kModeDown) {
                // each epilogue warp keeps its own copy: no barrier across warps
                __syncwarp();
                for (int c = lane; c < ti.n_valid; c += 32) {
                    ep_dest[c] = __ldg(a.row_dest + ti.b_row + c);
                    ep_wt[c] = __ldg(a.row_weight + ti.b_row + c);
                }
                __syncwarp();
            }
            for (int c = half; c < nchunks; c += 2) {
                float v[32];
                tmem_ld32(tb + c * 32, v);
                if (MODE == kModeGateUp) {
                    float u[32];
                    tmem_ld32(tb + BN + c * 32, u);
                    tmem_ld_wait();
                    const int f = ti.m0 + row;
                    uint16_t* hp = a.h + (size_t)(ti.b_row + c * 32) * a.ld_h + f;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (c * 32 + j < ti.n_valid) hp[(size_t)j * a.ld_h] = to_bf16_bits(silu(v[j]) * u[j]);
                } else if (MODE == kModeDown) {
                    tmem_ld_wait();
                    const int d = ti.m0 + row;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = c * 32 + j;
                        if (col < ti.n_valid)
                            a.slots[(size_t)ep_dest[col] * a.D + d] = ep_wt[col] * v[j];
                    }
                } else {
                    tmem_ld_wait();
                    const int e = ti.m0 + row;
                    if (e < a.E) {
                        const float be = a.bias ? __ldg(a.bias + e) : 0.0f;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int t = ti.b_row + c * 32 + j;
                            if (c * 32 + j < ti.n_valid)
                                a.logits[(size_t)t * a.E + e] = a.bias ? v[j] + be : v[j];
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tempty + b);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Tr::TMEM);
    }
}

template <int MODE>
static cudaError_t launch_tc(const TcMaps& maps, const TcArgs& a, int grid, bool pdl, cudaStream_t s) {
    constexpr int smem = tc_smem_bytes<MODE>();
    cudaError_t err = ensure_smem_attr((const void*)tc_gemm_kernel<MODE>, smem, 1 + MODE);
    if (err != cudaSuccess) return err;
    if (grid < 1) grid = 1;
    return launch_kernel(tc_gemm_kernel<MODE>, dim3(grid), dim3(kTcThreads), smem, s, pdl, maps, a);
}

cudaError_t launch_tc_router(const TcMaps& maps, const TcArgs& a, int num_sms, bool pdl,
                             cudaStream_t s) {
    const int items = ((a.T + kRtBN - 1) / kRtBN) * ((a.E + kTcM - 1) / kTcM);
    return launch_tc<kModeRouter>(maps, a, items < num_sms ? items : num_sms, pdl, s);
}

cudaError_t launch_tc_gate_up(const TcMaps& maps, const TcArgs& a, int num_sms, bool pdl,
                              cudaStream_t s) {
    return launch_tc<kModeGateUp>(maps, a, num_sms, pdl, s);
}

cudaError_t launch_tc_down(const TcMaps& maps, const TcArgs& a, int num_sms, bool pdl,
                           cudaStream_t s) {
    return launch_tc<kModeDown>(maps, a, num_sms, pdl, s);
}

}  // namespace moe
