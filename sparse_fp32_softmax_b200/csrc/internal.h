// internal.h -- declarations shared by the library's translation units (not public API).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Every bounded wait gives up after this long (unless the call sets a shorter limit) and
// reports it in the device error word.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

// Bits of the device error word (first int of the workspace).
enum : int {
    kErrWaitProducer = 1,   // TMA producer gave up waiting for a free stage
    kErrWaitMma = 2,        // MMA issuer gave up waiting for data or a free accumulator
    kErrWaitEpilogue = 4,   // epilogue gave up waiting for an accumulator
    kErrBadIndex = 8,       // an expert index outside [0, E) reached the permute stage
    kErrWaitTail = 16,      // producer gave up draining its last stages
    kErrWaitGrid = 32,      // a block of the decode kernel gave up waiting for the other blocks
};

// Tile geometry of the tcgen05 grouped GEMMs (swap-AB: weights on M, tokens on N).
constexpr int kTcM = 128;       // weight rows per tile (MMA M)
constexpr int kTcK = 64;        // K elements per pipeline stage (one 128-byte swizzle row)
// Wide gate_up tiles interleave gate and up rows in the MMA's M (16 gate rows of 16
// features, then their 16 up rows, four times: 64 features), so one accumulator of up to 256
// token columns holds both and every MMA has N up to 256 (a tcgen05.mma costs the issuing
// thread about the same whatever its N, so wider MMAs do more work per instruction).
constexpr int kGuBN = 256;      // token columns per wide gate_up tile
constexpr int kGuILFeatures = 64;  // features per wide (interleaved) gate_up tile
constexpr int kDnBN = 256;      // token columns per down tile
constexpr int kRtBN = 128;      // token columns per router-logit tile
constexpr int kStages = 4;      // shared-memory pipeline depth of the wide tiles
// Narrow tiles for small per-expert row counts (decode): the token box is at most 64 rows,
// so a stage is mostly weight bytes and the freed shared memory buys a deeper pipeline --
// more weight bytes in flight per SM, which is what a weight-streaming GEMM is bound by.
constexpr int kNarrowBN = 64;
constexpr int kGuNarrowStages = 5;   // 5 x (2 x 16 KB + 8 KB)
constexpr int kDnNarrowStages = 8;   // 8 x (16 KB + 8 KB)
// FP8 weights (narrow tiles): load stages of 8 KB per weight tile + 8 KB of tokens, plus a
// ring of three widened bf16 tiles
constexpr int kGuNarrowStagesF8 = 5;   // 5 x (2 x 8 KB + 8 KB) + 3 x 32 KB
constexpr int kDnNarrowStagesF8 = 8;   // 8 x (8 KB + 8 KB) + 3 x 16 KB
// The forward takes the narrow tiles when the mean rows per expert, T*k/E, is at most this.
constexpr int kNarrowMaxMeanRows = 32;
// Largest T for which gate_up gathers its token rows straight from x (tile::gather4, four
// rows per TMA operation) instead of reading a permuted copy: a tile then has at most 32
// rows, 8 gathers per stage.  Above, the TMA engine's cost per gather operation makes the
// expert GEMM slower by more than a separate copy costs (measured on B200).
constexpr int kGatherMaxT = 32;
// Tile families of the expert GEMMs.  Pair tiles (wide shapes, D % 256 == 0): two CTAs of a
// cluster share each tcgen05.mma of M = 256 (cta_group::2) -- 128 weight rows per SM, half
// of the 256 token rows per SM -- which halves the shared-memory operand traffic per FLOP
// of each SM; gate_up pair tiles cover 128 features, down pair tiles 256 output rows.
enum { kTilesNarrow = 0, kTilesWide = 1, kTilesPair = 2 };
constexpr int kPairStages = 6;   // 6 x (16 KB weights + 16 KB tokens) per CTA

// Split tail items of the narrow-tile GEMMs: at most this many K slices per item, and a
// fixed capacity of FP32 partial-sum slots (slices per item are capped so that the tail's
// slices fit; a device with fewer SMs splits less).  A tail is split only when it is at most
// half a wave of the grid, so at most grid / 2 items x 8 epilogue warps hold a ticket; the
// persistent expert GEMMs therefore run at most kMaxTcGrid CTAs.
constexpr int kMaxKSplit = 8;
constexpr int kSplitSlots = 148;
constexpr int kSplitTickets = 1024;   // per GEMM; the completion counters follow them
constexpr int kMaxTcGrid = 2 * kSplitTickets / 8;
static_assert(kMaxTcGrid / 2 * 8 <= kSplitTickets, "split-tail tickets");
__host__ __device__ inline bool use_narrow_tiles(long long T, int k, int E) {
    return T * k <= (long long)kNarrowMaxMeanRows * E;
}

// Largest supported expert count (and segments: experts + one shared expert).
constexpr int kMaxE = 512;
constexpr int kMaxK = 16;
constexpr int kMaxSegments = kMaxE + 1;

// Permute-stage geometry.
constexpr int kPermChunk = 4096;   // assignments per histogram / scatter block
constexpr int kPermThreads = 1024;

// Device tables written by the permute stage.  Segment s < E is routed expert s; when a
// shared expert is present it is segment E and owns the last T rows in token order.
struct SegTables {
    int* seg_count;   // [nseg] rows of each segment
    int* seg_start;   // [nseg] first permuted row of each segment
    int* gu_items;    // [nseg + 1] prefix sums of tcgen05 gate_up work items
    int* dn_items;    // [nseg + 1] prefix sums of tcgen05 down work items
};

struct PermuteArgs {
    const int32_t* topk_idx;  // [T, k]
    const float* topk_w;      // [T, k] or null
    int T, k, E, tile_m;
    int has_shared;           // adds segment E = all T tokens in order
    int slots_per_token;      // k (+1 with a shared expert): row_dest = t * S + j
    int D, I, I_s;
    int* chunk_counts;        // [nchunks, E] scratch
    int nchunks;
    int* counts;              // [E] (caller-visible), may alias tables.seg_count
    int* offsets;             // [E + 1] (caller-visible)
    int32_t* row_token;       // [cap]
    float* row_weight;        // [cap] or null
    int32_t* row_dest;        // [cap] or null
    int32_t* slot_row;        // [T * k]
    int cap;                  // rows available in row_* arrays
    SegTables tables;         // may be all-null (moe_permute alone)
    int gu_bn, dn_bn;         // token columns per gate_up / down tile (work-item tables)
    int gu_features;          // features per gate_up tile (128 narrow or pair, 64 interleaved)
    int dn_rows;              // output rows per down tile (128, or 256 for pair tiles)
    int* err;
};

// Selection and permutation of T*k <= kPermChunk assignments in one kernel: each block
// selects 32 tokens, the last block to finish performs the permutation.
struct RouteArgs {
    const float* bias;        // [E] or null
    int T, E, k, norm;
    float* logits_out;        // [T, E] (the caller's or workspace scratch)
    int32_t* topk_idx;        // [T, k]
    float* topk_w;            // [T, k]
    int* ticket;              // zero before the launch
    PermuteArgs perm;         // topk_idx / topk_w above are its inputs
    // selection from router partial sums (select_permute_kernel): logits = sum over the
    // nsplit partials [nsplit, T, E] in split order, then + bias
    const float* part;
    int nsplit;
};

// The router GEMM splits K so that small token counts still spread over the SMs; its
// partial sums are added in split order by the selection.  The split depends only on the
// shapes (not on the device), so results do not depend on the GPU the call runs on.
constexpr int kRouterMaxSplit = 8;
constexpr int kSplitTargetCtas = 148;
inline int router_splits(int T, int E, int D, int bn) {
    const long long items = (long long)((T + bn - 1) / bn) * ((E + 127) / 128);
    long long s = kSplitTargetCtas / (items > 0 ? items : 1);
    const int nk = D / 64;
    if (s > kRouterMaxSplit) s = kRouterMaxSplit;
    if (s > nk) s = nk;
    return s < 1 ? 1 : (int)s;
}

// Tensor maps of one grouped GEMM: the weight operand (routed experts, shared expert) and
// the token operand encoded at five box heights (16, 32, 64, 128, 256 rows), so that a work
// item loads only as many token rows as it has (rounded up to the next height).
constexpr int kNumBBoxes = 5;
struct alignas(64) TcMaps {
    CUtensorMap A;
    CUtensorMap A_shared;
    CUtensorMap B[kNumBBoxes];
    CUtensorMap A8;   // FP8 weights: [rows, K] bytes, 64 x 128 boxes, no swizzle (F8 kernels)
};

struct TcArgs {
    int D, I, I_s, E, nseg;
    SegTables tables;
    // gate_up token rows: gather = 1 -> gathered from x by row_token (map B = x with a
    // one-row box, four rows per TMA operation); gather = 0 -> tiles of the permuted copy
    const int32_t* row_token;
    int gather;
    // gate_up epilogue
    uint16_t* h;              // [rows, ld_h] bf16 SwiGLU output
    int ld_h;
    // down epilogue
    const float* row_weight;
    const int32_t* row_dest;
    float* slots;             // [T * S, D] FP32
    // split tail items (narrow tiles): FP32 partial accumulators, one slot of
    // NA x 128 x BN floats per slice (partial_slots slots), and one zeroed ticket per
    // (tail item, epilogue warp)
    float* partial;
    int* tickets;
    int partial_slots;
    // Per-expert completion of gate_up (narrow tiles): gate_up's epilogue warps add 1 to
    // seg_done[s] (and to seg_done[nseg]) once they have written their part of an item's h
    // tile; with dep_wait, the down kernel does not wait for the whole gate_up grid but its
    // producer waits until seg_done[s] reaches 8 x (gate_up items of segment s), read from
    // gu_prefix, so down starts on finished experts while gate_up's last wave runs.
    int* seg_done;
    const int* gu_prefix;
    int dep_wait;
    // narrow tiles: counter (zero at launch) from which the CTAs claim their units
    int* sched;
    // FP8 weights (F8 kernels): FP32 scale of every weight row (A row), [E * rows per expert]
    const float* a_scale;
    // narrow gate_up: before its dependency wait, CTA b requests into L2 the first spec_steps
    // K steps of the weight tiles of the unit it most likely starts with (feature tile
    // b % (I/128) of expert b / (I/128): the first unit when every expert received 1..64
    // rows); 0 = none.  Only a cache hint: nothing depends on the guess.
    int spec_steps;
    // dense (router) epilogue: partial sums over split s of K go to logits + s*T*E
    float* logits;            // [ksplit, T, E] FP32
    int ksplit;
    int T;
    int* err;
    unsigned long long wait_ns;   // limit of every bounded wait (kWaitLimitNs by default)
};

// Raise a kernel's dynamic shared-memory limit once per device (host-side attribute; done
// outside stream capture by the first call on each device).
cudaError_t ensure_smem_attr(const void* kernel, int bytes);

// Streaming multiprocessors of the current device (queried once per device; 0 on error).
// Launchers size their grids from it.
int device_sm_count();
// Records the cudaError_t behind a MOE_ERR_CUDA for moe_last_cuda_error (this host thread).
void note_cuda_error(int e);

// ---------------------------------------------------------------- launchers (return the
// launch error, cudaSuccess when all kernels were enqueued).  pdl: launch the first kernel
// as a programmatic dependent of the previous kernel on the stream (set for every launch
// after the first of an API call; later kernels of one launcher always chain).
cudaError_t launch_router_small(const uint16_t* x, const uint16_t* W_r, int T,
                                int D, int E, float* logits, bool pdl, cudaStream_t s);
cudaError_t launch_select(const float* part, int nsplit, const float* bias, int T, int E, int k,
                          int norm, int32_t* idx, float* w, float* logits_out, bool pdl,
                          cudaStream_t s);
cudaError_t launch_permute(const PermuteArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_select_permute(const RouteArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* row_token, int rows, int D,
                               uint16_t* x_perm, bool pdl, cudaStream_t s);
bool pair_tiles_available();
cudaError_t launch_tc_router(const TcMaps& maps, const TcArgs& a, int num_sms, bool pdl,
                             cudaStream_t s);
cudaError_t launch_tc_gate_up(const TcMaps& maps, const TcArgs& a, int num_sms, int tiles, bool f8,
                              bool pdl, cudaStream_t s);
cudaError_t launch_tc_down(const TcMaps& maps, const TcArgs& a, int num_sms, int tiles, bool f8,
                           bool pdl, cudaStream_t s);
cudaError_t launch_combine(const float* slots, int T, int D, int k, int has_shared,
                           const uint16_t* x, const uint16_t* shared_gate,
                           const uint16_t* residual, uint16_t* out, float* out_f32, bool pdl,
                           cudaStream_t s);

// ---------------------------------------------------------------- the decode kernel
// The whole block for one token in one persistent kernel (one block per SM, all resident at
// once): router, selection, gate_up, down and the combine, separated by two grid-wide
// barriers.  Used for T = 1 when the call needs nothing it does not do.
constexpr int kDecWarps = 8;           // compute warps (plus one copy warp)
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecMaxStages = 32;
constexpr int kDecMinStages = 2;
constexpr int kDecSmemBudget = 220 * 1024;   // dynamic shared memory per block
constexpr int kDecMaxD = 2048;         // a gate/up row is at most 8 16-byte pieces per lane
constexpr int kDecChunks = kDecMaxD / 256;      // 16-byte pieces of a bf16 gate/up row per lane
constexpr int kDecChunks8 = kDecMaxD / 512;     // the same for an E4M3 row

// Shared-memory layout of a decode block: the copy ring (a stage holds one expert's down
// rows for the block's output rows: nd_max rows of I; bf16 rows padded to whole 16-row MMA
// tiles, each row at a stride of 2I + 16 bytes so that the 8 rows an ldmatrix reads fall in
// distinct banks; E4M3 rows packed at a stride of I bytes), x as FP32 in two planes, h of every
// slot, the down results of the block's output rows, then the ring's barriers.
struct DecodeLayout {
    int stages, nd_max, rs;
    size_t sb, ring, xs, hs, val, bars, total;
};
__host__ __device__ inline DecodeLayout decode_layout(int D, int k, int I, int nd_max, int stages, bool f8) {
    DecodeLayout L;
    L.stages = stages;
    L.rs = f8 ? I : 2 * I + 16;
    L.sb = ((f8 ? (size_t)nd_max * L.rs : (size_t)((nd_max + 15) / 16) * 16 * L.rs) + 127) / 128 * 128;
    L.nd_max = nd_max;
    size_t off = 0;
    L.ring = off;
    off += (size_t)stages * L.sb;
    L.xs = off;
    off += (size_t)D * 4;
    L.hs = off;
    off += (size_t)k * I * 2;
    L.val = off;
    off += ((size_t)k * nd_max * 4 + 15) / 16 * 16;
    L.bars = off;
    off += (size_t)2 * stages * 8;
    L.total = off;
    return L;
}

struct DecodeArgs {
    const uint16_t* x;        // [D]
    const uint16_t* W_r;      // [E, D]
    const float* bias;        // [E] or null
    const uint16_t* W_gu;     // [E, 2I, D] (bf16 weights)
    const uint16_t* W_dn;     // [E, D, I]
    const uint8_t* W_gu8;     // [E, 2I, D] E4M3, or null (then the bf16 weights above)
    const uint8_t* W_dn8;     // [E, D, I] E4M3
    const float* gu_scale;    // [E * 2I] FP32 row scales of W_gu8
    const float* dn_scale;    // [E * D]
    const uint16_t* residual; // [D] or null (may alias out)
    uint16_t* out;            // [D]
    float* out_f32;           // [D] or null
    float* logits_out;        // [E] or null
    int32_t* idx_out;         // [k]
    float* w_out;             // [k]
    unsigned long long* lgf;  // workspace [E]: flag (high word) and logit before the bias (low
                              // word); zero before the launch
    uint16_t* h;              // workspace [k, I]: h of every slot
    unsigned* bar;            // workspace: the grid-barrier counter, zeroed before the launch
    int* err;
    int D, E, k, I, norm;
    int stages;
    unsigned long long wait_ns;
    int extra_blocks;         // 0; 1 makes every grid barrier wait for a block that does not exist
};

// Ring depth for this shape on a grid of `blocks` blocks, or 0 when the decode kernel does
// not apply (T != 1, D or I too wide for its buffers).
int decode_stages(int T, int D, int E, int k, int I, int blocks, bool f8);
cudaError_t launch_decode(const DecodeArgs& a, int blocks, bool pdl, cudaStream_t s);

}  // namespace moe
