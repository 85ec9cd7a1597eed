// moe_api.cu -- the C ABI: argument validation, workspace layout, TMA tensor maps and the
// launch sequence of the MoE block forward pass.  Host code only; kernels live in the other
// translation units.  Nothing here allocates device memory or synchronises the host, except
// moe_get_device_status, whose job is to synchronise.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/moe_b200.h"
#include "internal.h"

using namespace moe;

namespace moe {

cudaError_t ensure_smem_attr(const void* kernel, int bytes) {
    // once per (device, kernel): the attribute is a host-side setting, raised to the largest
    // size any launch of that kernel asks for
    struct Entry { int dev; const void* kernel; int bytes; };
    static std::mutex mu;
    static Entry done[256];
    static int n = 0;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (done[i].dev == dev && done[i].kernel == kernel && done[i].bytes >= bytes) return cudaSuccess;
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err != cudaSuccess) return err;
    for (int i = 0; i < n; ++i)
        if (done[i].dev == dev && done[i].kernel == kernel) {
            done[i].bytes = bytes;
            return cudaSuccess;
        }
    if (n < 256) done[n++] = Entry{dev, kernel, bytes};
    return cudaSuccess;
}

int device_sm_count() {
    static std::mutex mu;
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

}  // namespace moe

namespace {

constexpr size_t kAlign = 256;
// Ints of the ticket region: gate_up split tickets, down split tickets, the per-expert
// completion counters of gate_up (nseg + 1 <= kMaxSegments + 1), the same number of
// counters that stay zero (MOE_DIAG_UNSIGNALLED_HANDOFF points the down GEMM at them),
// the unit counters of the narrow gate_up and down kernels, and the grid-barrier counter of
// the decode kernel.
constexpr int kSchedAt = 2 * kSplitTickets + 2 * (kMaxSegments + 1);
constexpr int kDecBarAt = kSchedAt + 2;
constexpr int kTicketInts = kDecBarAt + 1;

// The cudaError_t of the last CUDA failure seen by this host thread (moe_last_cuda_error).
thread_local int g_last_cuda_error = 0;
constexpr int kRouterSmallMaxT = 64;     // below: CUDA-core router; above: tcgen05 router GEMM

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Byte offsets of every workspace region.
struct Plan {
    int T, D, E, k, I, I_s, has_shared, S, R, ld_h, nchunks, nseg, rsplit;
    size_t err, tickets, partial, logits, idx, w, counts, offsets, chunk, seg_count, seg_start, gu_items, dn_items,
        row_token, row_weight, row_dest, slot_row, x_perm, h, slots, total;
};

Plan make_plan(const moe_dims& d, const moe_opts* o) {
    Plan p{};
    p.T = d.T; p.D = d.D; p.E = d.E; p.k = d.k; p.I = d.I;
    p.has_shared = (o && o->shared_gate_up) ? 1 : 0;
    p.I_s = p.has_shared ? o->I_s : 0;
    p.S = p.k + p.has_shared;
    p.R = p.T * p.k + (p.has_shared ? p.T : 0);
    p.ld_h = p.I > p.I_s ? p.I : p.I_s;
    p.nchunks = (int)(((long)p.T * p.k + kPermChunk - 1) / kPermChunk);
    p.nseg = p.E + p.has_shared;
    p.rsplit = p.T <= kRouterSmallMaxT ? 1 : router_splits(p.T, p.E, p.D, kRtBN);
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t at = off; off += align_up(bytes); return at; };
    // [0] error word, [1] routing ticket; then (decode kernel) the E flagged logits
    p.err = take(kAlign + (size_t)p.E * 8);
    // split-tail tickets of gate_up and of down, the per-expert completion counters, and a
    // block of counters that no kernel increments (the watchdog diagnostic); all follow err,
    // so one memset clears the header
    p.tickets = take((size_t)kTicketInts * 4);
    // split-tail partial accumulators: gate_up (two accumulators), then down (one)
    p.partial = take(use_narrow_tiles(p.T, p.k, p.E)
                         ? (size_t)kSplitSlots * 3 * kTcM * kNarrowBN * 4 : 0);
    p.logits = take((size_t)p.rsplit * p.T * p.E * 4);   // router partial sums (or logits)
    p.idx = take((size_t)p.T * p.k * 4);
    p.w = take((size_t)p.T * p.k * 4);
    p.counts = take((size_t)(p.E + 1) * 4);
    p.offsets = take((size_t)(p.E + 2) * 4);
    p.chunk = take((size_t)p.nchunks * p.E * 4);
    p.seg_count = take((size_t)(p.nseg + 1) * 4);
    p.seg_start = take((size_t)(p.nseg + 1) * 4);
    p.gu_items = take((size_t)(p.nseg + 2) * 4);
    p.dn_items = take((size_t)(p.nseg + 2) * 4);
    p.row_token = take((size_t)p.R * 4);
    p.row_weight = take((size_t)p.R * 4);
    p.row_dest = take((size_t)p.R * 4);
    p.slot_row = take((size_t)p.T * p.k * 4);
    p.x_perm = take(p.T <= kGatherMaxT ? 0 : (size_t)p.R * p.D * 2);
    p.h = take((size_t)p.R * p.ld_h * 2);
    p.slots = take((size_t)p.T * p.S * p.D * 4);
    p.total = off;
    return p;
}

moe_status check_dims(const moe_dims* d) {
    if (!d) return MOE_ERR_INVALID_ARG;
    if (d->T < 1 || d->D < 1 || d->E < 1 || d->k < 1 || d->I < 1) return MOE_ERR_INVALID_ARG;
    if (d->norm_topk_prob != 0 && d->norm_topk_prob != 1) return MOE_ERR_INVALID_ARG;
    if (d->E > kMaxE || d->k > kMaxK || d->k > d->E) return MOE_ERR_UNSUPPORTED;
    if (d->D % 128 != 0 || d->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (d->tile_m < 1 || d->tile_m > 256) return MOE_ERR_UNSUPPORTED;
    if ((long long)d->T * (d->k + 1) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    if ((long long)d->T * d->D >= (1ll << 40)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

moe_status check_opts(const moe_dims* d, const moe_opts* o) {
    if (!o) return MOE_OK;
    if (o->shared_gate_up) {
        if (!o->shared_down) return MOE_ERR_INVALID_ARG;
        if (o->I_s < 1) return MOE_ERR_INVALID_ARG;
        if (o->I_s % 128 != 0) return MOE_ERR_UNSUPPORTED;
        if (!aligned(o->shared_gate_up, 16) || !aligned(o->shared_down, 16)) return MOE_ERR_INVALID_ARG;
        if (o->shared_gate && !aligned(o->shared_gate, 16)) return MOE_ERR_INVALID_ARG;
    } else if (o->shared_down || o->shared_gate) {
        return MOE_ERR_INVALID_ARG;
    }
    if (o->router_bias && !aligned(o->router_bias, 4)) return MOE_ERR_INVALID_ARG;
    if (o->residual && !aligned(o->residual, 16)) return MOE_ERR_INVALID_ARG;
    if (o->logits_out && !aligned(o->logits_out, 4)) return MOE_ERR_INVALID_ARG;
    if (o->topk_idx_out && !aligned(o->topk_idx_out, 4)) return MOE_ERR_INVALID_ARG;
    if (o->topk_w_out && !aligned(o->topk_w_out, 4)) return MOE_ERR_INVALID_ARG;
    if (o->path != MOE_PATH_AUTO && o->path != MOE_PATH_GROUPED && o->path != MOE_PATH_DECODE)
        return MOE_ERR_INVALID_ARG;
    if (o->expert_counts_out && !aligned(o->expert_counts_out, 4)) return MOE_ERR_INVALID_ARG;
    if (o->slot_row_out && !aligned(o->slot_row_out, 4)) return MOE_ERR_INVALID_ARG;
    if (o->diag != 0 && o->diag != MOE_DIAG_UNSIGNALLED_HANDOFF && o->diag != MOE_DIAG_DECODE_BARRIER)
        return MOE_ERR_INVALID_ARG;
    if (o->diag == MOE_DIAG_UNSIGNALLED_HANDOFF && !use_narrow_tiles(d->T, d->k, d->E))
        return MOE_ERR_UNSUPPORTED;
    if (o->n_stage_events != 0 && o->n_stage_events != 6) return MOE_ERR_INVALID_ARG;
    if (o->n_stage_events == 6 && !o->stage_events) return MOE_ERR_INVALID_ARG;
    if (o->out_f32 && !aligned(o->out_f32, 16)) return MOE_ERR_INVALID_ARG;
    if (o->W_gate_up_fp8 || o->W_down_fp8 || o->gate_up_scale || o->down_scale) {
        if (!o->W_gate_up_fp8 || !o->W_down_fp8 || !o->gate_up_scale || !o->down_scale)
            return MOE_ERR_INVALID_ARG;
        if (!aligned(o->W_gate_up_fp8, 16) || !aligned(o->W_down_fp8, 16) ||
            !aligned(o->gate_up_scale, 4) || !aligned(o->down_scale, 4))
            return MOE_ERR_INVALID_ARG;
        if (o->shared_gate_up || !use_narrow_tiles(d->T, d->k, d->E)) return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

// Ring depth of the decode kernel for this call on `sms` blocks, 0 when it does not apply:
// more than one token, or a feature it does not implement (shared expert, the
// permutation outputs, the grouped path's diagnostic).
int decode_stages_for(const moe_dims& d, const moe_opts* o, int sms) {
    if (o && (o->shared_gate_up || o->expert_counts_out || o->slot_row_out ||
              o->diag == MOE_DIAG_UNSIGNALLED_HANDOFF))
        return 0;
    return decode_stages(d.T, d.D, d.E, d.k, d.I, sms, o && o->W_gate_up_fp8);
}

// The path moe_forward_ex takes (arguments already checked).
int choose_path(const moe_dims& d, const moe_opts* o, int sms, int* dec_stages) {
    const int want = o ? o->path : MOE_PATH_AUTO;
    *dec_stages = want == MOE_PATH_GROUPED ? 0 : decode_stages_for(d, o, sms);
    if (want == MOE_PATH_DECODE || (o && o->diag == MOE_DIAG_DECODE_BARRIER))
        return *dec_stages > 0 ? MOE_PATH_DECODE : -1;
    return *dec_stages > 0 ? MOE_PATH_DECODE : MOE_PATH_GROUPED;
}

// ------------------------------------------------------------------ device properties / TMA

// SM count of the current device; on failure 0, with the CUDA error kept for
// moe_last_cuda_error.
int num_sms_of_current_device() {
    const int n = device_sm_count();
    if (n <= 0) {
        int dev = 0;
        const cudaError_t e = cudaGetDevice(&dev);
        g_last_cuda_error = e != cudaSuccess ? (int)e : (int)cudaErrorInvalidDevice;
    }
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 map over a row-major [rows, cols] tensor, box {64 columns, box_rows rows}, in the
// 128-byte swizzle layout that the tcgen05 shared-memory descriptors expect.
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)kTcK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) g_last_cuda_error = (int)cudaErrorInvalidValue;
    return r == CUDA_SUCCESS;
}

// FP8 weights [rows, cols] bytes: boxes of 64 columns (one K step) x 128 rows, unswizzled
// (the converter warps read them row by row).
bool make_map8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {(cuuint32_t)kTcK, (cuuint32_t)kTcM};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) g_last_cuda_error = (int)cudaErrorInvalidValue;
    return r == CUDA_SUCCESS;
}

// gate_up [E, 2*Iseg, D] (gate rows, then up rows, per expert) viewed as 5-D {D, 16 rows,
// gate|up, Iseg/16 groups, E} with box {64, 16, 2, 4, 1}: one load brings 64 columns of four
// 16-feature groups, each as 16 gate rows followed by the 16 matching up rows -- the
// interleaved A tile of the wide gate_up kernel (128 rows, 128-byte swizzle).
bool make_map_gate_up_il(CUtensorMap* m, const void* base, uint64_t D, uint64_t Iseg, uint64_t E) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[5] = {D, 16, 2, Iseg / 16, E};
    cuuint64_t strides[4] = {D * 2, Iseg * D * 2, 16 * D * 2, 2 * Iseg * D * 2};
    cuuint32_t box[5] = {(cuuint32_t)kTcK, 16, 2, (cuuint32_t)(kGuILFeatures / 16), 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) g_last_cuda_error = (int)cudaErrorInvalidValue;
    return r == CUDA_SUCCESS;
}

// The token-operand map at every box height up to max_rows.
bool make_b_maps(CUtensorMap* maps, const void* base, uint64_t cols, uint64_t rows, int max_rows) {
    for (int bi = 0; bi < kNumBBoxes; ++bi) {
        const uint32_t box = 16u << bi;
        if ((int)box > max_rows) {
            maps[bi] = maps[bi - 1];
            continue;
        }
        if (!make_map(&maps[bi], base, cols, rows, box)) return false;
    }
    return true;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

#define MOE_CUDA(expr)                                       \
    do {                                                     \
        const cudaError_t e_ = (expr);                       \
        if (e_ != cudaSuccess) {                             \
            g_last_cuda_error = (int)e_;                     \
            return MOE_ERR_CUDA;                             \
        }                                                    \
    } while (0)

// Stage events are recorded as external events so that, under stream capture, they become
// event-record nodes of the graph (a plain record would only order captured work).
moe_status record(const moe_opts* o, int i, cudaStream_t s) {
    if (o && o->n_stage_events == 6) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        MOE_CUDA(cudaStreamIsCapturing(s, &cs));
        const unsigned flags =
            cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
        MOE_CUDA(cudaEventRecordWithFlags(reinterpret_cast<cudaEvent_t>(o->stage_events[i]), s,
                                          flags));
    }
    return MOE_OK;
}

SegTables tables_of(const Plan& p, void* ws) {
    SegTables t;
    t.seg_count = at<int>(ws, p.seg_count);
    t.seg_start = at<int>(ws, p.seg_start);
    t.gu_items = at<int>(ws, p.gu_items);
    t.dn_items = at<int>(ws, p.dn_items);
    return t;
}

// Router logits without the bias, as p.rsplit partial sums [rsplit, T, E] at part: CUDA-core
// kernel for small T (one partial), tcgen05 GEMM with K split in rsplit slices otherwise.
// Launched without chaining: it reads the caller's x.
moe_status run_logits(const moe_bf16* x, const moe_bf16* W_r, const Plan& p, float* part, void* ws,
                      cudaStream_t s) {
    if (p.T <= kRouterSmallMaxT) {
        MOE_CUDA(launch_router_small(x, W_r, p.T, p.D, p.E, part, false, s));
        return MOE_OK;
    }
    TcMaps maps;
    if (!make_map(&maps.A, W_r, p.D, p.E, kTcM)) return MOE_ERR_CUDA;
    maps.A_shared = maps.A;
    if (!make_b_maps(maps.B, x, p.D, p.T, kRtBN)) return MOE_ERR_CUDA;
    TcArgs a{};
    a.D = p.D; a.E = p.E; a.T = p.T; a.I = p.I; a.nseg = 1;
    a.logits = part;
    a.ksplit = p.rsplit;
    a.err = at<int>(ws, p.err);
    a.wait_ns = kWaitLimitNs;
    const int sms = num_sms_of_current_device();
    if (sms <= 0) return MOE_ERR_CUDA;
    MOE_CUDA(launch_tc_router(maps, a, sms, false, s));
    return MOE_OK;
}

}  // namespace

namespace moe {
void note_cuda_error(int e) { g_last_cuda_error = e; }
}  // namespace moe

extern "C" {

size_t moe_workspace_size(const moe_dims* dims, const moe_opts* opts) {
    if (check_dims(dims) != MOE_OK || check_opts(dims, opts) != MOE_OK) return 0;
    return make_plan(*dims, opts).total;
}

int moe_last_cuda_error(void) { return g_last_cuda_error; }

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    }
    return "MOE_ERR_UNKNOWN";
}

moe_status moe_route(const moe_bf16* x, const moe_bf16* W_r, const float* bias,
                     const moe_dims* dims, float* logits, int32_t* topk_idx, float* topk_w,
                     void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!x || !W_r || !topk_idx || !topk_w || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(W_r, 16) || !aligned(ws, kAlign)) return MOE_ERR_INVALID_ARG;
    if ((bias && !aligned(bias, 4)) || (logits && !aligned(logits, 4)) ||
        !aligned(topk_idx, 4) || !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    const Plan p = make_plan(*dims, nullptr);
    if (ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    MOE_CUDA(cudaMemsetAsync(at<int>(ws, p.err), 0, sizeof(int), s));
    float* part = at<float>(ws, p.logits);
    moe_status st2 = run_logits(x, W_r, p, part, ws, s);
    if (st2 != MOE_OK) return st2;
    MOE_CUDA(launch_select(part, p.rsplit, bias, p.T, p.E, p.k, dims->norm_topk_prob, topk_idx,
                           topk_w, logits, true, s));
    return MOE_OK;
}

moe_status moe_permute(const int32_t* topk_idx, const float* topk_w, const moe_bf16* x,
                       const moe_dims* dims, int32_t* counts, int32_t* offsets,
                       int32_t* row_token, int32_t* slot_row, float* row_weight,
                       moe_bf16* x_perm, int cap, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if (!topk_idx || !counts || !offsets || !row_token || !slot_row || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(topk_idx, 4) || !aligned(counts, 4) || !aligned(offsets, 4) ||
        !aligned(row_token, 4) || !aligned(slot_row, 4) || !aligned(ws, kAlign))
        return MOE_ERR_INVALID_ARG;
    if ((topk_w && !aligned(topk_w, 4)) || (row_weight && !aligned(row_weight, 4)))
        return MOE_ERR_INVALID_ARG;
    if ((x_perm && !x) || (x && !aligned(x, 16)) || (x_perm && !aligned(x_perm, 16)))
        return MOE_ERR_INVALID_ARG;
    const long long need = (long long)dims->T * dims->k + (long long)dims->E * (dims->tile_m - 1);
    if (cap < need) return MOE_ERR_INVALID_ARG;
    const Plan p = make_plan(*dims, nullptr);
    if (ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    MOE_CUDA(cudaMemsetAsync(at<int>(ws, p.err), 0, sizeof(int), s));
    PermuteArgs a{};
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.T = p.T; a.k = p.k; a.E = p.E; a.tile_m = dims->tile_m;
    a.has_shared = 0;
    a.slots_per_token = p.k;
    a.D = p.D; a.I = p.I; a.I_s = 0;
    a.chunk_counts = at<int>(ws, p.chunk);
    a.nchunks = p.nchunks;
    a.counts = counts;
    a.offsets = offsets;
    a.row_token = row_token;
    a.row_weight = topk_w ? row_weight : nullptr;
    a.row_dest = nullptr;
    a.slot_row = slot_row;
    a.cap = cap;
    a.tables = SegTables{nullptr, nullptr, nullptr, nullptr};
    a.gu_bn = kGuBN;
    a.dn_bn = kDnBN;
    a.gu_features = kGuILFeatures;
    a.dn_rows = kTcM;
    a.err = at<int>(ws, p.err);
    // padding rows are only written per expert segment; rows past offsets[E] stay as given,
    // so mark every row as padding first
    MOE_CUDA(cudaMemsetAsync(row_token, 0xFF, (size_t)cap * sizeof(int32_t), s));
    if (a.row_weight) MOE_CUDA(cudaMemsetAsync(a.row_weight, 0, (size_t)cap * sizeof(float), s));
    MOE_CUDA(launch_permute(a, false, s));
    if (x_perm) MOE_CUDA(launch_gather_rows(x, row_token, cap, p.D, x_perm, true, s));
    return MOE_OK;
}

moe_status moe_forward_ex(const moe_bf16* x, const moe_bf16* W_r, const moe_bf16* W_gate_up,
                          const moe_bf16* W_down, const moe_dims* dims, const moe_opts* opts,
                          moe_bf16* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    st = check_opts(dims, opts);
    if (st != MOE_OK) return st;
    // FP8 weights replace the bf16 expert tensors (which may then be NULL)
    const bool f8 = opts && opts->W_gate_up_fp8;
    if (!x || !W_r || (!f8 && (!W_gate_up || !W_down)) || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(W_r, 16) || !aligned(W_gate_up, 16) || !aligned(W_down, 16) ||
        !aligned(out, 16) || !aligned(ws, kAlign))
        return MOE_ERR_INVALID_ARG;
    if (out == x) return MOE_ERR_INVALID_ARG;
    const Plan p = make_plan(*dims, opts);
    if (ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int sms = num_sms_of_current_device();
    if (sms <= 0) return MOE_ERR_CUDA;

    int* err = at<int>(ws, p.err);
    float* logits_user = opts ? opts->logits_out : nullptr;
    int32_t* idx = (opts && opts->topk_idx_out) ? opts->topk_idx_out : at<int32_t>(ws, p.idx);
    float* w = (opts && opts->topk_w_out) ? opts->topk_w_out : at<float>(ws, p.w);
    const float* bias = opts ? opts->router_bias : nullptr;
    const moe_bf16* sgu = opts ? opts->shared_gate_up : nullptr;
    const moe_bf16* sdn = opts ? opts->shared_down : nullptr;
    const moe_bf16* sg = opts ? opts->shared_gate : nullptr;
    const moe_bf16* residual = opts ? opts->residual : nullptr;
    float* out_f32 = opts ? opts->out_f32 : nullptr;
    const unsigned long long wait_ns =
        (opts && opts->wait_limit_us) ? (unsigned long long)opts->wait_limit_us * 1000ull : kWaitLimitNs;
    const bool chain = !(opts && opts->n_stage_events == 6);

    int dec_stages = 0;
    const int path = choose_path(*dims, opts, sms, &dec_stages);
    if (path < 0) return MOE_ERR_UNSUPPORTED;
    if (path == MOE_PATH_DECODE) {
        // one kernel: the stage events around it mark routing as the whole block
        MOE_CUDA(cudaMemsetAsync(err, 0, p.tickets - p.err + (size_t)kTicketInts * 4, s));
        if ((st = record(opts, 0, s)) != MOE_OK) return st;
        DecodeArgs da{};
        da.x = x; da.W_r = W_r; da.bias = bias; da.W_gu = W_gate_up; da.W_dn = W_down;
        if (f8) {
            da.W_gu8 = opts->W_gate_up_fp8; da.W_dn8 = opts->W_down_fp8;
            da.gu_scale = opts->gate_up_scale; da.dn_scale = opts->down_scale;
        }
        da.residual = residual; da.out = out; da.out_f32 = out_f32;
        da.logits_out = logits_user; da.idx_out = idx; da.w_out = w;
        da.lgf = reinterpret_cast<unsigned long long*>(at<char>(ws, p.err) + kAlign);
        da.h = at<uint16_t>(ws, p.h);
        da.bar = reinterpret_cast<unsigned*>(at<int>(ws, p.tickets) + kDecBarAt);
        da.err = err;
        da.D = p.D; da.E = p.E; da.k = p.k; da.I = p.I; da.norm = dims->norm_topk_prob;
        da.stages = dec_stages;
        da.wait_ns = wait_ns;
        da.extra_blocks = (opts && opts->diag == MOE_DIAG_DECODE_BARRIER) ? 1 : 0;
        MOE_CUDA(launch_decode(da, sms, chain, s));
        for (int i = 1; i < 6; ++i)
            if ((st = record(opts, i, s)) != MOE_OK) return st;
        return MOE_OK;
    }

    // tensor maps of the grouped path are encoded before anything is enqueued
    // narrow tiles (deeper pipelines) when experts average few rows; a segment with more
    // rows than a tile is simply split into several token tiles.  gate_up token rows: for
    // T <= kGatherMaxT gathered from x (one-row box, tile::gather4), else a permuted copy.
    const bool narrow = use_narrow_tiles(p.T, p.k, p.E);
    const bool gather = p.T <= kGatherMaxT;
    // Wide shapes: gate_up on CTA pairs; down on CTA pairs when its rows split into 256-row
    // tiles and experts average at least 256 rows (measured on B200: with fewer rows the
    // pair tiles' narrower N and halved item count cost more than the pairs save).
    // (devices that cannot co-schedule the pairs take the one-CTA wide tiles)
    const bool pairs = !narrow && pair_tiles_available();
    const int gu_tiles = narrow ? kTilesNarrow : (pairs ? kTilesPair : kTilesWide);
    const int dn_tiles = narrow ? kTilesNarrow
                         : (pairs && p.D % 256 == 0 && (long long)p.T * p.k >= 256ll * p.E)
                               ? kTilesPair
                               : kTilesWide;
    const int gu_bn = narrow ? kNarrowBN : kGuBN;
    const int dn_bn = narrow ? kNarrowBN : kDnBN;
    const int b_box_max = gu_tiles == kTilesPair ? kGuBN / 2 : gu_bn;   // token rows per CTA
    TcMaps mGu, mDn;
    {
        uint16_t* h = at<uint16_t>(ws, p.h);
        const bool gu_b_ok = gather ? make_map(&mGu.B[0], x, p.D, p.T, 1)
                                    : make_b_maps(mGu.B, at<uint16_t>(ws, p.x_perm), p.D, p.R, b_box_max);
        // weight maps: bf16, or (FP8 weights) the byte maps, with the bf16 slots holding copies
        // of those (the F8 kernels read only A8; every descriptor passed stays valid)
        bool a_ok;
        if (f8) {
            a_ok = make_map8(&mGu.A8, opts->W_gate_up_fp8, p.D, (uint64_t)p.E * 2 * p.I) &&
                   make_map8(&mDn.A8, opts->W_down_fp8, p.I, (uint64_t)p.E * p.D);
            mGu.A = mGu.A_shared = mGu.A8;
            mDn.A = mDn.A_shared = mDn.A8;
        } else {
            a_ok = (narrow ? make_map(&mGu.A, W_gate_up, p.D, (uint64_t)p.E * 2 * p.I, kTcM) &&
                                 make_map(&mGu.A_shared, sgu ? sgu : W_gate_up, p.D,
                                          sgu ? 2 * (uint64_t)p.I_s : 2 * (uint64_t)p.I, kTcM)
                           : make_map_gate_up_il(&mGu.A, W_gate_up, p.D, p.I, p.E) &&
                                 make_map_gate_up_il(&mGu.A_shared, sgu ? sgu : W_gate_up, p.D,
                                                     sgu ? p.I_s : p.I, 1)) &&
                   make_map(&mDn.A, W_down, p.I, (uint64_t)p.E * p.D, kTcM) &&
                   make_map(&mDn.A_shared, sdn ? sdn : W_down, sdn ? p.I_s : p.I, p.D, kTcM);
            mGu.A8 = mGu.A;
            mDn.A8 = mDn.A;
        }
        if (!a_ok || !gu_b_ok ||
            !make_b_maps(mDn.B, h, p.ld_h, p.R, dn_tiles == kTilesPair ? kDnBN / 2 : dn_bn))
            return MOE_ERR_CUDA;
        if (gather)
            for (int bi = 1; bi < kNumBBoxes; ++bi) mGu.B[bi] = mGu.B[0];
    }

    // the header of the workspace: device error word, routing ticket, tickets and counters
    MOE_CUDA(cudaMemsetAsync(err, 0, p.tickets - p.err + (size_t)kTicketInts * 4, s));
    if ((st = record(opts, 0, s)) != MOE_OK) return st;
    // Router logits (partial sums), then selection and permutation: one kernel while T*k
    // fits a single permutation block, else selection and the three permutation kernels.
    const bool select_permute = (long long)p.T * p.k <= kPermChunk;
    float* part = at<float>(ws, p.logits);
    if ((st = run_logits(x, W_r, p, part, ws, s)) != MOE_OK) return st;
    if (!select_permute)
        MOE_CUDA(launch_select(part, p.rsplit, bias, p.T, p.E, p.k, dims->norm_topk_prob, idx, w,
                               logits_user, true, s));
    if ((st = record(opts, 1, s)) != MOE_OK) return st;

    PermuteArgs pa{};
    pa.topk_idx = idx;
    pa.topk_w = w;
    pa.T = p.T; pa.k = p.k; pa.E = p.E; pa.tile_m = 1;
    pa.has_shared = p.has_shared;
    pa.slots_per_token = p.S;
    pa.D = p.D; pa.I = p.I; pa.I_s = p.I_s;
    pa.chunk_counts = at<int>(ws, p.chunk);
    pa.nchunks = p.nchunks;
    pa.counts = (opts && opts->expert_counts_out) ? opts->expert_counts_out : at<int>(ws, p.counts);
    pa.offsets = at<int>(ws, p.offsets);
    pa.row_token = at<int32_t>(ws, p.row_token);
    pa.row_weight = at<float>(ws, p.row_weight);
    pa.row_dest = at<int32_t>(ws, p.row_dest);
    pa.slot_row = (opts && opts->slot_row_out) ? opts->slot_row_out : at<int32_t>(ws, p.slot_row);
    pa.cap = p.R;
    pa.tables = tables_of(p, ws);
    pa.gu_bn = gu_bn;
    pa.dn_bn = dn_bn;
    pa.gu_features = gu_tiles == kTilesWide ? kGuILFeatures : kTcM;
    pa.dn_rows = dn_tiles == kTilesPair ? 2 * kTcM : kTcM;
    pa.err = err;
    // launch chaining between the forward's kernels (not across a stage-event record)
    RouteArgs ra{};
    ra.bias = bias;
    ra.T = p.T; ra.E = p.E; ra.k = p.k; ra.norm = dims->norm_topk_prob;
    ra.topk_idx = idx;
    ra.topk_w = w;
    ra.ticket = err + 1;
    ra.perm = pa;
    if (select_permute) {
        ra.logits_out = logits_user;
        ra.part = part;
        ra.nsplit = p.rsplit;
        MOE_CUDA(launch_select_permute(ra, chain, s));
    } else {
        MOE_CUDA(launch_permute(pa, chain, s));
    }
    if (!gather)
        MOE_CUDA(launch_gather_rows(x, pa.row_token, p.R, p.D, at<uint16_t>(ws, p.x_perm), true, s));
    if ((st = record(opts, 2, s)) != MOE_OK) return st;

    int* tickets = at<int>(ws, p.tickets);
    TcArgs ta{};
    ta.D = p.D; ta.I = p.I; ta.I_s = p.I_s; ta.E = p.E; ta.nseg = p.nseg; ta.T = p.T;
    ta.tables = pa.tables;
    ta.row_token = pa.row_token;
    ta.gather = gather ? 1 : 0;
    ta.h = at<uint16_t>(ws, p.h);
    ta.ld_h = p.ld_h;
    ta.row_weight = pa.row_weight;
    ta.row_dest = pa.row_dest;
    ta.slots = at<float>(ws, p.slots);
    ta.partial = narrow ? at<float>(ws, p.partial) : nullptr;
    ta.tickets = tickets;
    ta.partial_slots = narrow ? kSplitSlots : 0;
    // narrow tiles: gate_up reports each finished expert; down waits per expert
    ta.seg_done = narrow ? tickets + 2 * kSplitTickets : nullptr;
    ta.gu_prefix = pa.tables.gu_items;
    ta.sched = tickets + kSchedAt;
    // every expert very likely has rows (T*k >= 4E): the first wave of gate_up units is known
    // up to that guess, and its weights start towards L2 while routing runs (12 of the K steps
    // of each first unit: about 57 MB at D = 2048 on 148 SMs, well inside L2)
    ta.spec_steps = (narrow && (long long)p.T * p.k >= 4ll * p.E) ? min(12, p.D / kTcK) : 0;
    ta.err = err;
    ta.wait_ns = wait_ns;
    TcArgs tdn = ta;
    tdn.spec_steps = 0;
    tdn.dep_wait = narrow ? 1 : 0;
    tdn.sched = tickets + kSchedAt + 1;
    if (narrow) {
        tdn.partial = at<float>(ws, p.partial) + (size_t)kSplitSlots * 2 * kTcM * kNarrowBN;
        tdn.tickets = tickets + kSplitTickets;
        // watchdog diagnostic: down watches counters that no kernel increments
        if (opts && opts->diag == MOE_DIAG_UNSIGNALLED_HANDOFF)
            tdn.seg_done = tickets + 2 * kSplitTickets + (kMaxSegments + 1);
    }
    const int grid = sms < kMaxTcGrid ? sms : kMaxTcGrid;
    if (f8) {
        ta.a_scale = opts->gate_up_scale;
        tdn.a_scale = opts->down_scale;
    }
    MOE_CUDA(launch_tc_gate_up(mGu, ta, grid, gu_tiles, f8, chain, s));
    if ((st = record(opts, 3, s)) != MOE_OK) return st;
    MOE_CUDA(launch_tc_down(mDn, tdn, grid, dn_tiles, f8, chain, s));
    if ((st = record(opts, 4, s)) != MOE_OK) return st;
    MOE_CUDA(launch_combine(ta.slots, p.T, p.D, p.k, p.has_shared, x, sg, residual, out,
                            out_f32, chain, s));
    return record(opts, 5, s);
}

moe_status moe_forward_path(const moe_dims* dims, const moe_opts* opts, int* path_out) {
    moe_status st = check_dims(dims);
    if (st != MOE_OK) return st;
    if ((st = check_opts(dims, opts)) != MOE_OK) return st;
    if (!path_out) return MOE_ERR_INVALID_ARG;
    const int sms = num_sms_of_current_device();
    if (sms <= 0) return MOE_ERR_CUDA;
    int dec_stages = 0;
    const int path = choose_path(*dims, opts, sms, &dec_stages);
    if (path < 0) return MOE_ERR_UNSUPPORTED;
    *path_out = path;
    return MOE_OK;
}

moe_status moe_forward(const moe_bf16* x, const moe_bf16* W_r, const moe_bf16* W_gate_up,
                       const moe_bf16* W_down, const moe_dims* dims, moe_bf16* out, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
    return moe_forward_ex(x, W_r, W_gate_up, W_down, dims, nullptr, out, ws, ws_bytes, stream);
}

moe_status moe_get_device_status(const void* ws, moe_stream_t stream) {
    if (!ws || !aligned(ws, kAlign)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    int word = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        g_last_cuda_error = (int)e;
        return MOE_ERR_CUDA;
    }
    if (word & kErrBadIndex) return MOE_ERR_INVALID_ARG;
    if (word) return MOE_ERR_DEVICE_TIMEOUT;
    return MOE_OK;
}

}  // extern "C"
