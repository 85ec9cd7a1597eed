// stream.cu -- the small-T path: stream each touched expert's weights once.
//
// "27. Mixture of experts" (inference.shantanugoel.com), section "The economics of MoE
// inference": a decode step only reads the experts its tokens chose, and at small batch the
// layer is bound by those weight bytes, not by arithmetic.  These kernels therefore read
// every weight of a touched expert exactly once, from HBM straight into registers with
// coalesced 16-byte loads, and apply it to all of that expert's tokens (swap-AB: weight
// rows play the MMA's M, tokens its N).  The expert is the SwiGLU of the same page's
// section "Dispatch": down(silu(gate x) * up x), gate rows first in gate_up [2I, D].
//
// Both kernels use the warp-level m16n8k16 bf16 MMA as the FMA engine: its operands live in
// registers, so a weight fragment goes from the load straight into the multiply with no
// shared-memory or TMEM staging.  Each lane loads 8 consecutive bf16 of a row (16 bytes);
// A and B fragments apply the same permutation of K inside each 32-element chunk, which
// leaves every dot product unchanged.
//
// gate_up: a warp owns 8 features of one segment: MMA rows 0-7 are their gate rows and rows
//          8-15 their up rows, so one thread holds gate and up of the same (feature, token)
//          and applies SwiGLU in registers; h is written in bf16 (the precision the down
//          projection consumes).
// down:    a warp owns 16 output features of one segment; outputs are scaled by the routing
//          weight in FP32 and stored to the token's FP32 slot, summed later in slot order.
#include "common.cuh"

namespace moe {

constexpr int kStreamThreads = 128;

template <int NB>
__global__ void __launch_bounds__(kStreamThreads) stream_gate_up_kernel(StreamArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int nseg = a.nseg;
    const int total = __ldg(a.tables.gu_tasks + nseg);
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int D = a.D;
    for (int task = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; task < total; task += nwarps) {
        const int s = find_segment(a.tables.gu_tasks, nseg, task);
        const int fg = task - __ldg(a.tables.gu_tasks + s);
        const bool shared = (s == a.E);
        const int Iseg = shared ? a.I_s : a.I;
        const uint16_t* W = shared ? a.S_gu : a.W_gu + (size_t)s * 2 * a.I * D;
        const uint16_t* gate_row = W + (size_t)(fg * 8 + g) * D + q * 8;
        const uint16_t* up_row = W + (size_t)(Iseg + fg * 8 + g) * D + q * 8;
        const int cnt = __ldg(a.tables.seg_count + s);
        const int start = __ldg(a.tables.seg_start + s);
        for (int p0 = 0; p0 < cnt; p0 += NB * 8) {
            const int nb = min(NB, (cnt - p0 + 7) >> 3);
            const uint16_t* xr[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                int col = p0 + i * 8 + g;
                col = col < cnt ? col : cnt - 1;  // any valid row for padding columns
                const int t = __ldg(a.row_token + start + col);
                xr[i] = a.x + (size_t)t * D + q * 8;
            }
            float acc[NB][4];
#pragma unroll
            for (int i = 0; i < NB; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll 4
            for (int k0 = 0; k0 < D; k0 += 32) {
                const uint4 ga = ld_stream_v4(gate_row + k0);
                const uint4 ua = ld_stream_v4(up_row + k0);
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (i < nb) {
                        const uint4 xb = ld_v4(xr[i] + k0);
                        mma_bf16_16816(acc[i], ga.x, ua.x, ga.y, ua.y, xb.x, xb.y);
                        mma_bf16_16816(acc[i], ga.z, ua.z, ga.w, ua.w, xb.z, xb.w);
                    }
                }
            }
            const int f = fg * 8 + g;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                if (i < nb) {
                    const int col = p0 + i * 8 + 2 * q;
                    const float h0 = silu(acc[i][0]) * acc[i][2];
                    const float h1 = silu(acc[i][1]) * acc[i][3];
                    if (col < cnt) a.h[(size_t)(start + col) * a.ld_h + f] = to_bf16_bits(h0);
                    if (col + 1 < cnt) a.h[(size_t)(start + col + 1) * a.ld_h + f] = to_bf16_bits(h1);
                }
            }
        }
    }
}

template <int NB>
__global__ void __launch_bounds__(kStreamThreads) stream_down_kernel(StreamArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, q = lane & 3;
    const int nseg = a.nseg;
    const int total = __ldg(a.tables.dn_tasks + nseg);
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int D = a.D;
    for (int task = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; task < total; task += nwarps) {
        const int s = find_segment(a.tables.dn_tasks, nseg, task);
        const int dg = task - __ldg(a.tables.dn_tasks + s);
        const bool shared = (s == a.E);
        const int Iseg = shared ? a.I_s : a.I;
        const uint16_t* W = shared ? a.S_dn : a.W_dn + (size_t)s * D * a.I;
        const int d_lo = dg * 16 + g;
        const uint16_t* row_lo = W + (size_t)d_lo * Iseg + q * 8;
        const uint16_t* row_hi = W + (size_t)(d_lo + 8) * Iseg + q * 8;
        const int cnt = __ldg(a.tables.seg_count + s);
        const int start = __ldg(a.tables.seg_start + s);
        for (int p0 = 0; p0 < cnt; p0 += NB * 8) {
            const int nb = min(NB, (cnt - p0 + 7) >> 3);
            const uint16_t* hr[NB];
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                int col = p0 + i * 8 + g;
                col = col < cnt ? col : cnt - 1;
                hr[i] = a.h + (size_t)(start + col) * a.ld_h + q * 8;
            }
            float acc[NB][4];
#pragma unroll
            for (int i = 0; i < NB; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll 4
            for (int k0 = 0; k0 < Iseg; k0 += 32) {
                const uint4 al = ld_stream_v4(row_lo + k0);
                const uint4 ah = ld_stream_v4(row_hi + k0);
#pragma unroll
                for (int i = 0; i < NB; ++i) {
                    if (i < nb) {
                        const uint4 hb = ld_v4(hr[i] + k0);
                        mma_bf16_16816(acc[i], al.x, ah.x, al.y, ah.y, hb.x, hb.y);
                        mma_bf16_16816(acc[i], al.z, ah.z, al.w, ah.w, hb.z, hb.w);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                if (i < nb) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int col = p0 + i * 8 + 2 * q + c;
                        if (col < cnt) {
                            const int r = start + col;
                            const int dest = __ldg(a.row_dest + r);
                            const float wt = __ldg(a.row_weight + r);
                            float* o = a.slots + (size_t)dest * D;
                            o[d_lo] = wt * acc[i][c];
                            o[d_lo + 8] = wt * acc[i][2 + c];
                        }
                    }
                }
            }
        }
    }
}

static int stream_blocks(int max_tasks) {
    // enough resident warps to keep ~64 KB of loads in flight per SM, no more than the tasks
    const int warps = kStreamThreads / 32;
    int blocks = (max_tasks + warps - 1) / warps;
    const int cap = 148 * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return blocks;
}

cudaError_t launch_stream_gate_up(const StreamArgs& a, int max_rows, bool pdl, cudaStream_t s) {
    // upper bound of warp tasks: every segment touched
    const int max_tasks = a.E * (a.I / 8) + (a.S_gu ? a.I_s / 8 : 0);
    const int blocks = stream_blocks(max_tasks);
    return launch_kernel(max_rows <= 16 ? stream_gate_up_kernel<2> : stream_gate_up_kernel<4>,
                         dim3(blocks), dim3(kStreamThreads), 0, s, pdl, a);
}

cudaError_t launch_stream_down(const StreamArgs& a, int max_rows, bool pdl, cudaStream_t s) {
    const int max_tasks = (a.E + (a.S_dn ? 1 : 0)) * (a.D / 16);
    const int blocks = stream_blocks(max_tasks);
    return launch_kernel(max_rows <= 16 ? stream_down_kernel<2> : stream_down_kernel<4>,
                         dim3(blocks), dim3(kStreamThreads), 0, s, pdl, a);
}

}  // namespace moe
