// aux_loss.cu -- the Switch balance loss of the router and its gradient with respect to the
// router logits.
//
// "Qwen3-VL and Mixture of Experts" (gopikrishnatummala.com), the fixes for expert collapse,
// "An auxiliary balance loss": L = alpha * N * sum_i f_i P_i over the N experts, f_i the
// fraction of tokens sent to expert i, P_i the router's average probability for it.  The
// Qwen3-VL MoE walk-through (agent.csdn.net), "load_balancing_loss_func": P from the softmax
// of the gate logits averaged over tokens, f from the top-k one-hot averaged over tokens
// (f_i = count_i / T), their dot product times the number of experts.  The gradient holds f
// fixed (the selection is not differentiable):
//   dL/dl[t, e] = alpha * N / T * p[t, e] * (f_e - sum_i f_i p[t, i]).
//
// Three kernels, all sums in a fixed order (bitwise reproducible, no floating-point atomics):
//   1. stats: block b takes a contiguous token range, 16 tokens at a time: one warp per token
//      finds the row max and the sum of exp (as the router's selection does) and writes the
//      token's probabilities to shared memory, then thread e adds p[t, e] in token order; the
//      block counts its assignments per expert (integers);
//   2. finish: one block adds the per-block partials in a fixed order: f, P, the loss;
//   3. gradient (optional): one warp per token.
#include "../../include/moe_b200.h"
#include "common.cuh"

namespace moe {

constexpr int kAuxThreads = 512;        // >= the largest E
constexpr int kAuxMaxBlocks = 148;      // fixed (not the SM count): the sums' order depends only on T
constexpr int kAuxChunk = kAuxThreads / 32;   // tokens whose probabilities a block keeps at once

// Workspace: per-block probability sums [B, E] FP32, per-block counts [B, E] int32, f [E].
struct AuxPlan {
    int blocks, per_block;
    size_t psum, cnt, f, total;
};
inline AuxPlan aux_plan(int T, int E) {
    AuxPlan p;
    p.blocks = (T + kAuxChunk - 1) / kAuxChunk < kAuxMaxBlocks ? (T + kAuxChunk - 1) / kAuxChunk : kAuxMaxBlocks;
    p.per_block = (T + p.blocks - 1) / p.blocks;
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    p.psum = 0;
    p.cnt = up((size_t)p.blocks * E * 4);
    p.f = p.cnt + up((size_t)p.blocks * E * 4);
    p.total = p.f + up((size_t)E * 4);
    return p;
}

// Row max and sum of exp(l - max) of one token's E logits by one warp: lane L takes experts
// L, L + 32, ... in order, then a butterfly.
__device__ __forceinline__ void token_softmax_stats(const float* row, int E, float& m, float& s) {
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int e = lane; e < E; e += 32) mx = fmaxf(mx, row[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int e = lane; e < E; e += 32) sum += expf(row[e] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    m = mx;
    s = sum;
}

__global__ void __launch_bounds__(kAuxThreads) aux_stats_kernel(const float* __restrict__ logits,
                                                               const int32_t* __restrict__ idx, int T, int E,
                                                               int k, int per_block, float* __restrict__ psum,
                                                               int* __restrict__ cnt) {
    __shared__ float s_p[kAuxChunk][kAuxThreads];   // probabilities of the chunk's tokens
    __shared__ int s_cnt[kAuxThreads];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * per_block, t1 = min(T, t0 + per_block);
    s_cnt[threadIdx.x] = 0;
    float acc = 0.f;
    for (int c0 = t0; c0 < t1; c0 += kAuxChunk) {
        const int nt = min(kAuxChunk, t1 - c0);
        if (warp < nt) {   // one warp per token: statistics, then its probabilities
            const float* row = logits + (size_t)(c0 + warp) * E;
            float m, s;
            token_softmax_stats(row, E, m, s);
            for (int e = lane; e < E; e += 32) s_p[warp][e] = expf(row[e] - m) / s;
        }
        __syncthreads();
        const int e = threadIdx.x;
        if (e < E)
            for (int i = 0; i < nt; ++i) acc += s_p[i][e];   // token order
        for (int a = threadIdx.x; a < nt * k; a += kAuxThreads) {
            const int ex = idx[(size_t)c0 * k + a];
            if (ex >= 0 && ex < E) atomicAdd(&s_cnt[ex], 1);   // integers: order-free
        }
        __syncthreads();
    }
    if (threadIdx.x < E) {
        psum[(size_t)blockIdx.x * E + threadIdx.x] = acc;
        cnt[(size_t)blockIdx.x * E + threadIdx.x] = s_cnt[threadIdx.x];
    }
    pdl_launch_dependents();
}

__global__ void __launch_bounds__(kAuxThreads) aux_finish_kernel(const float* __restrict__ psum,
                                                                const int* __restrict__ cnt, int blocks, int T,
                                                                int E, float alpha, float* __restrict__ f,
                                                                float* __restrict__ loss) {
    __shared__ float s_part[kAuxThreads / 32];
    __shared__ float s_ps[kAuxThreads];
    __shared__ int s_c[kAuxThreads];
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // R threads per expert: thread (r, e) adds the partials of blocks r, r + R, ... in order,
    // then thread e adds the R results in order r = 0..R-1 (a fixed order for given T, E)
    const int R = kAuxThreads / E;
    if (threadIdx.x < R * E) {
        const int e = threadIdx.x % E, r = threadIdx.x / E;
        int c = 0;
        float ps = 0.f;
#pragma unroll 4
        for (int b = r; b < blocks; b += R) {
            c += cnt[(size_t)b * E + e];
            ps += psum[(size_t)b * E + e];
        }
        s_ps[threadIdx.x] = ps;
        s_c[threadIdx.x] = c;
    }
    __syncthreads();
    const int e = threadIdx.x;
    float prod = 0.f;
    if (e < E) {
        int c = 0;
        float ps = 0.f;
        for (int r = 0; r < R; ++r) {
            c += s_c[r * E + e];
            ps += s_ps[r * E + e];
        }
        const float fe = (float)c / (float)T, pe = ps / (float)T;
        f[e] = fe;
        prod = fe * pe;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) prod += __shfl_xor_sync(0xffffffffu, prod, o);
    if (lane == 0) s_part[warp] = prod;
    __syncthreads();
    if (threadIdx.x == 0) {
        float sum = 0.f;
        for (int w = 0; w < kAuxThreads / 32; ++w) sum += s_part[w];   // warp order
        *loss = alpha * (float)E * sum;
    }
}

__global__ void __launch_bounds__(256) aux_grad_kernel(const float* __restrict__ logits, const float* __restrict__ f,
                                                       int T, int E, float alpha, float* __restrict__ dlogits) {
    pdl_wait();
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const float c = alpha * (float)E / (float)T;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* row = logits + (size_t)t * E;
        float m, s;
        token_softmax_stats(row, E, m, s);
        float q = 0.f;
        for (int e = lane; e < E; e += 32) q += __ldg(f + e) * (expf(row[e] - m) / s);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        for (int e = lane; e < E; e += 32) {
            const float p = expf(row[e] - m) / s;
            dlogits[(size_t)t * E + e] = c * p * (__ldg(f + e) - q);
        }
    }
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_aux_loss_workspace_size(int T, int E) {
    if (T < 1 || E < 1 || E > kMaxE) return 0;
    return aux_plan(T, E).total;
}

extern "C" moe_status moe_aux_loss(const float* logits, const int32_t* topk_idx, int T, int E, int k, float alpha,
                                   float* loss, float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (T < 1 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
    if (E > kMaxE || k > kMaxK || k > E) return MOE_ERR_UNSUPPORTED;
    if ((long long)T * E >= (1ll << 31) || (long long)T * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    if (!logits || !topk_idx || !loss || !ws) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(topk_idx) |
         reinterpret_cast<uintptr_t>(loss) | reinterpret_cast<uintptr_t>(dlogits)) % 4 ||
        reinterpret_cast<uintptr_t>(ws) % 256)
        return MOE_ERR_INVALID_ARG;
    const AuxPlan p = aux_plan(T, E);
    if (ws_bytes < p.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* w = static_cast<char*>(ws);
    float* psum = reinterpret_cast<float*>(w + p.psum);
    int* cnt = reinterpret_cast<int*>(w + p.cnt);
    float* f = reinterpret_cast<float*>(w + p.f);
    cudaError_t e = launch_kernel(aux_stats_kernel, dim3(p.blocks), dim3(kAuxThreads), 0, s, false, logits, topk_idx,
                                  T, E, k, p.per_block, psum, cnt);
    if (e == cudaSuccess)
        e = launch_kernel(aux_finish_kernel, dim3(1), dim3(kAuxThreads), 0, s, true, (const float*)psum,
                          (const int*)cnt, p.blocks, T, E, alpha, f, loss);
    if (e == cudaSuccess && dlogits) {
        const int blocks = (T + 7) / 8 < 148 * 16 ? (T + 7) / 8 : 148 * 16;
        e = launch_kernel(aux_grad_kernel, dim3(blocks), dim3(256), 0, s, true, logits, (const float*)f, T, E,
                          alpha, dlogits);
    }
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
