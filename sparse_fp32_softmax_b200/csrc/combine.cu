// combine.cu -- weighted sum of each token's expert outputs back in token order.
//
// "27. Mixture of experts" (inference.shantanugoel.com), section "The router":
// y = sum_{i in top-k} w_i expert_i(x); section "The shared expert": + sigmoid(w_s . x) *
// shared(x).  The expert kernels already scaled each routed output by its weight and
// stored it in the token's slot j; this kernel adds the k slots in slot order j = 0..k-1 in
// FP32 (a fixed order, so results are bitwise reproducible), then the gated shared-expert
// slot, then the optional residual, and rounds once to bf16.
#include "common.cuh"

namespace moe {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* p, float (&v)[8]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
    v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
}

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(
    const float* __restrict__ slots, int T, int D, int k, int has_shared,
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ shared_gate,
    const uint16_t* residual, uint16_t* out, float* __restrict__ out_f32) {
    __shared__ float red[kCombineThreads / 32];
    pdl_wait();
    pdl_launch_dependents();
    const int S = k + has_shared;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        float gate = 1.0f;
        if (has_shared && shared_gate) {
            float z = 0.f;
            for (int d = threadIdx.x * 8; d < D; d += kCombineThreads * 8) {
                float xv[8], gv[8];
                load8<uint16_t>(x + (size_t)t * D + d, xv);
                load8<uint16_t>(shared_gate + d, gv);
#pragma unroll
                for (int i = 0; i < 8; ++i) z = fmaf(xv[i], gv[i], z);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = z;
            __syncthreads();
            z = 0.f;
#pragma unroll
            for (int w = 0; w < kCombineThreads / 32; ++w) z += red[w];
            __syncthreads();
            gate = 1.0f / (1.0f + expf(-z));
        }
        const float* base = slots + (size_t)t * S * D;
        for (int d = threadIdx.x * 8; d < D; d += kCombineThreads * 8) {
            float acc[8], v[8];
            load8<float>(base + d, acc);
            // slots j = 1..k-1 in groups of 8: all loads of a group are in flight together,
            // the additions still run in slot order
            for (int j0 = 1; j0 < k; j0 += 8) {
                float g[8][8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (j0 + q < k) load8<float>(base + (size_t)(j0 + q) * D + d, g[q]);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (j0 + q < k) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] += g[q][i];
                    }
            }
            if (has_shared) {
                load8<float>(base + (size_t)k * D + d, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(gate, v[i], acc[i]);
            }
            if (residual) {
                // out may be the residual buffer itself (a residual chain updated in place):
                // each thread reads its 8 elements here, before it writes them below, with a
                // coherent load (not the read-only path)
                const uint4 r = __ldcg(reinterpret_cast<const uint4*>(residual + (size_t)t * D + d));
                v[0] = bf16_lo(r.x); v[1] = bf16_hi(r.x); v[2] = bf16_lo(r.y); v[3] = bf16_hi(r.y);
                v[4] = bf16_lo(r.z); v[5] = bf16_hi(r.z); v[6] = bf16_lo(r.w); v[7] = bf16_hi(r.w);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += v[i];
            }
            if (out_f32) {
                float4* of = reinterpret_cast<float4*>(out_f32 + (size_t)t * D + d);
                of[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                of[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            *reinterpret_cast<uint4*>(out + (size_t)t * D + d) = o;
        }
    }
}

cudaError_t launch_combine(const float* slots, int T, int D, int k, int has_shared,
                           const uint16_t* x, const uint16_t* shared_gate,
                           const uint16_t* residual, uint16_t* out, float* out_f32, bool pdl,
                           cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const int blocks = T < sms * 16 ? T : sms * 16;
    return launch_kernel(combine_kernel, dim3(blocks), dim3(kCombineThreads), 0, s, pdl, slots, T,
                         D, k, has_shared, x, shared_gate, residual, out, out_f32);
}

}  // namespace moe
