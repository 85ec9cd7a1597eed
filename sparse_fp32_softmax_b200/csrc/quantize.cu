// quantize.cu -- per-row FP8 (E4M3) quantisation of expert weight matrices.
//
// Low-precision experts ("27. Mixture of experts", section "The economics of MoE inference":
// a decode step reads only the experts its token uses, and low-precision weights shrink those
// bytes; "Qwen3-VL and Mixture of Experts", section "Deploying it": FP8 halves the resident
// weights).  The pages fix no format; this is the plainest per-row (per output channel)
// scheme: scale[r] = max_c |W[r, c]| / 448 (FP32), q[r, c] = E4M3(W[r, c] / scale[r]) rounded to
// nearest even and saturated to +-448 (OCP E4M3 "fn": bias 7, no infinities).
#include "../../include/moe_b200.h"
#include "common.cuh"

namespace moe {

constexpr int kQuantThreads = 256;

// One warp per row: lanes take 16-byte pieces (8 bf16) L, L + 32, ... of the row; the row
// maximum of |w| by a butterfly, then every piece quantised and stored as 8 bytes.
__global__ void __launch_bounds__(kQuantThreads) quantize_fp8_rows_kernel(const uint16_t* __restrict__ W,
                                                                         long long rows, int cols,
                                                                         uint8_t* __restrict__ q,
                                                                         float* __restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const int pieces = cols >> 3;
    for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nw) {
        const uint4* src = reinterpret_cast<const uint4*>(W + (size_t)r * cols);
        float amax = 0.f;
        for (int i = lane; i < pieces; i += 32) {
            const uint4 v = __ldg(src + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        if (lane == 0) scale[r] = s;
        uint2* dst = reinterpret_cast<uint2*>(q + (size_t)r * cols);
        for (int i = lane; i < pieces; i += 32) {
            const uint4 v = __ldg(src + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = make_float2(__fdiv_rn(bf16_lo(w[j]), s), __fdiv_rn(bf16_hi(w[j]), s));
                const uint32_t two = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
                packed[j >> 1] |= (two & 0xFFFFu) << (16 * (j & 1));
            }
            dst[i] = make_uint2(packed[0], packed[1]);
        }
    }
}

}  // namespace moe

extern "C" moe_status moe_quantize_fp8_rows(const moe_bf16* W, int64_t rows, int cols, uint8_t* q,
                                            float* scale, moe_stream_t stream) {
    if (!W || !q || !scale || rows < 0 || cols <= 0 || cols % 16 != 0) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(scale)) % 16)
        return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    const int sms = moe::device_sm_count();
    if (sms <= 0) return MOE_ERR_CUDA;
    const long long per_block = moe::kQuantThreads / 32;
    long long blocks = (rows + per_block - 1) / per_block;
    if (blocks > (long long)sms * 16) blocks = (long long)sms * 16;
    moe::quantize_fp8_rows_kernel<<<(unsigned)blocks, moe::kQuantThreads, 0,
                                    reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint16_t*>(W), (long long)rows, cols, q, scale);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
