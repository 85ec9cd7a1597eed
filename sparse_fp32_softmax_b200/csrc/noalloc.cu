// noalloc.cu -- moe_forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point where they
// run the block: plugin hosts that hand a kernel only its input and output buffers and no
// workspace, and runtimes that plan all device memory up front and forbid allocation once
// they have started.  For them the scratch memory of the forward pass lives in a fixed
// array in the library's own device memory, declared below.  Every GPU that loads this
// part of the library keeps that array until the process exits.
//
// The array holds the same workspace moe_forward uses (routing tables, permutation, the
// SwiGLU intermediate and the FP32 slot buffer).  Its size bounds the problem: calls whose
// workspace would exceed it are refused with MOE_ERR_WORKSPACE before anything runs.
// All calls on a device share the one array and each call leaves its contents behind; the
// forward pass clears what must start at zero (the device error word, tickets and counters
// at the start of the array) and overwrites the rest before reading it.  Calls whose work
// can overlap on the GPU (different streams, or different host threads without ordering)
// race on the array and must not be issued.  The error word the last call left stays in
// the array's first int, where moe_get_device_status_noalloc reads it.
#include <mutex>

#include "../../include/moe_b200.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 64ull << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array on the current device, looked up once per device (the
// symbol's host-side name is only a stand-in and must never be passed to a kernel).
void* scratch_address_of_current_device() {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

moe_status moe_forward_noalloc(const moe_bf16* x, const moe_bf16* W_r, const moe_bf16* W_gate_up,
                               const moe_bf16* W_down, const moe_dims* dims, moe_bf16* out,
                               moe_stream_t stream) {
    const size_t need = moe_workspace_size(dims, nullptr);
    if (need == 0) {
        // invalid or unsupported dims: let the regular entry point name the error
        return moe_forward(x, W_r, W_gate_up, W_down, dims, out, nullptr, 0, stream);
    }
    if (need > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
    void* ws = scratch_address_of_current_device();
    if (!ws) return MOE_ERR_CUDA;
    return moe_forward(x, W_r, W_gate_up, W_down, dims, out, ws, kNoAllocScratchBytes, stream);
}

moe_status moe_get_device_status_noalloc(moe_stream_t stream) {
    void* ws = scratch_address_of_current_device();
    if (!ws) return MOE_ERR_CUDA;
    return moe_get_device_status(ws, stream);
}

}  // extern "C"
