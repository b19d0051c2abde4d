// neox_peer.cu -- CUDA IPC helpers of libneoxshard.so: export a device
// allocation to another process of the same node and map a peer's exported
// allocation, so that the step's kernels can read the peers' gradient slices
// (the ZeRO-2 reduce-scatter fused with pass 1) and store into the peers'
// weight buffers (the all-gather fused with the cast) directly over NVLink.
// Host code only.  C ABI in include/neox_shard.h.
//
// Pages followed: "GPT-NeoX: how it opened the door to democratised
// 100B-scale training" (ainews.cool), "技术深度解析" (technical deep-dive):
// data parallelism with ZeRO pairs with reduce-scatter and all-gather.

#include "neox_shard.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(neox_ipc_handle), "an IPC handle is 64 bytes");

namespace {

thread_local char g_ipc_error[256];

neox_status ipc_fail(const char* what, int code) {
    snprintf(g_ipc_error, sizeof(g_ipc_error), "%s failed (error %d)", what, code);
    return NEOX_ERR_CUDA;
}

// cuMemGetAddressRange through the runtime's driver entry point, so the
// library needs no link-time dependency on the driver library.
using GetRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

GetRangeFn address_range_fn() {
    static GetRangeFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<GetRangeFn>(nullptr);
        return reinterpret_cast<GetRangeFn>(p);
    }();
    return fn;
}

}  // namespace

extern "C" {

const char* neox_ipc_last_error(void) { return g_ipc_error; }

neox_status neox_ipc_export(const void* dev_ptr, neox_ipc_handle* handle, uint64_t* offset) {
    g_ipc_error[0] = 0;
    if (!dev_ptr || !handle || !offset) {
        snprintf(g_ipc_error, sizeof(g_ipc_error), "dev_ptr, handle and offset must be non-NULL");
        return NEOX_ERR_INVALID_ARGUMENT;
    }
    GetRangeFn range = address_range_fn();
    if (!range) return ipc_fail("looking up cuMemGetAddressRange", -1);
    CUdeviceptr base = 0;
    size_t size = 0;
    const CUresult r = range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr));
    if (r != CUDA_SUCCESS) return ipc_fail("cuMemGetAddressRange", (int)r);
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
    if (e != cudaSuccess) return ipc_fail("cudaIpcGetMemHandle", (int)e);
    memcpy(handle->bytes, &h, sizeof(h));
    *offset = reinterpret_cast<CUdeviceptr>(dev_ptr) - base;
    return NEOX_OK;
}

neox_status neox_ipc_open(const neox_ipc_handle* handle, void** base) {
    g_ipc_error[0] = 0;
    if (!handle || !base) {
        snprintf(g_ipc_error, sizeof(g_ipc_error), "handle and base must be non-NULL");
        return NEOX_ERR_INVALID_ARGUMENT;
    }
    cudaIpcMemHandle_t h;
    memcpy(&h, handle->bytes, sizeof(h));
    void* p = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return ipc_fail("cudaIpcOpenMemHandle", (int)e);
    *base = p;
    return NEOX_OK;
}

neox_status neox_ipc_close(void* base) {
    g_ipc_error[0] = 0;
    if (!base) {
        snprintf(g_ipc_error, sizeof(g_ipc_error), "base must be non-NULL");
        return NEOX_ERR_INVALID_ARGUMENT;
    }
    const cudaError_t e = cudaIpcCloseMemHandle(base);
    if (e != cudaSuccess) return ipc_fail("cudaIpcCloseMemHandle", (int)e);
    return NEOX_OK;
}

}  // extern "C"
