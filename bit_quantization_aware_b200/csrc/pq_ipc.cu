// Peer-readable device buffers across processes by CUDA IPC (host code only).
//
// The row-sharded step reads other GPUs' packed codes, scales and gradients
// with plain loads. Its buffers are ordinary device allocations shared by
// CUDA IPC handles: the owner exports the allocation that holds a buffer,
// every other process maps it with cudaIpcOpenMemHandle (peer access enabled
// lazily). These are point-to-point peer mappings: no NVLink multicast
// object is created and nothing is bound to one.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <stdint.h>
#include <string.h>

#include <mutex>

#include "pq.h"

namespace {

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(pq_ipc_handle_t),
              "pq_ipc_handle_t must hold a cudaIpcMemHandle_t");

PFN_cuMemGetAddressRange_v3020 address_range_fn() {
    static PFN_cuMemGetAddressRange_v3020 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(f);
    });
    return fn;
}

}  // namespace

extern "C" {

pq_status_t pq_ipc_export(const void* dev_ptr, pq_ipc_handle_t* handle_out,
                          int64_t* offset_out) {
    if (!dev_ptr || !handle_out || !offset_out) return PQ_ERR_INVALID_ARG;
    auto range = address_range_fn();
    if (!range) return PQ_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
        return PQ_ERR_INVALID_ARG;  // not device memory of this context
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return PQ_ERR_CUDA;
    memcpy(handle_out->bytes, &h, sizeof h);
    *offset_out = static_cast<int64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
    return PQ_OK;
}

pq_status_t pq_ipc_open(const pq_ipc_handle_t* handle, void** base_out) {
    if (!handle || !base_out) return PQ_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle->bytes, sizeof h);
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return PQ_ERR_CUDA;
    *base_out = base;
    return PQ_OK;
}

pq_status_t pq_ipc_close(void* base) {
    if (!base) return PQ_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(base) == cudaSuccess ? PQ_OK : PQ_ERR_CUDA;
}

}  // extern "C"
