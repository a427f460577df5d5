// Sharing device buffers between the processes of a multi-GPU job (CUDA IPC),
// for the peer-memory form of the step: each rank reads its owned slice of
// every replica's gradient buffer through peer loads (the reduce-scatter)
// and writes its bf16 results into every rank's parameter buffer through
// peer stores (the all-gather), over NVLink / NVSwitch.
//
// A buffer from a caching allocator is usually a piece of a larger
// allocation, and an IPC handle names a whole allocation, so the exported
// handle carries the buffer's offset inside it.  The allocation's base comes
// from the driver (cuMemGetAddressRange), fetched through the runtime's
// entry-point query so that the library does not link the driver library
// itself (it must load on machines without a GPU driver).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "zr_internal.hpp"

namespace {

using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

AddressRangeFn address_range_fn() {
    static std::once_flag once;
    static AddressRangeFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddressRangeFn>(f);
    });
    return fn;
}

zr_status allocation_of(const void* ptr, uintptr_t* base, size_t* size) {
    AddressRangeFn fn = address_range_fn();
    if (!fn) return ZR_ERR_CUDA;
    CUdeviceptr b = 0;
    size_t s = 0;
    if (fn(&b, &s, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return ZR_ERR_CUDA;
    *base = static_cast<uintptr_t>(b);
    *size = s;
    return ZR_OK;
}

}  // namespace

extern "C" {

zr_status zr_ipc_export(const void* device_ptr, zr_ipc_handle* out) {
    if (!device_ptr || !out) return ZR_ERR_INVALID_ARG;
    uintptr_t base = 0;
    size_t size = 0;
    zr_status st = allocation_of(device_ptr, &base, &size);
    if (st != ZR_OK) return st;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return ZR_ERR_CUDA;
    static_assert(sizeof(h) == sizeof(out->handle), "CUDA IPC handles are 64 bytes");
    std::memcpy(out->handle, &h, sizeof h);
    out->offset = static_cast<uint64_t>(reinterpret_cast<uintptr_t>(device_ptr) - base);
    out->allocation_bytes = static_cast<uint64_t>(size);
    return ZR_OK;
}

zr_status zr_ipc_open(const zr_ipc_handle* h, void** device_ptr) {
    if (!h || !device_ptr || h->offset >= h->allocation_bytes) return ZR_ERR_INVALID_ARG;
    cudaIpcMemHandle_t mh;
    std::memcpy(&mh, h->handle, sizeof mh);
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, mh, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return ZR_ERR_CUDA;
    *device_ptr = static_cast<char*>(base) + h->offset;
    return ZR_OK;
}

zr_status zr_ipc_close(void* device_ptr) {
    if (!device_ptr) return ZR_ERR_INVALID_ARG;
    uintptr_t base = 0;
    size_t size = 0;
    zr_status st = allocation_of(device_ptr, &base, &size);
    if (st != ZR_OK) return st;
    return cudaIpcCloseMemHandle(reinterpret_cast<void*>(base)) == cudaSuccess ? ZR_OK : ZR_ERR_CUDA;
}

}  // extern "C"
