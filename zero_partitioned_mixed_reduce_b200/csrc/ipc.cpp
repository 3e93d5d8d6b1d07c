// Device buffers shared between the processes of a multi-GPU job through
// CUDA IPC. A rank exports the allocation that holds one of its buffers (the
// allocation's IPC handle and the buffer's offset in it); every peer opens
// the handle, which maps that allocation into its own address space as a
// plain peer mapping over NVLink. The library's kernels then read peers'
// gradient replicas and parameter shards through those pointers with plain
// loads or 1-D bulk copies. No multicast object is created, and the library
// allocates nothing: the buffers stay the caller's.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "internal.h"

namespace {

using GetAddressRange = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the runtime's driver entry point (the library
// links no driver library).
GetAddressRange address_range() {
    static const GetAddressRange fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            p = nullptr;
        }
        return reinterpret_cast<GetAddressRange>(p);
    }();
    return fn;
}

// Allocations of other processes mapped into this one, by reading device and
// handle: the same allocation may carry several exported buffers, and is
// mapped once per device that reads it.
struct Mapping {
    void* base = nullptr;
    int refs = 0;
};
std::mutex g_mu;
std::map<std::string, Mapping> g_mapped;

std::string key_of(const zero_ipc_handle* h, int device) {
    return std::to_string(device) + ":" +
           std::string(reinterpret_cast<const char*>(h->handle), sizeof h->handle);
}

zero_status ipc_fail(const char* where, cudaError_t e, const char* hint = "") {
    cudaGetLastError();
    return zb_fail(ZERO_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e) + hint);
}

}  // namespace

extern "C" zero_status zero_ipc_export(const void* ptr, zero_ipc_handle* out) {
    return zb_guarded("zero_ipc_export", [&]() -> zero_status {
        if (!ptr || !out) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ipc_export: NULL pointer or output");
        cudaPointerAttributes attr{};
        cudaError_t e = cudaPointerGetAttributes(&attr, ptr);
        if (e != cudaSuccess) return ipc_fail("zero_ipc_export", e);
        if (attr.type != cudaMemoryTypeDevice)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ipc_export: not device memory");
        const GetAddressRange range = address_range();
        if (!range) return zb_fail(ZERO_ERR_CUDA, "zero_ipc_export: the driver's address-range query is unavailable");
        CUdeviceptr base = 0;
        size_t size = 0;
        if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS || base == 0)
            return zb_fail(ZERO_ERR_CUDA, "zero_ipc_export: cannot find the allocation holding the pointer");
        cudaIpcMemHandle_t h;
        e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
        if (e != cudaSuccess)
            return ipc_fail("zero_ipc_export", e,
                            " (the buffer must come from cudaMalloc, not from a virtual-memory pool such as "
                            "an allocator's expandable segments)");
        static_assert(sizeof(h) == sizeof out->handle, "an IPC handle is 64 bytes");
        std::memcpy(out->handle, &h, sizeof h);
        out->offset = static_cast<int64_t>(reinterpret_cast<uintptr_t>(ptr) - static_cast<uintptr_t>(base));
        out->alloc_bytes = static_cast<int64_t>(size);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_ipc_open(const zero_ipc_handle* h, void** out) {
    return zb_guarded("zero_ipc_open", [&]() -> zero_status {
        if (!h || !out) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ipc_open: NULL handle or output");
        if (h->offset < 0 || h->offset >= h->alloc_bytes)
            return zb_fail(ZERO_ERR_RANGE, "zero_ipc_open: offset outside the exported allocation");
        int dev = 0;
        cudaError_t de = cudaGetDevice(&dev);
        if (de != cudaSuccess) return ipc_fail("zero_ipc_open", de);
        const std::string key = key_of(h, dev);
        std::lock_guard<std::mutex> lock(g_mu);
        Mapping& m = g_mapped[key];
        if (m.refs == 0) {
            cudaIpcMemHandle_t ch;
            std::memcpy(&ch, h->handle, sizeof ch);
            void* base = nullptr;
            const cudaError_t e = cudaIpcOpenMemHandle(&base, ch, cudaIpcMemLazyEnablePeerAccess);
            if (e != cudaSuccess) {
                g_mapped.erase(key);
                return ipc_fail("zero_ipc_open", e);
            }
            m.base = base;
        }
        ++m.refs;
        *out = static_cast<char*>(m.base) + h->offset;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_ipc_close(const zero_ipc_handle* h) {
    return zb_guarded("zero_ipc_close", [&]() -> zero_status {
        if (!h) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ipc_close: NULL handle");
        int dev = 0;
        cudaError_t de = cudaGetDevice(&dev);
        if (de != cudaSuccess) {
            cudaGetLastError();
            dev = -1;  // no device: nothing can be open
        }
        std::lock_guard<std::mutex> lock(g_mu);
        auto it = g_mapped.find(key_of(h, dev));
        if (it == g_mapped.end() || it->second.refs <= 0)
            return zb_fail(ZERO_ERR_STATE, "zero_ipc_close: the handle is not open in this process");
        if (--it->second.refs > 0) return ZERO_OK;
        void* base = it->second.base;
        g_mapped.erase(it);
        const cudaError_t e = cudaIpcCloseMemHandle(base);
        if (e != cudaSuccess) return ipc_fail("zero_ipc_close", e);
        return ZERO_OK;
    });
}
