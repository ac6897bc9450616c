// ep_ipc.cu -- CUDA IPC mapping of another process's device buffers, for the
// rank tables of the expert-parallel entry points.
//
// The pages' dispatch is an all-to-all that sends each token's rows to the
// GPU holding its experts, and combine is the reverse exchange ("DeepEP是什麼？
// MoE Dispatch、Combine、All-to-all與V2架構", section MoE為什麼需要All-to-all).
// Here every rank's receive (and expert-output) buffer lives in its own
// process; ep_dispatch_ranks / ep_combine_ranks store and load the rows
// through a table of the ranks' buffers.  These three calls put another
// process's buffer into that table: the owner exports an IPC handle of the
// allocation holding the buffer plus the buffer's offset in it, the handles
// travel to the other ranks (over the process group, outside this library),
// and each rank opens its peers' handles.  On one GPU the mapping is
// another process's memory on the same device; on several GPUs it is peer
// memory reached over NVLink (plain loads and stores in the kernels).
//
// The allocation base comes from the driver's address-range query, reached
// through cudaGetDriverEntryPoint, so the library links no driver library.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "ep_internal.cuh"

static_assert(sizeof(cudaIpcMemHandle_t) == EP_IPC_HANDLE_BYTES, "IPC handle size");

namespace ep {
namespace {

typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

// The driver's cuMemGetAddressRange, looked up once.
AddressRangeFn address_range()
{
    static std::once_flag once;
    static AddressRangeFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddressRangeFn>(p);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

}  // namespace
}  // namespace ep

extern "C" {

ep_status_t ep_ipc_export(const void* ptr, void* handle, uint64_t* offset)
{
    if (!ptr || !handle || !offset)
        return EP_ERR_INVALID_ARG;
    ep::AddressRangeFn fn = ep::address_range();
    if (!fn)
        return ep::fail_message(EP_ERR_CUDA, "ep_ipc_export: the driver has no address-range query");
    CUdeviceptr base = 0;
    size_t size = 0;
    if (fn(&base, &size, (CUdeviceptr)(uintptr_t)ptr) != CUDA_SUCCESS)
        return ep::fail_message(EP_ERR_INVALID_ARG,
                                "ep_ipc_export: the pointer is not in a device allocation");
    cudaIpcMemHandle_t h;
    const cudaError_t rc = cudaIpcGetMemHandle(&h, (void*)(uintptr_t)base);
    if (rc != cudaSuccess)
        return ep::cuda_fail(rc, "ep_ipc_export");
    memcpy(handle, &h, sizeof h);
    *offset = (uint64_t)((uintptr_t)ptr - (uintptr_t)base);
    return EP_OK;
}

ep_status_t ep_ipc_open(const void* handle, uint64_t offset, void** base, void** ptr)
{
    if (!handle || !base || !ptr)
        return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof h);
    void* b = nullptr;
    const cudaError_t rc = cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess);
    if (rc != cudaSuccess)
        return ep::cuda_fail(rc, "ep_ipc_open");
    *base = b;
    *ptr = static_cast<char*>(b) + offset;
    return EP_OK;
}

ep_status_t ep_ipc_close(void* base)
{
    if (!base)
        return EP_ERR_INVALID_ARG;
    const cudaError_t rc = cudaIpcCloseMemHandle(base);
    return rc == cudaSuccess ? EP_OK : ep::cuda_fail(rc, "ep_ipc_close");
}

}  // extern "C"
