// Host-side identity of the CUDA context current on the calling thread.
//
// Anything the library caches per device (a kernel's shared-memory attribute, a
// module variable's device address) belongs to a context, not to a device
// ordinal: after cudaDeviceReset the primary context is rebuilt, with a new
// context id, and the cached state must be set up again.  The CUDA driver entry
// points are looked up through the CUDA runtime, so the library needs no link
// against libcuda.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

struct CtxKey {
    int dev = -1;
    unsigned long long id = 0;  // the driver's process-unique context id; 0 = none current
    bool operator==(const CtxKey& o) const { return dev == o.dev && id == o.id; }
};

template <typename Fn>
inline Fn driver_entry_point(const char* name)
{
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// Device ordinal and context id of the current context.  Returns false if no
// context is current yet (any runtime call that needs the device creates it) or
// the driver does not provide context ids.
inline bool current_ctx(CtxKey* key)
{
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static const GetCurrentFn get_current = driver_entry_point<GetCurrentFn>("cuCtxGetCurrent");
    static const GetIdFn get_id = driver_entry_point<GetIdFn>("cuCtxGetId");
    if (!get_current || !get_id) return false;
    if (cudaGetDevice(&key->dev) != cudaSuccess) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, &key->id) == CUDA_SUCCESS && key->id != 0;
}

} // namespace fa
