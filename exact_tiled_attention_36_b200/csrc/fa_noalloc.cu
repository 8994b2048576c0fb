// fa_noalloc.cu: fa_bwd_noalloc, the backward pass for callers that cannot
// allocate device memory.
//
// fa_bwd needs a caller-owned workspace (the per-row D values and the fp32 dQ
// accumulator). Some callers have no way to provide one: code that runs under
// a host framework which owns every device allocation and forbids raw
// cudaMalloc, latency-critical loops that must not pay for cudaMalloc's
// implicit device-wide synchronisation, or plugins with a fixed memory budget
// decided before they are loaded. For them this file keeps one workspace in a
// file-scope device array of FA_BWD_NOALLOC_MAX_BYTES bytes. Each GPU that
// loads this module holds that memory until the process exits. The kernels
// are the same as fa_bwd's: this entry point only supplies the workspace.
//
// The array lives in its own translation unit, so it forms a module of its
// own. Under CUDA's lazy module loading (the default) a GPU loads that module,
// and reserves the memory, only when fa_bwd_noalloc first runs on it; with
// CUDA_MODULE_LOADING=EAGER every GPU context the process creates loads it.
#include <cuda_runtime.h>

#include <cstddef>

#include "fa.h"
#include "per_device.h"

namespace {

static __device__ __align__(256) unsigned char g_bwd_scratch[FA_BWD_NOALLOC_MAX_BYTES];

// Device address of g_bwd_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
fa_status scratch_on_current_device(void** out) {
    static fa::PerDevice<void*> ptrs;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    const bool ok = ptrs.get(dev, [](void*& p) {
        return cudaGetSymbolAddress(&p, g_bwd_scratch) == cudaSuccess && p != nullptr;
    }, out);
    return ok ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                    const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                                    int Nk, int d, float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
    if (B < 1 || Hq < 1 || Nq < 0) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const size_t need = fa_bwd_workspace_size(B, Hq, Nq, d);
    if (need > static_cast<size_t>(FA_BWD_NOALLOC_MAX_BYTES)) return FA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const fa_status st = scratch_on_current_device(&scratch);
    if (st != FA_OK) return st;
    // fa_bwd's first kernel rewrites every byte of the workspace it reads
    // (D, and the dQ accumulator, which it sets to zero), so what an earlier
    // call left in the array does not matter.
    return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, scratch, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream);
}
