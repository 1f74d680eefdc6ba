// moe_forward_noalloc: the MoE forward for callers that cannot allocate device
// memory themselves.
//
// Some callers have no way to call cudaMalloc on the hot path.  A plugin
// inside a serving runtime that owns every device allocation is one.  A
// latency-critical loop that must not call cudaMalloc, because cudaMalloc can
// synchronise the device, is another.  For them the library carries its own
// scratch: a file-scope device array of MOE_NOALLOC_SCRATCH_BYTES that every GPU
// loading the library holds until the process exits.  The entry point runs the
// same kernels as moe_forward with that array as the workspace.
//
// Set-up: the first call on each device looks up the array's device address
// with cudaGetSymbolAddress while that device is current.  The host-side name
// of the array is only a stand-in, not a device address, so it is never passed
// to a kernel.  The address is cached per device.  Make the first call on a
// device before any stream capture, since the set-up call is not a stream
// operation.  The cache is never refreshed: after cudaDeviceReset in the same
// process the cached address is stale, so this entry point must not be used on
// a device that was reset after its first call.
//
// Sharing: every call on a device uses the same array and the array keeps the
// last call's contents.  Everything the kernels need zeroed or initialised per
// call (counters, histograms, tile tables, padding-row markers) is rewritten by
// the dispatch kernels at the start of each call.  Two calls whose kernels
// overlap on the GPU (different streams, or different host threads without
// ordering) race on the array.  Serialise them, e.g. one stream per device.
#include <cuda_runtime.h>

#include <mutex>

#include "moe.h"

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
void *g_scratch_addr[kMaxScratchDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once).
// Only an sm_100 device can load this library's kernels, so any other device is
// refused before the lookup, which would otherwise try to load the module there.
int scratch_on_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
    }
    if (major != 10) return MOE_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            // leave no sticky error behind for the next call's launch check
            cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

bool ok_ptr(const void *p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int moe_forward_noalloc(const void *x, const void *gate_up, const void *down,
                                   const void *sh_gate, const void *sh_up, const void *sh_down,
                                   const int32_t *topk_idx, const float *topk_w, int N, int D,
                                   int E, int d_moe, int d_sh, int k, int dtype, void *y,
                                   void *stream) {
    if (dtype != MOE_F32 && dtype != MOE_BF16) return MOE_ERR_DTYPE;
    const size_t need = moe_forward_workspace(N, D, E, d_moe, d_sh, k, dtype);
    if (need == 0) return MOE_ERR_SHAPE;
    // Sizes whose workspace does not fit the built-in scratch are refused here,
    // before any launch, with the workspace error code.
    if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
    if (N == 0) return MOE_OK;
    // The caller's pointers are checked before the set-up below touches the device.
    const void *ptrs[] = {x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, y};
    for (const void *q : ptrs)
        if (!ok_ptr(q)) return MOE_ERR_ARG;
    void *scratch = nullptr;
    const int rc = scratch_on_current_device(&scratch);
    if (rc != MOE_OK) return rc;
    return moe_forward(x, gate_up, down, sh_gate, sh_up, sh_down, topk_idx, topk_w, N, D, E, d_moe,
                       d_sh, k, dtype, y, scratch, MOE_NOALLOC_SCRATCH_BYTES, stream);
}
