// tsa_score_fixed_scratch: Dynamic Token Coverage scoring for callers that cannot
// allocate device memory when they call in.  Examples are an engine whose device
// memory is fully planned up front by its own allocator, or a host thread that must not
// enter the CUDA allocator.  Such callers cannot create the workspace tsa_score needs.
// This entry point gets its scratch from a fixed array that is part of the library's
// device image.  Every GPU that loads the library holds that array until the process
// exits.
//
// The scoring itself is tsa_score's: the same validation, kernels and results, with
// the workspace pointing into the fixed array.
#include <stdio.h>

#include <mutex>

#include "common.cuh"

namespace tsa {

constexpr size_t kFixedScratchBytes = size_t(2) << 20;  // 2 MiB

// The scratch.  In host code this name is only a stand-in for the device array, not a
// device address: host code must use the address from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_score_scratch[kFixedScratchBytes];

tsa_status set_error(tsa_status s, const char *msg);  // defined in api.cu

// Device address of g_score_scratch on `dev`, looked up once per device (with that
// device current) and cached.  Returns nullptr if the lookup fails.  The cached address
// belongs to the device's current primary context: after cudaDeviceReset (or any other
// teardown of that context) it is stale, and tsa_score_fixed_scratch_forget() must be
// called before the next call on that device.
static std::mutex g_mu;
static void *g_addr[64] = {};

static void *scratch_address(int dev) {
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_score_scratch) != cudaSuccess) return nullptr;
        g_addr[dev] = p;
    }
    return g_addr[dev];
}

}  // namespace tsa

using namespace tsa;

extern "C" TSA_API tsa_status tsa_score_fixed_scratch(const tsa_dims *dims, const void *Q,
                                                      const void *K, int32_t q, float scale,
                                                      float *s_h, float *s_l, void *stream) {
    const size_t need = tsa_workspace_size(dims, q);
    if (need == 0)  // invalid dims or q: tsa_score reports which, before any device work
        return tsa_score(dims, Q, K, q, scale, s_h, s_l, nullptr, 0, stream);
    if (need > kFixedScratchBytes) {
        char msg[192];
        snprintf(msg, sizeof msg,
                 "tsa_score_fixed_scratch: these dims need %zu bytes of scratch, more than "
                 "the fixed %zu bytes; use tsa_score with a workspace",
                 need, kFixedScratchBytes);
        return set_error(TSA_ERR_WORKSPACE, msg);
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return set_error(TSA_ERR_CUDA, "tsa_score_fixed_scratch: cudaGetDevice failed");
    void *ws = scratch_address(dev);
    if (!ws)
        return set_error(TSA_ERR_CUDA,
                         "tsa_score_fixed_scratch: cudaGetSymbolAddress of the scratch failed");
    // The scratch keeps the previous call's contents.  The scoring writes every byte of
    // it that it reads before reading it, and the grid barriers in the control block
    // return to their initial state at the end of every launch that completes.  The
    // device error word is sticky: it keeps the first error until
    // tsa_score_fixed_scratch_status reads and clears it (which also resets the barriers
    // a failed launch may have left part-way).
    return tsa_score(dims, Q, K, q, scale, s_h, s_l, ws, kFixedScratchBytes, stream);
}

extern "C" TSA_API tsa_status tsa_score_fixed_scratch_status(void *stream) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return set_error(TSA_ERR_CUDA, "tsa_score_fixed_scratch_status: cudaGetDevice failed");
    void *ws = scratch_address(dev);
    if (!ws)
        return set_error(TSA_ERR_CUDA,
                         "tsa_score_fixed_scratch_status: cudaGetSymbolAddress of the scratch "
                         "failed");
    return tsa_get_device_status(ws, stream);
}

extern "C" TSA_API void tsa_score_fixed_scratch_forget(void) {
    std::lock_guard<std::mutex> lock(g_mu);
    for (void *&a : g_addr) a = nullptr;
}
