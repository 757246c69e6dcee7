// Allocation-free entry point: atlaskv_attend with its scratch in a static
// device array owned by the library instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: a host program that talks
// to it through the plain C ABI without any device allocator of its own, or a
// serving process whose device memory is entirely pre-partitioned by another
// runtime, or a hot loop where a device allocation (which can synchronise the
// device and take unbounded time) is not allowed.  For them this entry point
// takes the scratch from g_static_scratch below.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "atlaskv.h"
#include "internal.h"

namespace {

// Every GPU that loads this library holds this array until the process exits.
__device__ __align__(256) unsigned char g_static_scratch[ATLASKV_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices];   // device address of g_static_scratch per device, once set up

// Host code cannot use &g_static_scratch (that is a host-side stand-in, not a
// device address); ask the runtime for the device address, once per device,
// with that device current.
atlaskv_status scratch_address(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return akv_report(ATLASKV_ECUDA, "atlaskv_attend_static: no current CUDA device");
    }
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "atlaskv_attend_static: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
            cudaGetLastError();
            return akv_report(ATLASKV_ECUDA, msg);
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return ATLASKV_OK;
}

}  // namespace

extern "C" atlaskv_status atlaskv_attend_static(atlaskv_tree *tree, const atlaskv_params *params,
                                                const atlaskv_io *io, void *stream)
{
    if (!io) return akv_report(ATLASKV_EINVAL, "atlaskv_attend_static: null io");
    size_t need = 0;
    const atlaskv_status st = atlaskv_workspace_size(tree, params, io->B, io->N, io->H, io->T, &need);
    if (st != ATLASKV_OK) return st;
    if (need > (size_t)ATLASKV_STATIC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "atlaskv_attend_static: these sizes need %zu bytes of scratch, above the static maximum of %zu "
                 "bytes; use atlaskv_attend with a workspace",
                 need, (size_t)ATLASKV_STATIC_SCRATCH_BYTES);
        return akv_report(ATLASKV_ENOMEM, msg);
    }
    void *scratch = nullptr;
    const atlaskv_status s2 = scratch_address(&scratch);
    if (s2 != ATLASKV_OK) return s2;
    // Nothing in the scratch has to start at zero: every kernel of the path
    // writes each scratch word it later reads within the same call.
    return atlaskv_attend(tree, params, io, scratch, (size_t)ATLASKV_STATIC_SCRATCH_BYTES, stream);
}
