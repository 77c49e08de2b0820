// bra_route_noalloc.cu -- bra_route_noalloc: the routing step (region means, affinity,
// top-k) with its fp32 scratch in a fixed device array instead of memory from the
// library's pool.
//
// Who needs it: callers that cannot allocate device memory when they call us. Some hand
// every byte of HBM to their own allocator at start-up, so a driver allocation would fail
// or fragment their arena. Others run latency-critical loops that must not take the
// allocator's locks or meet an out-of-memory error halfway through a step. bra_route takes
// its scratch from a stream-ordered pool (cudaMallocFromPoolAsync), which those callers
// cannot accept. This entry point never allocates: no cudaMalloc, cudaFree, pool call or
// allocating library routine.
//
// The scratch is g_route_scratch below: kNoAllocScratchBytes (8 MiB) of fp32 space for the
// query and key region means, 2 * B * R * C floats. Every GPU that loads this library
// holds that array until the process exits. Calls that need more are rejected with
// BRA_ERR_UNSUPPORTED before anything runs. One-token regions (R <= 256) need no scratch:
// their means are the tokens, and routing reads q and k directly, as in bra_route. All calls
// on a device share the one array and it keeps the last call's contents; the kernels
// overwrite every element they read, so nothing needs clearing between calls. Two calls
// whose kernels overlap on the GPU (two streams, or two host threads) race on the array:
// order them on one stream.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "bra.h"
#include "bra_launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

// Device-side scratch for the region means. In host code this name is a host-side
// stand-in, not a device address: only the pointer from cudaGetSymbolAddress may be given
// to a kernel.
static __device__ __align__(256) float g_route_scratch[kNoAllocScratchBytes / sizeof(float)];

struct NoAllocDevice {
    std::atomic<bool> ready{false};  // set (release) after scratch and num_sms
    float *scratch = nullptr;  // device address of g_route_scratch on this device
    int num_sms = 0;
};

std::mutex g_noalloc_mutex;
NoAllocDevice g_noalloc_devices[64];

// Once per device, with that device current: the device address of the scratch array and
// the SM count. Neither call allocates.
bra_status noalloc_setup(NoAllocDevice **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        bra::set_last_error(std::string("cudaGetDevice: ") + cudaGetErrorString(e));
        return BRA_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) {
        bra::set_last_error("device ordinal out of range");
        return BRA_ERR_UNSUPPORTED;
    }
    NoAllocDevice &st = g_noalloc_devices[dev];
    if (!st.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        if (!st.ready.load(std::memory_order_relaxed)) {
            float *p = nullptr;
            e = cudaGetSymbolAddress((void **)&p, g_route_scratch);
            if (e != cudaSuccess) {
                bra::set_last_error(std::string("cudaGetSymbolAddress(route scratch): ") + cudaGetErrorString(e));
                return BRA_ERR_CUDA;
            }
            int sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e != cudaSuccess) {
                bra::set_last_error(std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
                return BRA_ERR_CUDA;
            }
            st.scratch = p;
            st.num_sms = sms;
            st.ready.store(true, std::memory_order_release);
        }
    }
    *out = &st;
    return BRA_OK;
}

}  // namespace

extern "C" {

bra_status bra_route_noalloc(const void *q, const void *k, int32_t *idx, int B, int H, int W, int C, int n_win,
                             int topk, bra_dtype dtype, void *stream)
{
    bra::Geometry g;
    bra_status s = bra::check_route_args(q, k, idx, B, H, W, C, n_win, topk, dtype, &g);
    if (s != BRA_OK || B == 0) return s;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (g.rs == 1 && g.R <= 256) {
        // one-token regions: the means are the tokens; the same kernels as bra_route, no scratch
        const cudaError_t e = bra::launch_route_topk_tokens(q, k, idx, g, dtype == BRA_BF16, cs);
        if (e != cudaSuccess) {
            bra::set_last_error(std::string("routing kernel: ") + cudaGetErrorString(e));
            return BRA_ERR_CUDA;
        }
        return BRA_OK;
    }
    const size_t need = (size_t)2 * g.B * g.R * g.C * sizeof(float);
    if (need > kNoAllocScratchBytes) {
        char msg[200];
        std::snprintf(msg, sizeof(msg),
                      "bra_route_noalloc: these sizes need %zu bytes of scratch, more than its fixed %zu bytes "
                      "(2 * B * n_win^2 * C * 4 must not exceed it)",
                      need, kNoAllocScratchBytes);
        bra::set_last_error(msg);
        return BRA_ERR_UNSUPPORTED;
    }
    NoAllocDevice *st = nullptr;
    if ((s = noalloc_setup(&st)) != BRA_OK) return s;
    float *qm = st->scratch;
    float *km = qm + (size_t)g.B * g.R * g.C;
    cudaError_t e = bra::launch_region_means(q, k, qm, km, g, dtype == BRA_BF16, st->num_sms, cs);
    if (e == cudaSuccess) e = bra::launch_route_topk(qm, km, idx, g, cs);
    if (e != cudaSuccess) {
        bra::set_last_error(std::string("routing kernels: ") + cudaGetErrorString(e));
        return BRA_ERR_CUDA;
    }
    return BRA_OK;
}

}  // extern "C"
