// Reconstruct+attend for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: plugin hooks of inference engines that
// receive no workspace argument, code running while the serving engine has reserved the
// whole HBM for its KV-cache pool, and latency-critical paths where an allocation's
// implicit device synchronisation is not allowed.  This entry point gives them the
// selective / dense reconstruct+attend of xkv_reconstruct_attend with no workspace: the
// split-K partial results live in a fixed array of device memory that is part of the
// library itself.
//
// The array is a file-scope __device__ variable of XKV_NOALLOC_SCRATCH_BYTES (16 MiB).
// Every GPU that loads the library holds it until the process exits.  Host code cannot
// use the variable's name as a device address, so the first call on each device (with
// that device current) asks the runtime for its address once and keeps it.  The kept
// address belongs to the device's current context: a cudaDeviceReset would replace it,
// so the entry point must not be used after one.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "xkv_internal.cuh"

namespace {

constexpr size_t XKV_NOALLOC_SCRATCH_BYTES = (size_t)16 << 20;

// Shared by every call on a device; keeps the previous call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[XKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {nullptr};

}  // namespace

extern "C" xkv_status xkv_reconstruct_attend_noalloc(const xkv_dims *dims, const void *Ak_win,
                                                     const void *Av_win, const void *Bkt_layer,
                                                     const void *Bvt_layer, const void *q,
                                                     const int32_t *sel, int32_t n_sel,
                                                     float *out, void *stream) {
    const char *who = "xkv_reconstruct_attend_noalloc";
    char msg[320];
    // Every argument rule first, on the host, under this entry point's name (and its
    // XKV_FAULT injection); no CUDA call happens before they pass.
    xkv_status st = xkv::attend_validate(who, dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q,
                                         sel, n_sel, nullptr, nullptr, 0, 0, out, nullptr,
                                         XKV_NOALLOC_SCRATCH_BYTES, false, nullptr);
    if (st != XKV_OK) return st;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        snprintf(msg, sizeof msg, "%s: no usable current device (%s)", who,
                 e != cudaSuccess ? cudaGetErrorString(e) : "device index out of range");
        xkv::set_last_error(msg);
        return XKV_ERR_CUDA;
    }
    void *scratch;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p) {
                snprintf(msg, sizeof msg, "%s: cudaGetSymbolAddress of the scratch array: %s",
                         who, cudaGetErrorString(e));
                xkv::set_last_error(msg);
                return XKV_ERR_CUDA;
            }
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    // The partials need no clearing (every one is written before it is read) and the
    // status word is reset by the call's first kernel.
    return xkv::attend_launch(who, dims, Ak_win, Av_win, Bkt_layer, Bvt_layer, q, sel, n_sel,
                              nullptr, nullptr, 0, 0, out, scratch, stream);
}
