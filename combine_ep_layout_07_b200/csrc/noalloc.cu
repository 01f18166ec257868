// ep_roundtrip_host_noalloc: the host round trip for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the
// point where they need a dispatch/combine pass: code that runs while
// another component owns the device allocator (a caching allocator that
// must not be bypassed, or a memory pool fixed at start-up), plugins loaded
// into a host that forbids allocation after initialisation, or latency
// paths where an allocation's implicit synchronisation is not acceptable.
// For them this entry point runs the same pass as ep_roundtrip_host, with
// its device scratch in a fixed array of EPX_NOALLOC_SCRATCH_BYTES that is
// part of this library's device image: every GPU that loads the library
// holds that array until the process exits.
//
// The scratch is shared by all calls and keeps the last call's contents.
// Nothing in it needs to start at zero: every intermediate the pass reads
// was written earlier in the same call (the routing layout, including its
// error word, is rewritten in full; only the recv / expanded / expert-output
// rows below the counts the layout just produced are read).  Calls whose
// device work overlaps (two streams, or two host threads) race on the
// array; order them on one stream or synchronise between them.
#include <mutex>

#include "epx_internal.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[EPX_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in, so the address is looked up once per device
// with that device current.
ep_status_t scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return EP_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return EP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return EP_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return EP_OK;
}

}  // namespace

extern "C" ep_status_t ep_roundtrip_host_noalloc(const void *x_host, const void *topk_idx_host,
                                                 const float *topk_weights_host, int32_t T,
                                                 int32_t H, int32_t k, int32_t E, int32_t R,
                                                 int32_t idx_bits, void *out_host,
                                                 int32_t *dev_err_host, void *stream)
{
    const size_t need = ep_roundtrip_device_bytes(T, H, k, E, R, idx_bits);
    if (need == 0) return EP_ERR_INVALID_ARG;
    if (need > (size_t)EPX_NOALLOC_SCRATCH_BYTES) return EP_ERR_UNSUPPORTED;
    void *base = nullptr;
    const ep_status_t st = scratch_address(&base);
    if (st != EP_OK) return st;
    return ep_roundtrip_host(x_host, topk_idx_host, topk_weights_host, T, H, k, E, R, idx_bits,
                             base, (size_t)EPX_NOALLOC_SCRATCH_BYTES, out_host, dev_err_host,
                             stream);
}
