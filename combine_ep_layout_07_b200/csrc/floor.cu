// Latency floor of a chain of dependent launches (measurement helper).
//
// The low-batch steps of the path (the regime of DeepEP issue #760's report:
// a handful of tokens per rank) move a few hundred KB, so their time is set
// by fixed costs, not by bandwidth: one launch per kernel, the hand-off from
// each kernel to the next, and at least one DRAM round trip per kernel after
// its predecessor is done.  ep_latency_floor issues that skeleton and nothing
// else -- n launches of a one-warp kernel chained exactly like the path's
// kernels (programmatic dependent launch: each lets the next start launching
// at once and waits for its predecessor before touching global memory), each
// doing one load from global memory after that wait and one store -- so a
// step time can be quoted as a multiple of this floor.
#include "epx_internal.cuh"

namespace epx {
namespace {

struct FloorParams {
    int32_t *buf;
    int i, n;
};

// Kernel i loads buf[64 i] (a line of its own, cold after an L2 flush) and
// stores it, plus one, to buf[64 (n + 1 + i)] (a line no kernel loads).
__global__ void __launch_bounds__(32) latency_floor_kernel(FloorParams p)
{
    pdl_launch_dependents();
    pdl_wait_previous();
    if (threadIdx.x == 0) {
        const int v = *reinterpret_cast<volatile int32_t *>(p.buf + 64 * p.i);
        p.buf[64 * (p.n + 1 + p.i)] = v + 1;
    }
}

}  // namespace
}  // namespace epx

using namespace epx;

extern "C" ep_status_t ep_latency_floor(int32_t *buf, int64_t buf_words, int32_t n_kernels,
                                        void *stream)
{
    if (!buf || n_kernels < 1 || n_kernels > 64) return EP_ERR_INVALID_ARG;
    if (buf_words < 64 * (2 * (int64_t)n_kernels + 2)) return EP_ERR_INVALID_ARG;
    if ((uintptr_t)buf % 16) return EP_ERR_MISALIGNED;
    for (int i = 0; i < n_kernels; ++i) {
        FloorParams p{buf, i, n_kernels};
        if (launch_pdl(latency_floor_kernel, dim3(1), dim3(32), 0,
                       static_cast<cudaStream_t>(stream), p) != cudaSuccess)
            return EP_ERR_CUDA;
    }
    return EP_OK;
}
