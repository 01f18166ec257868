// Routing that travels with every received row of a multi-GPU dispatch.
//
// In expert parallelism across GPUs a token is sent once to every rank that
// owns one of its experts, together with its top-k routing, and the rank
// duplicates it once per local expert (DeepEP issue #48, question: token A
// on rank 0 "dispatched only once" to rank 1 for experts M and N).  The
// receiving rank needs, per received row, which of its own experts the row
// goes to and with which gate weight -- for the expand there and for the
// local reduce before the combine travels back (issue #48, answer on the
// reduction before the combine all2all).  This kernel writes that per
// (token, rank) pair, in the send order of the layout (row recv_pos[t, r]):
// the token's k routes with every expert that is not on rank r replaced by
// -1 and its weight by 0.
#include "epx_internal.cuh"

namespace epx {
namespace {

__device__ __forceinline__ int meta_rank_of(int e, float inv_epr)
{
    // floor(e / epr), exact for e < 2^22 (see the layout kernels)
    return __float2int_rd(__fmul_rn(__fadd_rn((float)e, 0.5f), inv_epr));
}

// One warp per token, lane j = top-k slot j.
template <typename IdxT>
__global__ void __launch_bounds__(128) route_meta_kernel(MetaParams p)
{
    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < p.T; t += gridDim.x * warps) {
        int e = -1, r = -1;
        float wj = 0.f;
        if (lane < p.k) {
            const long long ev = (long long)idx[(size_t)t * p.k + lane];
            if (ev >= 0 && ev < p.E) {
                e = (int)ev;
                r = meta_rank_of(e, p.inv_epr);
            }
            wj = p.w[(size_t)t * p.k + lane];
        }
        for (int r0 = 0; r0 < p.R; r0 += 32) {
            const int q = r0 + lane < p.R ? p.recv_pos[(size_t)t * p.R + r0 + lane] : -1;
            unsigned m = __ballot_sync(kFull, q >= 0);
            while (m) {
                const int src = __ffs(m) - 1;
                m &= m - 1u;
                const int row = __shfl_sync(kFull, q, src);
                if ((int64_t)row >= p.rows) {
                    if (lane == 0) atomicOr(p.err, (int)EP_DEVERR_RECV_CAP);
                    continue;
                }
                if (lane < p.k) {
                    const bool mine = r == r0 + src;
                    p.meta_idx[(size_t)row * p.k + lane] = mine ? e : -1;
                    p.meta_w[(size_t)row * p.k + lane] = mine ? wj : 0.f;
                }
            }
        }
    }
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_route_meta(const MetaParams &p0, int idx_bits, cudaStream_t s)
{
    MetaParams p = p0;
    if (p.T == 0) return cudaSuccess;
    long long blocks = ((long long)p.T + 3) / 4;
    if (blocks > 65535LL * 16) blocks = 65535LL * 16;
    p.early_pdl = early_trigger(blocks);
    if (idx_bits == 64)
        return launch_pdl(route_meta_kernel<long long>, dim3((unsigned)blocks), dim3(128), 0, s, p);
    return launch_pdl(route_meta_kernel<int>, dim3((unsigned)blocks), dim3(128), 0, s, p);
}

}  // namespace epx
