// Dispatch over peer memory: every row goes straight from x into the buffer
// of the rank that owns its experts.
//
// The pages' multi-GPU setting: a token is sent once to every rank that
// owns one of its experts, together with its top-k routing (DeepEP issue
// #48, question: token A on rank 0 "dispatched only once" to rank 1 for
// experts M and N), and the receiving rank expands it per local expert.  On
// B200 the ranks of one node share NVLink through NVSwitch, so a GPU can
// store into another GPU's memory directly: this kernel derives each row's
// place in the receiver's buffer from the layout and the rows the receiver
// gets from lower ranks (peers[r].row0), and writes the row and its routing
// there -- placement and transfer in one kernel, no staging buffer and no
// separate all-to-all.  Plain 16-byte stores only (no TMA copy touches
// another GPU's memory); nothing waits on another GPU.
#include <cuda_runtime.h>

#include "epx_internal.cuh"

namespace epx {
namespace {

__device__ __forceinline__ int p2p_rank_of(int e, float inv_epr)
{
    // floor(e / epr), exact for e < 2^22 (see the layout kernels)
    return __float2int_rd(__fmul_rn(__fadd_rn((float)e, 0.5f), inv_epr));
}

// CTA (chunk c, token t): warp 0 lists the destination rows of token t (one
// per rank it reaches), the CTA copies its chunk of x[t] to each, and chunk
// 0's warp 0 writes the routing kept on each destination rank.
template <typename IdxT>
__global__ void __launch_bounds__(128) dispatch_p2p_kernel(const __grid_constant__ P2PDispatchParams p)
{
    __shared__ uint4 *s_dst[EPX_MAX_RANKS];
    __shared__ int s_rank[EPX_MAX_RANKS];
    __shared__ long long s_row[EPX_MAX_RANKS];
    __shared__ int s_n;
    const int lane = threadIdx.x & 31;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    const int v0 = blockIdx.x * p.vpc;
    const int v1 = min(p.V, v0 + p.vpc);
    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
        if (threadIdx.x < 32) {
            const unsigned lt = lanemask_lt();
            unsigned flag = 0;
            int n = 0;
            for (int r0 = 0; r0 < p.R; r0 += 32) {
                const int r = r0 + lane;
                const int q = r < p.R ? p.recv_pos[(size_t)t * p.R + r] : -1;
                long long row = -1;
                if (q >= 0) {
                    row = p.peer[r].row0 + (long long)(q - p.off_r[r]);
                    if (row < 0 || row >= p.peer[r].cap) {
                        flag |= EP_DEVERR_RECV_CAP;
                        row = -1;
                    }
                }
                const bool ok = row >= 0;
                const unsigned m = __ballot_sync(kFull, ok);
                if (ok) {
                    const int slot = n + __popc(m & lt);
                    s_dst[slot] = p.peer[r].rows + (size_t)row * p.V;
                    s_rank[slot] = r;
                    s_row[slot] = row;
                }
                n += __popc(m);
            }
            if (flag) atomicOr(p.err, (int)flag);
            if (lane == 0) s_n = n;
        }
        __syncthreads();
        const int n = s_n;
        if (n > 0) {
            const uint4 *src = p.x + (size_t)t * p.V;
            for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
                const uint4 val = ld_nc_v4(src + v);
                for (int i = 0; i < n; ++i) st_v4(s_dst[i] + v, val);
            }
            if (blockIdx.x == 0 && threadIdx.x < 32) {
                // routing of the row: lane j = slot j; experts on another
                // rank read -1 with weight 0
                int e = -1, re = -1;
                float wj = 0.f;
                if (lane < p.k) {
                    const long long ev = (long long)idx[(size_t)t * p.k + lane];
                    if (ev >= 0 && ev < p.E) {
                        e = (int)ev;
                        re = p2p_rank_of(e, p.inv_epr);
                    }
                    wj = p.w[(size_t)t * p.k + lane];
                }
                for (int i = 0; i < n; ++i) {
                    const int r = s_rank[i];
                    const size_t at = (size_t)s_row[i] * p.k + lane;
                    if (lane < p.k && p.peer[r].meta_idx) p.peer[r].meta_idx[at] = re == r ? e : -1;
                    if (lane < p.k && p.peer[r].meta_w) p.peer[r].meta_w[at] = re == r ? wj : 0.f;
                }
            }
        }
        __syncthreads();
    }
    // rows stored into other GPUs' memory are ordered before whatever this
    // GPU writes next (a collective that tells their owners)
    __threadfence_system();
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_dispatch_p2p(const P2PDispatchParams &p0, cudaStream_t s)
{
    P2PDispatchParams p = p0;
    if (p.T == 0) return cudaSuccess;
    // chunks of a row as in the vector dispatch: ~16 CTAs per SM at small
    // batches, chunks of down to 64 vectors
    const int nsm = current_sm_count();
    int chunks = (16 * nsm + p.T - 1) / p.T;
    const int max_chunks = (p.V + 63) / 64;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    p.vpc = (p.V + chunks - 1) / chunks;
    chunks = (p.V + p.vpc - 1) / p.vpc;
    const int threads = p.vpc < 128 ? ((p.vpc + 31) / 32) * 32 : 128;
    const int gy = p.T < 65535 ? p.T : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy);
    if (p.idx_bits == 64)
        return launch_pdl(dispatch_p2p_kernel<long long>, dim3(chunks, gy), dim3(threads), 0, s, p);
    return launch_pdl(dispatch_p2p_kernel<int>, dim3(chunks, gy), dim3(threads), 0, s, p);
}

}  // namespace epx
