// Dispatch without expand: a consumer reads the received rows through a
// gather index instead of an expanded, expert-contiguous copy -- the
// do_expand=False option of the pages' dispatch (DeepEP issue #760,
// Reproduction) and the VRAM side of the expand tradeoff (DeepEP issue #48,
// answer on the VRAM / performance tradeoff).
//
//  * expand_index_kernel: src[pos[t, j]] = recv_pos[t, rank(e_j)] -- the recv
//    row that serves each expert-contiguous row;
//  * standin_gather_kernel: the deterministic stand-in expert applied to
//    recv[src[p]] instead of expanded[p] (same values, no expanded buffer).
#include <cuda_bf16.h>

#include "epx_internal.cuh"

namespace epx {
namespace {

// rank owning expanded row q: rank r's rows are [bound[r], bound[r + 1])
__device__ __forceinline__ int rank_of_row(const int32_t *bound, int R, int q)
{
    int lo = 0, hi = R - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (bound[mid] <= q)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(256) expand_index_kernel(IndexParams p)
{
    __shared__ int32_t s_bound[EPX_MAX_RANKS + 1];
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    for (int i = threadIdx.x; i <= p.R; i += blockDim.x) s_bound[i] = p.off_e[i * p.epr];
    __syncthreads();
    const long long n = (long long)p.T * p.k;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int q = p.pos[i];
        if (q < 0) continue;
        if ((int64_t)q >= p.rows) {
            atomicOr(p.err, (int)EP_DEVERR_EXP_CAP);
            continue;
        }
        const long long t = i / p.k;
        p.src[q] = p.recv_pos[t * p.R + rank_of_row(s_bound, p.R, q)];
    }
    pdl_launch_dependents();
}

// expert owning expanded row q (largest e with off_e[e] <= q)
__device__ __forceinline__ int expert_of_row(const int32_t *off_e, int E, int q)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off_e[mid] <= q)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(128) standin_gather_kernel(GatherParams p)
{
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    const int64_t n_route = p.totals[0];
    const int64_t rows = n_route < p.rows ? n_route : p.rows;
    for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const int32_t sr = p.src[row];
        if (sr < 0 || (int64_t)sr >= p.recv_rows) {
            if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(p.err, (int)EP_DEVERR_RECV_CAP);
            continue;
        }
        const int e = expert_of_row(p.off_e, p.E, (int)row);
        const float scale = __fadd_rn(1.0f, __fdiv_rn((float)e, (float)p.E));
        const int v0 = blockIdx.x * p.vpc;
        const int v1 = min(p.V, v0 + p.vpc);
        for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            const uint4 q = ld_v4(p.recv + (size_t)sr * p.V + v);
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = __fmul_rn(__uint_as_float(u[i] << 16), scale);
                const float hi = __fmul_rn(__uint_as_float(u[i] & 0xffff0000u), scale);
                __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
                o[i] = *reinterpret_cast<uint32_t *>(&b);
            }
            st_v4(p.y + (size_t)row * p.V + v, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_expand_index(const IndexParams &p, cudaStream_t s)
{
    if (p.T == 0) return cudaSuccess;
    const long long n = (long long)p.T * p.k;
    long long blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    IndexParams q = p;
    q.early_pdl = early_trigger(blocks);
    return launch_pdl(expand_index_kernel, dim3((unsigned)blocks), dim3(256), 0, s, q);
}

cudaError_t launch_standin_gather(const GatherParams &p0, cudaStream_t s)
{
    GatherParams p = p0;
    if (p.rows <= 0) return cudaSuccess;
    const int chunks = (p.V + 255) / 256;
    p.vpc = (p.V + chunks - 1) / chunks;
    const int64_t gy = p.rows < 65535 ? p.rows : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy);
    return launch_pdl(standin_gather_kernel, dim3(chunks, (unsigned)gy), dim3(128), 0, s, p);
}

}  // namespace epx
