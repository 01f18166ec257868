// Two-stage combine: the structure the pages describe for a multi-rank
// system, kept on one GPU.
//
//  * local reduce -- every rank sums, for each token it received, the
//    weighted outputs of its own experts into one partial row per
//    (token, rank), stored in the receive layout (DeepEP issue #48, answer:
//    a reduction kernel runs before the combine all2all).  Exporting these
//    rows is the "skip the epilogue, let the consumer finish" option of
//    DeepEP issue #760 (second proposed fix);
//  * epilogue -- each token's partial rows, in rank order, are summed into
//    its bf16 output (DeepEP issue #760, combine_reduce_epilogue), here with
//    an optional fused residual add (the fusion with a downstream op that the
//    same proposal mentions).
//
// Partials are fp32 (the plain reading) or bf16 (the width a wire transfer
// would use).  Both kernels use the split schedule of the single-stage
// combine: CTA (hidden chunk, token), all loads of a vector in flight.
#include <cuda_bf16.h>

#include <type_traits>

#include "epx_internal.cuh"

namespace epx {
namespace {

constexpr int kNoRank = 127;

__device__ __forceinline__ void fma8(float (&acc)[8], const uint4 &q, float w)
{
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xffff0000u), acc[2 * i + 1]);
    }
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 &q)
{
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(u[i] << 16);
        acc[2 * i + 1] += __uint_as_float(u[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&acc)[8])
{
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        u[i] = *reinterpret_cast<uint32_t *>(&b);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
}

// store 8 partial values of vector v of the partial row starting at `row`
__device__ __forceinline__ void store_partial(int part_bits, char *row, int v,
                                              const float (&acc)[8])
{
    if (part_bits == 32) {
        float4 *dst = reinterpret_cast<float4 *>(row) + (size_t)v * 2;
        dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
        reinterpret_cast<uint4 *>(row)[v] = pack_bf16x8(acc);
    }
}

// Where partial row d goes: this rank's partial buffer, or (peer-memory
// form) the entry whose range holds d; nullptr (flagged) when nowhere.
__device__ __forceinline__ char *partial_row(const LocalParams &p, int64_t d)
{
    const size_t row_bytes = (size_t)p.V * 16 * (p.part_bits == 32 ? 2 : 1);
    return static_cast<char *>(p.partial) + (size_t)d * row_bytes;
}

__device__ __forceinline__ char *partial_row(const LocalP2PParams &p, int64_t d)
{
    const size_t row_bytes = (size_t)p.V * 16 * (p.part_bits == 32 ? 2 : 1);
    for (int s = 0; s < p.n_peer; ++s) {
        const PeerRows &e = p.peer[s];
        if (d >= e.first && d < e.first + e.count) {
            const int64_t q = e.row0 + (d - e.first);
            if (q < 0 || q >= e.cap) break;
            return reinterpret_cast<char *>(e.rows) + (size_t)q * row_bytes;
        }
    }
    atomicOr(p.err, (int)EP_DEVERR_RECV_CAP);
    return nullptr;
}

// Warp 0: token t's valid routes sorted (stably) by rank into s_pos / s_w,
// and its groups -- one per rank reached, in rank order -- as [start, end)
// ranges with their partial row.  Returns the number of groups.
__device__ int build_groups(const LocalParams &p, int t, const int32_t *s_bound, int *s_pos,
                            float *s_w, int *s_rank, int *s_gend, int64_t *s_grow, int *s_n)
{
    const int lane = threadIdx.x & 31;
    int q = -1;
    float w = 0.f;
    if (lane < p.k) {
        q = p.pos[(size_t)t * p.k + lane];
        w = p.w[(size_t)t * p.k + lane];
    }
    const bool over = q >= 0 && (int64_t)q >= p.y_rows;
    if (over) atomicOr(p.err, (int)EP_DEVERR_Y_ROWS);
    const bool ok = q >= 0 && !over;
    // rank of the route: the expanded buffer is rank-contiguous, rank r's
    // rows being [s_bound[r], s_bound[r + 1])
    int r = kNoRank;
    if (ok) {
        int lo = 0, hi = p.R - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_bound[mid] <= q)
                lo = mid;
            else
                hi = mid - 1;
        }
        r = lo;
    }
    // stable position by (rank, slot)
    int slot = 0;
    for (int i = 0; i < 32; ++i) {
        const int ri = __shfl_sync(kFull, r, i);
        slot += (ri < r || (ri == r && i < lane)) ? 1 : 0;
    }
    const int n = __popc(__ballot_sync(kFull, ok));
    if (ok) {
        s_pos[slot] = q;
        s_w[slot] = w;
        s_rank[slot] = r;
    }
    __syncwarp();
    // group ends: the last slot of each rank
    const bool last = lane < n && (lane == n - 1 || s_rank[lane + 1] != s_rank[lane]);
    const unsigned lm = __ballot_sync(kFull, last);
    if (last) {
        const int g = __popc(lm & lanemask_lt());
        s_gend[g] = lane + 1;
        int64_t d = p.recv_pos[(size_t)t * p.R + s_rank[lane]];
        if (d < 0 || d >= p.part_cap) {
            atomicOr(p.err, (int)EP_DEVERR_RECV_CAP);
            d = -1;
        }
        s_grow[g] = d;
    }
    if (lane == 0) *s_n = n;
    __syncwarp();
    return __popc(lm);
}

// P = LocalParams (partial rows in this rank's buffer) or LocalP2PParams
// (each partial row stored at its source rank); the arithmetic is the same.
template <int G, typename P>
__global__ void __launch_bounds__(128) local_reduce_kernel(const __grid_constant__ P p)
{
    __shared__ int32_t s_bound[EPX_MAX_RANKS + 1];
    __shared__ int s_pos[EPX_MAX_TOPK], s_rank[EPX_MAX_TOPK], s_gend[EPX_MAX_TOPK];
    __shared__ float s_w[EPX_MAX_TOPK];
    __shared__ int64_t s_grow[EPX_MAX_TOPK];
    __shared__ char *s_gptr[EPX_MAX_TOPK];
    __shared__ int s_n, s_ng;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    for (int i = threadIdx.x; i <= p.R; i += blockDim.x) s_bound[i] = p.off_e[i * p.epr];
    __syncthreads();
    for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
        if (threadIdx.x < 32) {
            const int ng = build_groups(p, t, s_bound, s_pos, s_w, s_rank, s_gend, s_grow, &s_n);
            for (int g = threadIdx.x; g < ng; g += 32)
                s_gptr[g] = s_grow[g] >= 0 ? partial_row(p, s_grow[g]) : nullptr;
            if (threadIdx.x == 0) s_ng = ng;
        }
        __syncthreads();
        const int n = s_n, ng = s_ng;
        const int v0 = blockIdx.x * p.vpc;
        const int v1 = min(p.V, v0 + p.vpc);
        for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            int g = 0;
            for (int i0 = 0; i0 < n; i0 += G) {
                uint4 q[G];
#pragma unroll
                for (int u = 0; u < G; ++u)
                    if (i0 + u < n) q[u] = ld_v4(p.y + (size_t)s_pos[i0 + u] * p.V + v);
#pragma unroll
                for (int u = 0; u < G; ++u) {
                    const int i = i0 + u;
                    if (i < n) {
                        fma8(acc, q[u], s_w[i]);
                        if (i + 1 == s_gend[g]) {  // last route of this rank
                            if (s_gptr[g]) store_partial(p.part_bits, s_gptr[g], v, acc);
#pragma unroll
                            for (int a = 0; a < 8; ++a) acc[a] = 0.f;
                            ++g;
                        }
                    }
                }
            }
            (void)ng;
        }
        __syncthreads();
    }
    // partial rows stored into other GPUs' memory are ordered before
    // whatever this GPU writes next (a collective that tells their owners)
    if constexpr (std::is_same<P, LocalP2PParams>::value) __threadfence_system();
    pdl_launch_dependents();
}

// Warp 0: token t's partial rows in rank order.  Returns their number.
__device__ int epilogue_rows(const EpilogueParams &p, int t, int64_t *s_row)
{
    const int lane = threadIdx.x & 31;
    const unsigned lt = lanemask_lt();
    int n = 0;
    for (int r0 = 0; r0 < p.R; r0 += 32) {
        const int r = r0 + lane;
        int64_t d = r < p.R ? p.recv_pos[(size_t)t * p.R + r] : -1;
        const bool over = d >= p.part_cap;
        if (over) atomicOr(p.err, (int)EP_DEVERR_RECV_CAP);
        const bool ok = d >= 0 && !over;
        const unsigned m = __ballot_sync(kFull, ok);
        if (ok) s_row[n + __popc(m & lt)] = d;
        n += __popc(m);
    }
    __syncwarp();
    return n;
}

template <int G, int BITS>
__global__ void __launch_bounds__(128) epilogue_kernel(EpilogueParams p)
{
    __shared__ int64_t s_row[EPX_MAX_RANKS];
    __shared__ int s_n;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
        if (threadIdx.x < 32) {
            const int n = epilogue_rows(p, t, s_row);
            if (threadIdx.x == 0) s_n = n;
        }
        __syncthreads();
        const int n = s_n;
        const int v0 = blockIdx.x * p.vpc;
        const int v1 = min(p.V, v0 + p.vpc);
        for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            if (p.residual) add_bf16x8(acc, ld_v4(p.residual + (size_t)t * p.V + v));
            for (int i0 = 0; i0 < n; i0 += G) {
                if (BITS == 32) {
                    float4 q[G][2];
#pragma unroll
                    for (int u = 0; u < G; ++u)
                        if (i0 + u < n) {
                            const float4 *src = reinterpret_cast<const float4 *>(p.partial) +
                                                ((size_t)s_row[i0 + u] * p.V + v) * 2;
                            q[u][0] = src[0];
                            q[u][1] = src[1];
                        }
#pragma unroll
                    for (int u = 0; u < G; ++u)
                        if (i0 + u < n) {
                            acc[0] += q[u][0].x; acc[1] += q[u][0].y;
                            acc[2] += q[u][0].z; acc[3] += q[u][0].w;
                            acc[4] += q[u][1].x; acc[5] += q[u][1].y;
                            acc[6] += q[u][1].z; acc[7] += q[u][1].w;
                        }
                } else {
                    uint4 q[G];
#pragma unroll
                    for (int u = 0; u < G; ++u)
                        if (i0 + u < n)
                            q[u] = ld_v4(reinterpret_cast<const uint4 *>(p.partial) +
                                         (size_t)s_row[i0 + u] * p.V + v);
#pragma unroll
                    for (int u = 0; u < G; ++u)
                        if (i0 + u < n) add_bf16x8(acc, q[u]);
                }
            }
            st_v4(p.out + (size_t)t * p.V + v, pack_bf16x8(acc));
        }
        __syncthreads();
    }
    pdl_launch_dependents();
}

// chunks of a row so that a few tokens still spread over the SMs
void split_rows(int T, int V, int &chunks, int &vpc, int &threads)
{
    const int nsm = current_sm_count();
    chunks = (4 * nsm + T - 1) / T;
    const int max_chunks = (V + 31) / 32;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    vpc = (V + chunks - 1) / chunks;
    chunks = (V + vpc - 1) / vpc;
    threads = vpc < 128 ? ((vpc + 31) / 32) * 32 : 128;
}

}  // namespace

cudaError_t launch_local_reduce(const LocalParams &p0, cudaStream_t s)
{
    LocalParams p = p0;
    if (p.T == 0) return cudaSuccess;
    int chunks, threads;
    split_rows(p.T, p.V, chunks, p.vpc, threads);
    const int gy = p.T < 65535 ? p.T : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy);
    if (p.k > 8)
        return launch_pdl(local_reduce_kernel<16, LocalParams>, dim3(chunks, gy), dim3(threads),
                          0, s, p);
    return launch_pdl(local_reduce_kernel<8, LocalParams>, dim3(chunks, gy), dim3(threads), 0, s,
                      p);
}

cudaError_t launch_local_reduce_p2p(const LocalP2PParams &p0, cudaStream_t s)
{
    LocalP2PParams p = p0;
    if (p.T == 0) return cudaSuccess;
    int chunks, threads;
    split_rows(p.T, p.V, chunks, p.vpc, threads);
    const int gy = p.T < 65535 ? p.T : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy);
    if (p.k > 8)
        return launch_pdl(local_reduce_kernel<16, LocalP2PParams>, dim3(chunks, gy),
                          dim3(threads), 0, s, p);
    return launch_pdl(local_reduce_kernel<8, LocalP2PParams>, dim3(chunks, gy), dim3(threads), 0,
                      s, p);
}

cudaError_t launch_epilogue(const EpilogueParams &p0, cudaStream_t s)
{
    EpilogueParams p = p0;
    if (p.T == 0) return cudaSuccess;
    int chunks, threads;
    split_rows(p.T, p.V, chunks, p.vpc, threads);
    const int gy = p.T < 65535 ? p.T : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy);
    if (p.part_bits == 32)
        return launch_pdl(epilogue_kernel<4, 32>, dim3(chunks, gy), dim3(threads), 0, s, p);
    return launch_pdl(epilogue_kernel<8, 16>, dim3(chunks, gy), dim3(threads), 0, s, p);
}

}  // namespace epx
