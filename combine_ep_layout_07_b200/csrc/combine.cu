// Combine reduce: out[t] = bf16_rn( sum over valid j, in k order, of
// w[t, j] * expert_out[pos[t, j]] ), accumulated in fp32; +0 rows for tokens
// with no valid route.
//
// The pages: the per-expert outputs of a token are reduced back into one row
// (DeepEP issue #48, answer on the reduction before the combine all2all),
// and the combine epilogue that gives each output token one warp starves the
// GPU when only a handful of tokens exist per rank (DeepEP issue #760, the
// report and its first proposed fix: several warps per output token).
//
// Schedules (same arithmetic, same result):
//  * split: CTA (chunk c, token t) owns vectors [c*vpc, (c+1)*vpc) of row t;
//    each thread keeps all valid routes' 16-byte loads of one vector in
//    flight, then accumulates them in k order.  At low T the host picks many
//    small chunks so the hidden dimension is spread over many SMs.
//  * warp-per-token: one warp walks a whole output row (the DeepEP V2
//    epilogue's schedule), kept as a measured baseline.
#include <cuda_bf16.h>

#include "epx_internal.cuh"

namespace epx {
namespace {

__device__ __forceinline__ void fma8(float (&acc)[8], const uint4 &q, float w)
{
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(u[i] << 16);
        const float hi = __uint_as_float(u[i] & 0xffff0000u);
        acc[2 * i] = fmaf(w, lo, acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, hi, acc[2 * i + 1]);
    }
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8])
{
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        u[i] = *reinterpret_cast<uint32_t *>(&b);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
}

// Warp-collective: compact token t's valid routes (k order) into s_pos /
// s_slot (the route's slot j); returns the count on every lane.  The
// weights are not loaded here: the y loads that follow need only the
// positions, so each thread reads its weights after issuing them, and the
// weights' DRAM latency overlaps theirs.
__device__ __forceinline__ int build_routes(const CombineParams &p, int t, int *s_pos,
                                            int *s_slot)
{
    const int lane = threadIdx.x & 31;
    int q = -1;
    if (lane < p.k) q = p.pos[(size_t)t * p.k + lane];
    const bool over = q >= 0 && (int64_t)q >= p.y_rows;
    const bool ok = q >= 0 && !over;
    if (over) atomicOr(p.err, (int)EP_DEVERR_Y_ROWS);
    const unsigned m = __ballot_sync(kFull, ok);
    if (ok) {
        const int slot = __popc(m & lanemask_lt());
        s_pos[slot] = q;
        s_slot[slot] = lane;
    }
    __syncwarp();
    return __popc(m);
}

// Accumulate vector v of token t's n routes; G loads are kept in flight at
// once, the routes' weights read after them.
template <int G>
__device__ __forceinline__ uint4 reduce_vector(const CombineParams &p, const int *s_pos,
                                               const int *s_slot, int t, int n, int v)
{
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    const float *wt = p.w + (size_t)t * p.k;
    for (int i0 = 0; i0 < n; i0 += G) {
        uint4 q[G];
        float w[G];
#pragma unroll
        for (int u = 0; u < G; ++u)
            if (i0 + u < n) q[u] = ld_v4(p.y + (size_t)s_pos[i0 + u] * p.V + v);
#pragma unroll
        for (int u = 0; u < G; ++u)
            if (i0 + u < n) w[u] = __ldg(wt + s_slot[i0 + u]);
#pragma unroll
        for (int u = 0; u < G; ++u)
            if (i0 + u < n) fma8(acc, q[u], w[u]);
    }
    return pack8(acc);
}

template <int G>
__global__ void __launch_bounds__(128) combine_split_kernel(CombineParams p)
{
    __shared__ int s_pos[EPX_MAX_TOPK];
    __shared__ int s_slot[EPX_MAX_TOPK];
    __shared__ int s_n;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
        if (threadIdx.x < 32) {
            int n = build_routes(p, t, s_pos, s_slot);
            if (threadIdx.x == 0) s_n = n;
        }
        __syncthreads();
        const int n = s_n;
        const int v0 = blockIdx.x * p.vpc;
        const int v1 = min(p.V, v0 + p.vpc);
        for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x)
            st_v4(p.out + (size_t)t * p.V + v, reduce_vector<G>(p, s_pos, s_slot, t, n, v));
        __syncthreads();
    }
    pdl_launch_dependents();
}

template <int G>
__global__ void __launch_bounds__(128) combine_warp_per_token_kernel(CombineParams p)
{
    __shared__ int s_pos[4][EPX_MAX_TOPK];
    __shared__ int s_slot[4][EPX_MAX_TOPK];
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    for (int t = blockIdx.x * 4 + wid; t < p.T; t += gridDim.x * 4) {
        const int n = build_routes(p, t, s_pos[wid], s_slot[wid]);
        for (int v = lane; v < p.V; v += 32)
            st_v4(p.out + (size_t)t * p.V + v,
                  reduce_vector<G>(p, s_pos[wid], s_slot[wid], t, n, v));
        __syncwarp();
    }
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_combine(const CombineParams &p0, int variant, cudaStream_t s)
{
    CombineParams p = p0;
    if (p.T == 0) return cudaSuccess;
    const int nsm = current_sm_count();
    const bool big_k = p.k > 8;
    if (variant == 1) {
        int blocks = (p.T + 3) / 4;
        if (blocks > 65535 * 16) blocks = 65535 * 16;
        p.early_pdl = early_trigger(blocks);
        if (big_k)
            return launch_pdl(combine_warp_per_token_kernel<16>, dim3(blocks), dim3(128), 0, s, p);
        return launch_pdl(combine_warp_per_token_kernel<8>, dim3(blocks), dim3(128), 0, s, p);
    }
    // split: enough CTAs for ~4 per SM, at least 32 vectors per CTA
    int chunks = (4 * nsm + p.T - 1) / p.T;
    const int max_chunks = (p.V + 31) / 32;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    // at large batch still two chunks per row: CTAs half as long give the
    // grid a shorter ragged tail (measured 1.4 us off a 241 us prefill step on
    // two boxes; four or seven chunks per row were no better)
    if (chunks < 2 && p.V >= 256) chunks = 2;
    // when one vector per thread fits in one wave (seven 128-thread CTAs
    // per SM at this kernel's register count), take it: a thread's second
    // vector would wait for its first one's loads
    const int one_each = (p.V + 127) / 128;
    if (chunks < one_each && (long long)p.T * one_each <= 7ll * nsm) chunks = one_each;
    p.vpc = (p.V + chunks - 1) / chunks;
    chunks = (p.V + p.vpc - 1) / p.vpc;
    int threads = p.vpc < 128 ? ((p.vpc + 31) / 32) * 32 : 128;
    const int gy = p.T < 65535 ? p.T : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy, 1024 / threads > 16 ? 16 : 1024 / threads);
    if (big_k)
        return launch_pdl(combine_split_kernel<16>, dim3(chunks, gy), dim3(threads), 0, s, p);
    return launch_pdl(combine_split_kernel<8>, dim3(chunks, gy), dim3(threads), 0, s, p);
}

}  // namespace epx
