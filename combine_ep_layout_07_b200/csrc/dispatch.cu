// Dispatch + expand: every token with at least one valid route is read from
// x once and written to one `recv` row per destination rank and one
// `expanded` row per valid route.
//
// The pages' structure: a token is received once per destination rank
// together with its top-k indices, and a grouped-GEMM consumer then needs it
// duplicated once per local expert (DeepEP issue #48, question and the
// answers on DeepGEMM and on the VRAM / performance tradeoff).  On one GPU
// both copies are made straight from the single read of x[t].
//
// Two copy engines, same result:
//  * vector: 16-byte loads into registers, then 16-byte stores to every
//    destination row (coalesced: a warp moves 512 contiguous bytes per row);
//  * bulk: the row (or a chunk of it) is staged in shared memory by one TMA
//    bulk load (cp.async.bulk, completion on an mbarrier) and written out by
//    one TMA bulk store per destination row, issued by the warp's lanes in
//    parallel.  Every copy is a plain global<->shared::cta bulk copy of
//    this GPU's own memory, issued by the CTA that uses it.
#include "epx_internal.cuh"

namespace epx {
namespace {

constexpr int kMaxDst = EPX_MAX_TOPK + EPX_MAX_RANKS;

// Warp-collective: compact the destination rows of token t into dst[0..n).
// Expanded rows first (k order; none when p.expanded is null), then recv rows
// (rank order; none when p.recv is null).  Rows beyond a capacity are dropped and flagged.  Returns n
// on every lane.
__device__ __forceinline__ int build_dst_list(const DispatchParams &p, int t,
                                              uint4 **dst)
{
    const int lane = threadIdx.x & 31;
    const unsigned lt = lanemask_lt();
    unsigned flag = 0;
    int n = 0;
    if (p.expanded) {  // null: dispatch only (no expanded copy)
        int q = lane < p.k ? p.pos[(size_t)t * p.k + lane] : -1;
        bool over = q >= 0 && (int64_t)q >= p.exp_cap;
        bool ok = q >= 0 && !over;
        flag |= over ? EP_DEVERR_EXP_CAP : 0u;
        unsigned m = __ballot_sync(kFull, ok);
        if (ok) dst[__popc(m & lt)] = p.expanded + (size_t)q * p.V;
        n = __popc(m);
    }
    // null: expand only (no recv copy)
    for (int r0 = 0; p.recv && r0 < p.R; r0 += 32) {
        const int r = r0 + lane;
        int q = r < p.R ? p.recv_pos[(size_t)t * p.R + r] : -1;
        bool over = q >= 0 && (int64_t)q >= p.recv_cap;
        bool ok = q >= 0 && !over;
        flag |= over ? EP_DEVERR_RECV_CAP : 0u;
        unsigned m = __ballot_sync(kFull, ok);
        if (ok) dst[n + __popc(m & lt)] = p.recv + (size_t)q * p.V;
        n += __popc(m);
    }
    if (flag) atomicOr(p.err, (int)flag);
    __syncwarp();
    return n;
}

// ---------------------------------------------------------------- vector

// Whether token t has a valid route (warp-collective, from topk_idx).
__device__ __forceinline__ bool token_has_route(const DispatchParams &p, int t)
{
    const int lane = threadIdx.x & 31;
    long long e = -1;
    if (lane < p.k)
        e = p.idx_bits == 64 ? static_cast<const long long *>(p.idx)[(size_t)t * p.k + lane]
                             : (long long)static_cast<const int *>(p.idx)[(size_t)t * p.k + lane];
    return __any_sync(kFull, e >= 0 && e < p.E);
}

template <int VPT, bool STREAM>
__global__ void __launch_bounds__(128) dispatch_vec_kernel(DispatchParams p)
{
    __shared__ uint4 *s_dst[kMaxDst];
    __shared__ int s_n;
    __shared__ int s_pre;
    if (p.early_pdl) pdl_launch_dependents();
    // with prefetch, the first token's chunk of x is loaded before the wait
    // (only if the token has a route: rows without one are never read), so
    // its DRAM latency overlaps the layout kernel
    uint4 pre[VPT];
    bool have_pre = false;
    const int v0 = blockIdx.x * p.vpc;
    const int v1 = min(p.V, v0 + p.vpc);
    if (p.prefetch) {
        if (threadIdx.x < 32) {
            const bool ok = token_has_route(p, blockIdx.y);
            if (threadIdx.x == 0) s_pre = ok;
        }
        __syncthreads();
        if (s_pre) {
            const uint4 *src = p.x + (size_t)blockIdx.y * p.V;
#pragma unroll
            for (int u = 0; u < VPT; ++u) {
                const int vv = v0 + threadIdx.x + u * blockDim.x;
                if (vv < v1) pre[u] = ld_nc_v4(src + vv);
            }
            have_pre = true;
        }
    }
    pdl_wait_previous();
    for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
        if (threadIdx.x < 32) {
            int n = build_dst_list(p, t, s_dst);
            if (threadIdx.x == 0) s_n = n;
        }
        __syncthreads();
        const int n = s_n;
        if (n > 0) {
            const uint4 *src = p.x + (size_t)t * p.V;
            for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x * VPT) {
                uint4 val[VPT];
                const bool use_pre = have_pre && t == (int)blockIdx.y && v == v0 + (int)threadIdx.x;
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    const int vv = v + u * blockDim.x;
                    if (vv < v1) val[u] = use_pre ? pre[u] : ld_nc_v4(src + vv);
                }
                for (int i = 0; i < n; ++i) {
                    uint4 *d = s_dst[i];
#pragma unroll
                    for (int u = 0; u < VPT; ++u) {
                        const int vv = v + u * blockDim.x;
                        if (vv < v1) {
                            if (STREAM)
                                st_cs_v4(d + vv, val[u]);
                            else
                                st_v4(d + vv, val[u]);
                        }
                    }
                }
            }
        }
        __syncthreads();
    }
    pdl_launch_dependents();
}

// ------------------------------------------------------------------ bulk

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Warp-collective bounded wait for phase `parity` of the barrier.  Every
// lane polls, and the warp leaves the loop together once every lane has
// seen the phase complete, so all lanes return the same answer after the
// same number of polls; false if `limit` polls ran out.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, unsigned parity, long long limit)
{
    const uint32_t a = smem_addr(bar);
    for (long long i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred P;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, P;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (__all_sync(kFull, done != 0u)) return true;
    }
    return false;
}

__device__ __forceinline__ void bulk_g2s(void *sdst, const void *gsrc, unsigned bytes,
                                         uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(sdst)),
        "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_s2g(void *gdst, const void *ssrc, unsigned bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                 "r"(smem_addr(ssrc)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_and_wait_read()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// try_wait polls; each poll may suspend for a hardware-defined time, so this
// bound is far above any real completion time while still ending.
constexpr long long kWaitLimit = 1ll << 22;

}  // namespace

std::atomic<long long> dispatch_first_wait_limit{-1};

namespace {

// One warp per CTA; the CTA handles chunk blockIdx.x (vpc vectors) of token t.
// With prefetch, the bulk load of the first token's chunk of x is issued
// before the wait (if the token has a route), so that the first wave of
// CTAs reads its rows while the layout kernel runs; the CTA always waits for
// that load before it leaves or reuses the buffer.
__global__ void __launch_bounds__(32) dispatch_bulk_kernel(DispatchParams p)
{
    extern __shared__ __align__(128) uint4 sbuf[];
    __shared__ uint4 *s_dst[kMaxDst];
    __shared__ __align__(8) uint64_t bar;
    const int lane = threadIdx.x;
    if (p.early_pdl) pdl_launch_dependents();
    const int v0 = blockIdx.x * p.vpc;
    const int nv = min(p.V, v0 + p.vpc) - v0;
    if (nv <= 0) return;
    const unsigned bytes = (unsigned)nv * 16u;
    if (lane == 0) mbar_init(&bar, 1);
    __syncwarp();
    bool in_flight = false;  // a load of token blockIdx.y issued before the wait
    if (p.prefetch && token_has_route(p, blockIdx.y)) {
        if (lane == 0) {
            mbar_expect_tx(&bar, bytes);
            bulk_g2s(sbuf, p.x + (size_t)blockIdx.y * p.V + v0, bytes, &bar);
        }
        in_flight = true;
    }
    pdl_wait_previous();
    unsigned phase = 0;
    bool first = true;
    for (int t = blockIdx.y; t < p.T; t += gridDim.y) {
        const int n = build_dst_list(p, t, s_dst);
        if (n == 0 && !in_flight) continue;
        if (!in_flight && lane == 0) {
            mbar_expect_tx(&bar, bytes);
            bulk_g2s(sbuf, p.x + (size_t)t * p.V + v0, bytes, &bar);
        }
        in_flight = false;
        // the first wait of the CTA may take a shorter limit (a test setting;
        // kWaitLimit unless changed)
        const long long limit = first ? p.first_wait_limit : kWaitLimit;
        first = false;
        if (!mbar_wait_warp(&bar, phase, limit)) {
            if (lane == 0) atomicOr(p.err, (int)EP_DEVERR_TIMEOUT);
            // leave only once the copy in flight has landed in shared memory
            // (again a bounded wait)
            mbar_wait_warp(&bar, phase, kWaitLimit);
            return;
        }
        phase ^= 1u;
        if (n == 0) continue;  // prefetched, but every route was dropped
        for (int i = lane; i < n; i += 32) bulk_s2g(s_dst[i] + v0, sbuf, bytes);
        bulk_commit_and_wait_read();  // sbuf and s_dst are reused next token
        __syncwarp();
    }
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_dispatch(const DispatchParams &p0, int variant, cudaStream_t s)
{
    DispatchParams p = p0;
    if (p.T == 0) return cudaSuccess;
    const int nsm = current_sm_count();
    const int gy = p.T < 65535 ? p.T : 65535;
    // automatic: TMA bulk copies for large batches (measured faster at 4096
    // rows of 14 KB), register copies for small ones (fewer fixed costs)
    if (variant == 0) variant = p.T >= 1024 ? 2 : 1;
    if (variant == 2) {
        // chunks so that at least ~2 CTAs per SM exist; chunk <= 32 KB
        int chunks = (2 * nsm + p.T - 1) / p.T;
        const int max_chunks = (p.V + 63) / 64;  // >= 1 KB per chunk
        if (chunks > max_chunks) chunks = max_chunks;
        int vpc = (p.V + chunks - 1) / chunks;
        if (vpc > 2048) vpc = 2048;
        chunks = (p.V + vpc - 1) / vpc;
        p.vpc = vpc;
        const size_t smem = (size_t)vpc * 16;  // <= 32 KB: no opt-in needed
        p.early_pdl = early_trigger((long long)chunks * gy);
        const long long fw = dispatch_first_wait_limit.load(std::memory_order_relaxed);
        p.first_wait_limit = fw < 0 ? kWaitLimit : fw;
        return launch_pdl(dispatch_bulk_kernel, dim3(chunks, gy), dim3(32), smem, s, p);
    }
    // vector engine: up to 128 threads x 2 vectors per pass.  Small batches
    // split the row into chunks of down to 64 vectors (one warp) so that the
    // stores of a few tokens spread over ~16 CTAs per SM rather than a few SMs
    int chunks = (16 * nsm + p.T - 1) / p.T;
    const int max_chunks = (p.V + 63) / 64;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    p.vpc = (p.V + chunks - 1) / chunks;
    chunks = (p.V + p.vpc - 1) / p.vpc;
    int threads = ((p.vpc + 1) / 2 + 31) / 32 * 32;
    if (threads > 128) threads = 128;
    p.early_pdl = early_trigger((long long)chunks * gy, 1024 / threads > 16 ? 16 : 1024 / threads);
    return launch_pdl(dispatch_vec_kernel<2, false>, dim3(chunks, gy), dim3(threads), 0, s, p);
}

}  // namespace epx
