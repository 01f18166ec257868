// Routing layout: per-expert / per-rank counts, exclusive scans and the
// deterministic row of every route and every (token, rank) pair.
//
// What is computed follows the pages' dispatch API: the layout ("handle")
// that dispatch derives from topk_idx and combine consumes again (DeepEP
// issue #48, question; DeepEP issue #760, Reproduction: dispatch returns
// handle, combine takes it), with -1 as a padding route (issue #760,
// Reproduction: padding rows of -1) and experts on ranks in contiguous
// blocks of E/R (issue #760, Reproduction: local_experts).
//
// A route's row is off_e[e] + (routes to e from earlier tokens) + (earlier
// slots of its own token with the same expert); a (token, rank) pair's row
// is off_r[r] + (earlier tokens that reach r).  Both middle terms are column
// prefix sums of a token x expert (and token x rank) count matrix, so they
// are computed here without any ordering primitive:
//  * one launch of one CTA, or of one thread-block cluster of up to 16 CTAs
//    of 1024 threads; CTA c owns a contiguous range of tokens;
//  * build: one thread per token loads its k indices, validates them,
//    computes each route's rank, marks the first route of every
//    (token, rank) pair and counts the token's row of the count matrix in
//    shared memory -- counts are packed two 16-bit columns per 32-bit word,
//    and the count seen before incrementing is the route's rank among equal
//    experts of its own token;
//  * column scan: every column of the matrix is prefix-summed over the
//    tokens, several threads per column combined with warp shuffles (packed
//    16-bit halves add independently); the column sums are the CTA totals;
//  * cluster exchange: each CTA pushes its totals into every peer's shared
//    memory (distributed shared memory stores); after one cluster barrier
//    every CTA reads them locally; a single CTA skips this;
//  * global scan: one block-wide scan of packed 64-bit (expert, rank) counts
//    gives both exclusive scans at once, plus this CTA's base;
//  * positions: one thread per token again, reading its prefixes back.
// When a CTA's tokens do not fit in shared memory at once, it counts all of
// them first (atomics into its totals) and then builds, scans and places the
// tokens chunk by chunk with a running cursor per column.
#include <cooperative_groups.h>

#include "epx_internal.cuh"

namespace cg = cooperative_groups;

namespace epx {
namespace {

constexpr int kScanInts = 2 * 34;  // 64-bit block-scan scratch
constexpr int kMaxPer = EPX_MAX_EXPERTS / 1024;

// route code in shared memory: -1 = no route (or a dropped bad index), else
// expert | rank << 12 | (rank among equal experts of the token) << 18 |
// (first route of its rank) << 23
__device__ __forceinline__ int code_e(int c) { return c & 0xfff; }
__device__ __forceinline__ int code_r(int c) { return (c >> 12) & 0x3f; }
__device__ __forceinline__ int code_dup(int c) { return (c >> 18) & 0x1f; }
__device__ __forceinline__ bool code_first(int c) { return (c >> 23) & 1; }

__device__ unsigned long long block_exclusive_scan64(unsigned long long v,
                                                     unsigned long long *sm,
                                                     unsigned long long *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
    unsigned long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long n = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) sm[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        const unsigned long long s = lane < nw ? sm[lane] : 0ull;
        unsigned long long si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long n = __shfl_up_sync(kFull, si, o);
            if (lane >= o) si += n;
        }
        if (lane < nw) sm[lane] = si - s;
        if (lane == 31) sm[32] = si;
    }
    __syncthreads();
    *total = sm[32];
    return sm[wid] + inc - v;
}

__device__ __forceinline__ int rank_of(int e, float inv_epr)
{
    // exact for e < 2^22: (e + 1/2) / epr is at least 1/(2 epr) away from an
    // integer, far more than the two fp32 roundings can move it
    return __float2int_rd(__fmul_rn(__fadd_rn((float)e, 0.5f), inv_epr));
}

// Thread-per-token pass over tokens [t0, t0 + n).  With M != nullptr it
// builds the count-matrix rows (zeroed beforehand) and the route codes; with
// tot != nullptr it counts into the CTA totals with atomics instead.  Returns
// the number of this thread's tokens with a valid route; *bad is set if an
// index < -1 or >= E was seen.
template <typename IdxT>
__device__ int build_tokens(const LayoutParams &p, const IdxT *__restrict__ idx, int t0, int n,
                            uint32_t *M, int32_t *codes, int32_t *tot, bool *bad)
{
    const int k = p.k, E = p.E;
    int nreal = 0;
    for (int u = threadIdx.x; u < n; u += blockDim.x) {
        const IdxT *row = idx + (size_t)(t0 + u) * k;
        uint32_t *mrow = M ? M + (size_t)u * p.wds : nullptr;
        unsigned long long mask = 0ull;
        for (int j0 = 0; j0 < k; j0 += 8) {
            long long ev[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) ev[q] = j0 + q < k ? (long long)row[j0 + q] : -1;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int j = j0 + q;
                if (j >= k) break;
                const long long e = ev[q];
                *bad |= (e < -1 || e >= E);
                int code = -1;
                if (e >= 0 && e < E) {
                    const int ei = (int)e;
                    const int r = rank_of(ei, p.inv_epr);
                    const bool first = !((mask >> r) & 1ull);
                    mask |= 1ull << r;
                    if (mrow) {
                        const int sh = (ei & 1) * 16;
                        const uint32_t w = mrow[ei >> 1];
                        const int dup = (int)((w >> sh) & 0xffffu);
                        mrow[ei >> 1] = w + (1u << sh);
                        if (first) mrow[p.wde + (r >> 1)] += 1u << ((r & 1) * 16);
                        code = ei | (r << 12) | (dup << 18) | ((int)first << 23);
                    } else {
                        atomicAdd(&tot[ei], 1);
                        if (first) atomicAdd(&tot[E + r], 1);
                    }
                }
                if (codes) codes[(size_t)u * k + j] = code;
            }
        }
        nreal += mask != 0ull;
    }
    return nreal;
}

// Exclusive prefix of every column of M (n rows, wde + wdr packed columns)
// over its rows.  Lanes take consecutive columns (conflict-free shared
// memory), warps take row segments: pass 1 sums each segment, pass 2 turns
// the segment into an exclusive prefix starting from the sum of the segments
// above it.  seg has max(1024, wde + wdr) words.  The column sums go to
// csum[E + R] (experts first, then ranks).
__device__ void column_scan(const LayoutParams &p, uint32_t *M, int n, uint32_t *seg,
                            int32_t *csum)
{
    const int wdt = p.wde + p.wdr;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int ncb = (wdt + 31) >> 5;                     // 32-column blocks
    const int nsg = ncb >= nwarps ? 1 : nwarps / ncb;    // row segments per block
    const int rps = (n + nsg - 1) / nsg;
    // pass 1: segment sums
    for (int job = wid; job < ncb * nsg; job += nwarps) {
        const int cb = job / nsg, sg = job - cb * nsg;
        const int c = cb * 32 + lane;
        const int ra = min(n, sg * rps), rb = min(n, ra + rps);
        uint32_t sum = 0;
        if (c < wdt)
            for (int r = ra; r < rb; ++r) sum += M[(size_t)r * p.wds + c];
        if (c < wdt) seg[sg * wdt + c] = sum;
    }
    __syncthreads();
    // pass 2: prefixes
    for (int job = wid; job < ncb * nsg; job += nwarps) {
        const int cb = job / nsg, sg = job - cb * nsg;
        const int c = cb * 32 + lane;
        if (c >= wdt) continue;
        const int ra = min(n, sg * rps), rb = min(n, ra + rps);
        uint32_t run = 0, total = 0;
        for (int q = 0; q < nsg; ++q) {
            const uint32_t v = seg[q * wdt + c];
            run += q < sg ? v : 0u;
            total += v;
        }
        for (int r = ra; r < rb; ++r) {
            const uint32_t v = M[(size_t)r * p.wds + c];
            M[(size_t)r * p.wds + c] = run;
            run += v;
        }
        if (sg == 0) {
            const bool er = c < p.wde;
            const int col0 = er ? 2 * c : 2 * (c - p.wde);
            const int lim = er ? p.E : p.R;
            int32_t *dst = er ? csum : csum + p.E;
            dst[col0] = (int32_t)(total & 0xffffu);
            if (col0 + 1 < lim) dst[col0 + 1] = (int32_t)(total >> 16);
        }
    }
}

// Write pos and recv_pos of tokens [t0, t0 + n) from the scanned matrix,
// the route codes, the chunk's column sums and the per-column bases; one
// thread per route, then one per (token, rank), so stores are coalesced.
__device__ __forceinline__ int div_small(int i, float inv)
{
    // floor(i / d) for i < 2^22 with inv = 1/d (same argument as rank_of)
    return __float2int_rd(__fmul_rn(__fadd_rn((float)i, 0.5f), inv));
}

__device__ void place_tokens(const LayoutParams &p, int t0, int n, const uint32_t *M,
                             const int32_t *codes, const int32_t *csum, const int32_t *base)
{
    const int k = p.k, E = p.E, R = p.R;
    const float inv_k = 1.0f / (float)k, inv_r = 1.0f / (float)R;
    for (int i = threadIdx.x; i < n * k; i += blockDim.x) {
        const int u = div_small(i, inv_k);
        const int c = codes[i];
        int v = -1;
        if (c >= 0) {
            const int e = code_e(c);
            v = base[e] + (int)((M[(size_t)u * p.wds + (e >> 1)] >> ((e & 1) * 16)) & 0xffffu) +
                code_dup(c);
        }
        p.pos[(size_t)t0 * k + i] = v;
    }
    for (int i = threadIdx.x; i < n * R; i += blockDim.x) {
        const int u = div_small(i, inv_r);
        const int r = i - u * R;
        const int col = p.wde + (r >> 1), sh = (r & 1) * 16;
        const int here = (int)((M[(size_t)u * p.wds + col] >> sh) & 0xffffu);
        const int next = u + 1 < n ? (int)((M[(size_t)(u + 1) * p.wds + col] >> sh) & 0xffffu)
                                   : csum[E + r];
        p.recv_pos[(size_t)t0 * R + i] = next > here ? base[E + r] + here : -1;
    }
}

__device__ void zero_words(uint32_t *a, int n)
{
    // a is 16-byte aligned; vector stores for the bulk, scalars for the tail
    uint4 *a4 = reinterpret_cast<uint4 *>(a);
    const int n4 = n >> 2;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) a4[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = (n4 << 2) + threadIdx.x; i < n; i += blockDim.x) a[i] = 0u;
}

template <typename IdxT, bool CLUSTER>
__global__ void __launch_bounds__(1024, 1) layout_kernel(LayoutParams p)
{
    extern __shared__ __align__(16) int32_t smem[];
    const int tid = threadIdx.x;
    const int E = p.E, R = p.R, T = p.T;

    int crank = 0, csize = 1;
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        crank = (int)cluster.block_rank();
        csize = (int)cluster.num_blocks();
        // every CTA must be running before a peer writes into its shared
        // memory: arrive now, wait just before the first remote store
        asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    }

    const int W = E + R + 2;  // one CTA's published totals: experts, ranks, bad, real
    unsigned long long *scan = reinterpret_cast<unsigned long long *>(smem);
    uint32_t *M = reinterpret_cast<uint32_t *>(smem + kScanInts);  // [tch][wds]
    const size_t m_words = ((size_t)p.tch * p.wds + 3) & ~(size_t)3;
    int32_t *codes = smem + kScanInts + m_words;   // [tch][k]
    uint32_t *seg = reinterpret_cast<uint32_t *>(codes + (size_t)p.tch * p.k);  // column-scan sums
    int32_t *tot = reinterpret_cast<int32_t *>(seg) + p.seg_words;  // [E + R] totals / chunk sums
    int32_t *base = tot + E + R;                   // [E + R] this CTA's row bases
    int32_t *all_tot = base + E + R;               // [csize][W]
    int32_t *misc = all_tot + csize * W;           // [2] bad flag, real tokens

    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    const int c0 = min(T, crank * p.tpc);
    const int nt = min(T, c0 + p.tpc) - c0;
    const int nchunks = (nt + p.tch - 1) / p.tch;
    bool bad = false;
    int nreal = 0;

    if (tid < 2) misc[tid] = 0;
    if (nchunks <= 1) {
        zero_words(M, p.tch * p.wds);
        __syncthreads();
        nreal = build_tokens(p, idx, c0, nt, M, codes, nullptr, &bad);
        __syncthreads();
        column_scan(p, M, nt, seg, tot);
    } else {
        for (int i = tid; i < E + R; i += blockDim.x) tot[i] = 0;
        __syncthreads();
        nreal = build_tokens(p, idx, c0, nt, nullptr, nullptr, tot, &bad);
    }
    if (__any_sync(kFull, bad) && (tid & 31) == 0) atomicOr(&misc[0], 1);
    if (nreal) atomicAdd(&misc[1], nreal);
    __syncthreads();

    // ---- publish this CTA's totals (to every CTA of the cluster)
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
        for (int i = tid; i < E + R + 2; i += blockDim.x) {
            const int v = i < E + R ? tot[i] : misc[i - E - R];
            for (int c = 0; c < csize; ++c) cluster.map_shared_rank(all_tot, c)[crank * W + i] = v;
        }
        cluster.sync();
    } else {
        for (int i = tid; i < E + R + 2; i += blockDim.x)
            all_tot[i] = i < E + R ? tot[i] : misc[i - E - R];
        __syncthreads();
    }

    // ---- global exclusive scans (one packed 64-bit block scan) and bases
    {
        const int per = (E + (int)blockDim.x - 1) / (int)blockDim.x;
        int glob[kMaxPer], cbase[kMaxPer];
        unsigned int contrib_e = 0;
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            glob[q] = 0;
            cbase[q] = 0;
            const int e = tid * per + q;
            if (q < per && e < E) {
                for (int c = 0; c < csize; ++c) {
                    const int v = all_tot[c * W + e];
                    cbase[q] += c < crank ? v : 0;
                    glob[q] += v;
                }
                contrib_e += glob[q];
            }
        }
        int glob_r = 0, cbase_r = 0;
        if (tid < R)
            for (int c = 0; c < csize; ++c) {
                const int v = all_tot[c * W + E + tid];
                cbase_r += c < crank ? v : 0;
                glob_r += v;
            }
        const unsigned long long v = ((unsigned long long)contrib_e << 32) | (unsigned)glob_r;
        unsigned long long total;
        const unsigned long long ex = block_exclusive_scan64(v, scan, &total);
        unsigned int run = (unsigned int)(ex >> 32);
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            const int e = tid * per + q;
            if (q < per && e < E) {
                base[e] = (int)run + cbase[q];
                if (crank == 0) {
                    p.cnt_e[e] = glob[q];
                    p.off_e[e] = (int)run;
                }
                run += glob[q];
            }
        }
        if (tid < R) {
            const int off_r = (int)(unsigned int)(ex & 0xffffffffull);
            base[E + tid] = off_r + cbase_r;
            if (crank == 0) {
                p.cnt_r[tid] = glob_r;
                p.off_r[tid] = off_r;
            }
        }
        if (tid == 0 && crank == 0) {
            int errc = 0, nr = 0;
            for (int c = 0; c < csize; ++c) {
                errc |= all_tot[c * W + E + R];
                nr += all_tot[c * W + E + R + 1];
            }
            const int n_route = (int)(total >> 32);
            const int n_recv = (int)(total & 0xffffffffull);
            p.off_e[E] = n_route;
            p.off_r[R] = n_recv;
            p.totals[0] = n_route;
            p.totals[1] = n_recv;
            p.totals[2] = nr;
            p.totals[3] = errc ? (int32_t)EP_DEVERR_BAD_INDEX : 0;
        }
    }
    __syncthreads();

    // ---- positions
    if (nchunks <= 1) {
        place_tokens(p, c0, nt, M, codes, tot, base);
        return;
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = c0 + ch * p.tch;
        const int n = min(p.tch, c0 + nt - t0);
        zero_words(M, p.tch * p.wds);
        __syncthreads();
        bool b2 = false;
        build_tokens(p, idx, t0, n, M, codes, nullptr, &b2);
        __syncthreads();
        column_scan(p, M, n, seg, tot);  // tot <- this chunk's column sums
        __syncthreads();
        place_tokens(p, t0, n, M, codes, tot, base);
        __syncthreads();
        for (int i = tid; i < E + R; i += blockDim.x) base[i] += tot[i];
        __syncthreads();
    }
}

// ------------------------------------------------------------------- host

struct Geometry {
    int csize, tpc, tch, wde, wdr, wds, seg_words;
    size_t smem;
};

size_t fixed_smem_ints(int E, int R, int csize)
{
    return (size_t)kScanInts + 2 * (size_t)(E + R) + (size_t)csize * (E + R + 2) + 2;
}

// Cluster size, chunking and column-scan mapping for a layout problem.
Geometry plan(int T, int k, int E, int R, int csize)
{
    Geometry g;
    g.wde = (E + 1) / 2;
    g.wdr = (R + 1) / 2;
    g.wds = (g.wde + g.wdr) | 1;
    // the exchange area grows with the cluster: shrink the cluster if the
    // fixed part would crowd out the count matrix
    while (csize > 1 && fixed_smem_ints(E, R, csize) * 4 + (size_t)(g.wds + 4 + k) * 4 * 16 >
                            (size_t)kMaxDynSmem)
        csize >>= 1;
    g.csize = csize;
    g.tpc = (T + csize - 1) / csize;
    const int wdt_all = g.wde + g.wdr;
    const size_t fixed = (fixed_smem_ints(E, R, csize) + (wdt_all > 1024 ? wdt_all : 1024)) * 4;
    const size_t per_tok = (size_t)(g.wds + k) * 4;
    long long cap = ((long long)kMaxDynSmem - (long long)fixed - 16) / (long long)per_tok;
    if (cap > 1024) cap = 1024;             // one token per thread
    if (cap > 65535 / k) cap = 65535 / k;   // 16-bit column counts cannot overflow
    if (cap < 1) cap = 1;
    g.tch = g.tpc < cap ? (g.tpc < 1 ? 1 : g.tpc) : (int)cap;
    const size_t m_words = ((size_t)g.tch * g.wds + 3) & ~(size_t)3;
    g.seg_words = wdt_all > 1024 ? wdt_all : 1024;
    g.smem = (m_words + (size_t)g.tch * k) * 4 + fixed;  // fixed: scan scratch, seg sums, totals
    return g;
}

template <typename IdxT>
int max_clusters(int csize, size_t smem, int dev)
{
    struct Entry {
        int dev, csize;
        size_t smem;
        int result;
    };
    static Entry cache[64];
    static int n_cache = 0;
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].dev == dev && cache[i].csize == csize && cache[i].smem == smem)
            return cache[i].result;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize, 1, 1);
    cfg.blockDim = dim3(1024, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, layout_kernel<IdxT, true>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (n_cache < 64) cache[n_cache++] = Entry{dev, csize, smem, n};
    return n;
}

template <typename IdxT>
cudaError_t set_attributes_once(int dev)
{
    static unsigned done = 0;  // per device (up to 32)
    if (dev < 32 && (done & (1u << dev))) return cudaSuccess;
    cudaError_t err = cudaFuncSetAttribute(layout_kernel<IdxT, false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kMaxDynSmem);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(layout_kernel<IdxT, true>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(layout_kernel<IdxT, true>,
                                   cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err == cudaSuccess && dev < 32) done |= 1u << dev;
    return err;
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutParams &p0, cudaStream_t s)
{
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    err = set_attributes_once<IdxT>(dev);
    if (err != cudaSuccess) return err;

    LayoutParams p = p0;
    const long long routes = (long long)p.T * p.k;
    // one CTA up to ~2K routes, then a cluster of up to 16 CTAs
    int csize = (int)((routes + 2047) / 2048);
    csize = csize < 1 ? 1 : (csize > 16 ? 16 : csize);
    Geometry g = plan(p.T, p.k, p.E, p.R, csize);
    while (g.csize > 1 && max_clusters<IdxT>(g.csize, g.smem, dev) == 0)
        g = plan(p.T, p.k, p.E, p.R, g.csize > 8 ? 8 : g.csize >> 1);
    p.tpc = g.tpc;
    p.tch = g.tch;
    p.wde = g.wde;
    p.wdr = g.wdr;
    p.wds = g.wds;
    p.seg_words = g.seg_words;

    if (g.csize == 1) {
        layout_kernel<IdxT, false><<<1, 1024, g.smem, s>>>(p);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.csize, 1, 1);
    cfg.blockDim = dim3(1024, 1, 1);
    cfg.dynamicSmemBytes = g.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g.csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, layout_kernel<IdxT, true>, p);
}

}  // namespace

cudaError_t launch_layout(const LayoutParams &p, int idx_bits, cudaStream_t s)
{
    return idx_bits == 64 ? launch_layout_t<long long>(p, s) : launch_layout_t<int>(p, s);
}

}  // namespace epx
