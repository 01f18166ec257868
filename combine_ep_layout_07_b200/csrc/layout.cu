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
// Design: one launch of one CTA, or of one thread-block cluster of up to 16
// CTAs, each of 1024 threads.
//  * tokens are split into contiguous ranges: CTA c of the cluster, then
//    walker warp w of the CTA; a walker walks its range in steps of
//    floor(32/k) whole tokens, one route per lane, so lane order inside a
//    step is (token, slot) order;
//  * staging + counting: the CTA loads its routes with coalesced loads into
//    shared memory (one DRAM round trip), then one thread per token
//    validates the indices, computes each route's rank, marks the first
//    route of every (token, rank) pair and counts both into the walker's
//    histogram row with shared-memory atomics (order does not matter for
//    counts);
//  * walker scans: per expert (and per rank) an exclusive scan over the
//    walkers, several threads per expert, combined with warp shuffles;
//  * cluster exchange: each CTA pushes its totals into every peer's shared
//    memory (distributed shared memory stores) and one cluster barrier later
//    reads them all locally; a single CTA skips this;
//  * global scan: one block-wide scan of packed 64-bit (expert, rank) counts
//    gives both exclusive scans at once; the walker cursors become
//    offset + CTA base + walker prefix;
//  * ordered walk: __match_any_sync groups a step's lanes by expert (and the
//    first routes by rank); each lane takes its walker's cursor plus the
//    number of lower lanes in its group and the group leader advances it.
// Rows come out ordered by token, then slot, inside every expert segment and
// every rank segment, independent of scheduling.
#include <cooperative_groups.h>

#include "epx_internal.cuh"

namespace cg = cooperative_groups;

namespace epx {
namespace {

// staged route code: -2 = no token here, -1 = no route (or a dropped bad
// index), else expert | rank << 16 | (first route of its rank) << 30
constexpr int kAbsent = -2;
constexpr int kMaxPer = EPX_MAX_EXPERTS / 1024;  // experts per thread at most
constexpr int kScanInts = 2 * 34;                 // 64-bit block-scan scratch

// Exclusive scan of one 64-bit value per thread across the CTA.  No barrier
// after the last read of `sm`: the caller separates reuses with a barrier.
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

// Exclusive scan inside aligned groups of `width` lanes (a power of two);
// every lane of the warp takes part.  *total gets the group's sum.
__device__ __forceinline__ int group_exclusive_scan(int v, int width, int *total)
{
    const int sub = (threadIdx.x & 31) & (width - 1);
    int inc = v;
    for (int o = 1; o < width; o <<= 1) {
        const int n = __shfl_up_sync(kFull, inc, o, width);
        if (sub >= o) inc += n;
    }
    *total = __shfl_sync(kFull, inc, width - 1, width);
    return inc - v;
}

struct Ranges {
    int c0, c1;  // this CTA's tokens
    int tpw;     // tokens per walker warp
    __device__ int w0(int w) const { return min(c1, c0 + w * tpw); }
    __device__ int w1(int w) const { return min(c1, c0 + (w + 1) * tpw); }
};

__device__ __forceinline__ int rank_of(int e, float inv_epr)
{
    // exact for e < 2^22: (e + 1/2) / epr is at least 1/(2 epr) away from an
    // integer, far more than the two fp32 roundings can move it
    return __float2int_rd(__fmul_rn(__fadd_rn((float)e, 0.5f), inv_epr));
}

// Stage chunk c (tokens [w0 + c*S, w0 + c*S + S) of every walker w) into
// codes[w][s*k + j].  In the first pass also: fill recv_pos with -1 for the
// staged tokens, count every route into its walker's histograms and record
// bad indices / real tokens in misc[0] / misc[1].
template <typename IdxT>
__device__ void stage_chunk(const LayoutParams &p, const IdxT *__restrict__ idx,
                            const Ranges &rg, int c, int32_t *codes, int32_t *hist_e,
                            int32_t *hist_r, int32_t *misc, bool first_pass)
{
    const int k = p.k, S = p.S, E = p.E, R = p.R, NWW = p.nww;
    const int per_w = S * k;
    const int n = NWW * per_w;
    bool bad = false;
    // coalesced raw loads, four in flight per thread: consecutive threads
    // take consecutive routes of a walker's slice (contiguous in topk_idx)
    for (int i0 = threadIdx.x; i0 < n; i0 += 4 * blockDim.x) {
        long long e[4];
        bool in[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * blockDim.x;
            const int w = i / per_w;
            const int rem = i - w * per_w;
            in[u] = i < n && rg.w0(w) + c * S + rem / k < rg.w1(w);
            e[u] = in[u] ? (long long)idx[(size_t)rg.w0(w) * k + (size_t)c * per_w + rem] : -1;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * blockDim.x;
            if (i < n) {
                bad |= in[u] && (e[u] < -1 || e[u] >= E);
                codes[i] = !in[u] ? kAbsent : ((e[u] >= 0 && e[u] < E) ? (int)e[u] : -1);
            }
        }
    }
    if (first_pass) {
        const int per_wr = S * R;
        for (int i = threadIdx.x; i < NWW * per_wr; i += blockDim.x) {
            const int w = i / per_wr;
            const int rem = i - w * per_wr;
            if (rg.w0(w) + c * S + rem / R < rg.w1(w))
                p.recv_pos[(size_t)(rg.w0(w) + c * S) * R + rem] = -1;
        }
    }
    __syncthreads();
    // one thread per token: rank of each route, first route of each rank,
    // and (first pass) the counts
    int nreal = 0;
    for (int u = threadIdx.x; u < NWW * S; u += blockDim.x) {
        const int w = u / S;
        const int t = rg.w0(w) + c * S + (u - w * S);
        if (t >= rg.w1(w)) continue;
        int32_t *cd = codes + (size_t)u * k;
        unsigned long long mask = 0ull;
        for (int j = 0; j < k; ++j) {
            const int e = cd[j];
            if (e < 0) continue;
            const int r = rank_of(e, p.inv_epr);
            const bool f = !((mask >> r) & 1ull);
            mask |= 1ull << r;
            cd[j] = e | (r << 16) | ((int)f << 30);
            if (first_pass) {
                atomicAdd(&hist_e[w * E + e], 1);
                if (f) atomicAdd(&hist_r[w * R + r], 1);
            }
        }
        nreal += mask != 0ull;
    }
    if (first_pass) {
        if (__any_sync(kFull, bad) && (threadIdx.x & 31) == 0) atomicOr(&misc[0], 1);
        if (nreal) atomicAdd(&misc[1], nreal);
    }
    __syncthreads();
}

template <typename IdxT, bool CLUSTER>
__global__ void __launch_bounds__(1024, 1) layout_kernel(LayoutParams p)
{
    extern __shared__ __align__(16) int32_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int E = p.E, R = p.R, k = p.k, T = p.T, S = p.S, NWW = p.nww;

    int crank = 0, csize = 1;
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        crank = (int)cluster.block_rank();
        csize = (int)cluster.num_blocks();
        // every CTA must be running before a peer writes into its shared
        // memory: arrive now, wait just before the first remote store
        asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    }

    const int W = E + R + 2;  // one CTA's totals: experts, ranks, bad, real
    unsigned long long *scan = reinterpret_cast<unsigned long long *>(smem);
    int32_t *hist_e = smem + kScanInts;      // [NWW][E] walker counts, then cursors
    int32_t *hist_r = hist_e + NWW * E;      // [NWW][R]
    int32_t *all_tot = hist_r + NWW * R;     // [csize][W], row c = CTA c's totals
    int32_t *misc = all_tot + csize * W;     // [4]  0: bad-index flag, 1: real tokens
    int32_t *codes = misc + 4;               // [NWW][S*k] staged routes

    for (int i = tid; i < NWW * (E + R); i += blockDim.x) hist_e[i] = 0;
    if (tid < 4) misc[tid] = 0;
    __syncthreads();

    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    Ranges rg;
    rg.c0 = min(T, crank * p.tpc);
    rg.c1 = min(T, rg.c0 + p.tpc);
    rg.tpw = p.tpw;
    const int nchunks = (p.tpw + S - 1) / S;

    // ---- staging and counting
    for (int c = 0; c < nchunks; ++c) stage_chunk(p, idx, rg, c, codes, hist_e, hist_r, misc, true);

    if (CLUSTER) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");

    // ---- exclusive scans over walkers; publish this CTA's totals
    auto publish = [&](int slot, int v) {
        if (CLUSTER) {
            cg::cluster_group cluster = cg::this_cluster();
            for (int c = 0; c < csize; ++c) cluster.map_shared_rank(all_tot, c)[crank * W + slot] = v;
        } else {
            all_tot[slot] = v;
        }
    };
    const int tpe = p.tpe, per = p.per;
    const int g = tid / tpe, sub = tid & (tpe - 1);
    const int wps = (NWW + tpe - 1) / tpe;
    const int wa = min(NWW, sub * wps), wb = min(NWW, wa + wps);
#pragma unroll
    for (int q = 0; q < kMaxPer; ++q) {
        if (q >= per) break;
        const int e = g * per + q;
        const bool ok = e < E;
        int s = 0;
        if (ok)
            for (int w = wa; w < wb; ++w) s += hist_e[w * E + e];
        int tot;
        int run = group_exclusive_scan(s, tpe, &tot);
        if (ok) {
            for (int w = wa; w < wb; ++w) {
                const int v = hist_e[w * E + e];
                hist_e[w * E + e] = run;
                run += v;
            }
            if (sub == tpe - 1) publish(e, tot);
        }
    }
    const int tpr = p.tpr;
    const int gr = tid / tpr, subr = tid & (tpr - 1);
    const int wpr = (NWW + tpr - 1) / tpr;
    const int wra = min(NWW, subr * wpr), wrb = min(NWW, wra + wpr);
    {
        const bool ok = gr < R;
        int s = 0;
        if (ok)
            for (int w = wra; w < wrb; ++w) s += hist_r[w * R + gr];
        int tot;
        int run = group_exclusive_scan(s, tpr, &tot);
        if (ok) {
            for (int w = wra; w < wrb; ++w) {
                const int v = hist_r[w * R + gr];
                hist_r[w * R + gr] = run;
                run += v;
            }
            if (subr == tpr - 1) publish(E + gr, tot);
        }
    }
    if (tid == 0) {
        publish(E + R, misc[0]);
        publish(E + R + 1, misc[1]);
    }
    if (CLUSTER)
        cg::this_cluster().sync();  // all totals have arrived in every CTA
    else
        __syncthreads();

    // ---- global exclusive scans (one packed 64-bit block scan), cursors
    {
        int glob[kMaxPer], base[kMaxPer];
        unsigned int contrib_e = 0;
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            glob[q] = 0;
            base[q] = 0;
            const int e = g * per + q;
            if (q < per && e < E) {
                for (int c = 0; c < csize; ++c) {
                    const int v = all_tot[c * W + e];
                    base[q] += c < crank ? v : 0;
                    glob[q] += v;
                }
                contrib_e += glob[q];
            }
        }
        int glob_r = 0, base_r = 0;
        if (gr < R)
            for (int c = 0; c < csize; ++c) {
                const int v = all_tot[c * W + E + gr];
                base_r += c < crank ? v : 0;
                glob_r += v;
            }
        const unsigned long long v =
            ((unsigned long long)(sub == tpe - 1 ? contrib_e : 0u) << 32) |
            (unsigned long long)(gr < R && subr == tpr - 1 ? (unsigned)glob_r : 0u);
        unsigned long long total;
        const unsigned long long ex = block_exclusive_scan64(v, scan, &total);
        unsigned int run = (unsigned int)(ex >> 32);
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            const int e = g * per + q;
            if (q < per && e < E) {
                for (int w = wa; w < wb; ++w) hist_e[w * E + e] += (int)run + base[q];
                if (crank == 0 && sub == 0) {
                    p.cnt_e[e] = glob[q];
                    p.off_e[e] = (int)run;
                }
                run += glob[q];
            }
        }
        if (gr < R) {
            const int off_r = (int)(unsigned int)(ex & 0xffffffffull);
            for (int w = wra; w < wrb; ++w) hist_r[w * R + gr] += off_r + base_r;
            if (crank == 0 && subr == 0) {
                p.cnt_r[gr] = glob_r;
                p.off_r[gr] = off_r;
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
    __syncthreads();  // cursors visible to the walkers

    // ---- ordered walk: positions in (token, slot) order
    const int tps = 32 / k;
    const unsigned lt = lanemask_lt();
    const int tl = lane / k;
    const int j = lane - tl * k;
    for (int c = 0; c < nchunks; ++c) {
        if (nchunks > 1) stage_chunk(p, idx, rg, c, codes, hist_e, hist_r, misc, false);
        if (wid < NWW) {
            const int32_t *my_codes = codes + (size_t)wid * S * k;
            const int tb = rg.w0(wid) + c * S;  // first token of this walker's slice
            for (int s0 = 0; s0 < S; s0 += tps) {
                const int s = s0 + tl;
                const bool lane_ok = tl < tps && s < S;
                const int code = lane_ok ? my_codes[s * k + j] : kAbsent;
                const bool valid = code >= 0;
                const int e = valid ? (code & 0xffff) : -1;
                const bool first = valid && (code & (1 << 30));
                const int r = (code >> 16) & 0x3f;
                const unsigned pe = __match_any_sync(kFull, e);
                const unsigned pr = __match_any_sync(kFull, first ? r : -1);
                const int base = valid ? hist_e[wid * E + e] : 0;
                const int base_r = first ? hist_r[wid * R + r] : 0;
                __syncwarp();
                if (valid && lane == __ffs(pe) - 1) hist_e[wid * E + e] = base + __popc(pe);
                if (first && lane == __ffs(pr) - 1) hist_r[wid * R + r] = base_r + __popc(pr);
                const size_t t = (size_t)(tb + s);
                if (code != kAbsent) p.pos[t * k + j] = valid ? base + __popc(pe & lt) : -1;
                if (first) p.recv_pos[t * R + r] = base_r + __popc(pr & lt);
                __syncwarp();
            }
        }
        if (nchunks > 1) __syncthreads();  // codes are restaged next chunk
    }
}

size_t layout_smem_bytes(int nww, int E, int R, int S, int k, int csize)
{
    return sizeof(int32_t) * ((size_t)kScanInts + (size_t)nww * (E + R) +
                              (size_t)csize * (E + R + 2) + 4 + (size_t)nww * S * k);
}

int pow2_floor(int v)
{
    int p = 1;
    while (p * 2 <= v) p *= 2;
    return p;
}

int pow2_ceil(int v)
{
    int p = 1;
    while (p < v) p *= 2;
    return p;
}

struct Geometry {
    int csize, nww, tpc, tpw, S, tpe, per, tpr;
    size_t smem;
};

// Cluster size, walker warps, staging chunk and scan mapping for a layout
// problem (1024 threads per CTA).
Geometry plan(int T, int k, int E, int R, int csize)
{
    Geometry g;
    const int tps = 32 / k;
    g.csize = csize;
    g.tpc = (T + csize - 1) / csize;
    const int steps = (g.tpc + tps - 1) / tps;
    // one ordered step per walker when possible (at most 32 walkers)
    int nww = steps < 1 ? 1 : (steps > 32 ? 32 : steps);
    for (;;) {
        int tpw = (g.tpc + nww - 1) / nww;
        tpw = ((tpw + tps - 1) / tps) * tps;
        if (tpw < tps) tpw = tps;
        const size_t base = layout_smem_bytes(nww, E, R, 0, k, csize);
        const long long avail = (long long)kMaxDynSmem - (long long)base;
        int S = avail > 0 ? (int)(avail / ((long long)nww * k * 4)) : 0;
        S = (S / tps) * tps;
        if (S > tpw) S = tpw;
        if (S >= tps || nww == 1) {
            g.nww = nww;
            g.tpw = tpw;
            g.S = S < tps ? tps : S;
            g.smem = layout_smem_bytes(nww, E, R, g.S, k, csize);
            break;
        }
        --nww;
    }
    const int wcap = pow2_ceil(g.nww);
    if (E <= 1024) {
        g.per = 1;
        g.tpe = pow2_floor(1024 / E);
        if (g.tpe > 32) g.tpe = 32;
        if (g.tpe > wcap) g.tpe = wcap;
    } else {
        g.per = (E + 1023) / 1024;
        g.tpe = 1;
    }
    g.tpr = pow2_floor(1024 / R);
    if (g.tpr > 32) g.tpr = 32;
    if (g.tpr > wcap) g.tpr = wcap;
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
    p.tpw = g.tpw;
    p.S = g.S;
    p.nww = g.nww;
    p.tpe = g.tpe;
    p.per = g.per;
    p.tpr = g.tpr;
    p.inv_epr = 1.0f / (float)p.epr;

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
