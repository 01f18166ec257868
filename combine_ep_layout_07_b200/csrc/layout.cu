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
// Design (one launch, one thread-block cluster of up to 8 CTAs of 1024
// threads):
//  * tokens are split into contiguous ranges: CTA c of the cluster, then
//    walker warp w of the CTA; each walker walks its range in steps of
//    floor(32/k) whole tokens, one route per lane, so lane order inside a
//    step is (token, slot) order;
//  * staging: the CTA loads its routes with coalesced loads into shared
//    memory (one DRAM round trip instead of one per step), then one thread
//    per token validates the indices, computes each route's rank e / (E/R)
//    and marks the first route of every (token, rank) pair;
//  * pass 1: per-walker histograms of experts and of first routes per rank,
//    counted with shared-memory atomics (order does not matter for counts);
//  * scans: per expert, an exclusive scan over the CTA's walkers; each CTA
//    pushes its totals into every peer's shared memory (distributed shared
//    memory stores), one cluster barrier, then every CTA reads them locally
//    to get its base and the global exclusive scan over experts / ranks;
//  * pass 2: the ordered walk -- __match_any_sync groups a step's lanes by
//    expert (and first-routes by rank); each lane takes the walker's cursor
//    plus the number of lower lanes in its group, the group leader advances it.
// Expert-proportional work (zeroing, scans, writing counts and offsets) uses
// all 1024 threads, so it stays short even for a single token.
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

// Exclusive scan of one int per thread across the CTA.  `sm` has >= 34 ints.
__device__ int block_exclusive_scan(int v, int *sm, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) sm[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int s = lane < nw ? sm[lane] : 0;
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(kFull, si, o);
            if (lane >= o) si += n;
        }
        if (lane < nw) sm[lane] = si - s;
        if (lane == 31) sm[32] = si;
    }
    __syncthreads();
    int res = sm[wid] + inc - v;
    *total = sm[32];
    __syncthreads();
    return res;
}

struct Ranges {
    int c0, c1;  // this CTA's tokens
    int tpw;     // tokens per walker warp
    __device__ int w0(int w) const { return min(c1, c0 + w * tpw); }
    __device__ int w1(int w) const { return min(c1, c0 + (w + 1) * tpw); }
};

// Stage chunk c (tokens [w0 + c*S, w0 + c*S + S) of every walker w) into
// codes[w][s*k + j].  first_pass also fills recv_pos with -1 for the staged
// tokens and counts bad indices / real tokens into misc[0] / misc[1].
template <typename IdxT>
__device__ void stage_chunk(const LayoutParams &p, const IdxT *__restrict__ idx,
                            const Ranges &rg, int c, int32_t *codes, int32_t *misc,
                            bool first_pass)
{
    const int k = p.k, S = p.S, E = p.E, R = p.R, NWW = p.nww;
    const int per_w = S * k;
    bool bad = false;
    // coalesced raw load: consecutive threads take consecutive routes of a
    // walker's slice (the slice is contiguous in topk_idx)
    for (int i = threadIdx.x; i < NWW * per_w; i += blockDim.x) {
        const int w = i / per_w;
        const int rem = i - w * per_w;
        const int t = rg.w0(w) + c * S + rem / k;
        int code = kAbsent;
        if (t < rg.w1(w)) {
            const long long e = (long long)idx[(size_t)rg.w0(w) * k + (size_t)c * per_w + rem];
            bad |= (e < -1 || e >= E);
            code = (e >= 0 && e < E) ? (int)e : -1;
        }
        codes[i] = code;
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
    // one thread per token: rank of each route, first route of each rank
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
            const int r = e / p.epr;
            const bool f = !((mask >> r) & 1ull);
            mask |= 1ull << r;
            cd[j] = e | (r << 16) | ((int)f << 30);
        }
        nreal += mask != 0ull;
    }
    if (first_pass) {
        if (bad) atomicOr(&misc[0], 1);
        if (nreal) atomicAdd(&misc[1], nreal);
    }
    __syncthreads();
}

template <typename IdxT>
__global__ void __launch_bounds__(1024, 1) layout_kernel(LayoutParams p)
{
    extern __shared__ __align__(16) int32_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int E = p.E, R = p.R, k = p.k, T = p.T, S = p.S, NWW = p.nww;

    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int csize = (int)cluster.num_blocks();

    const int W = E + R + 2;                 // one CTA's totals: experts, ranks, bad, real
    int32_t *hist_e = smem;                  // [NWW][E] per-walker counts, then cursors
    int32_t *hist_r = hist_e + NWW * E;      // [NWW][R]
    int32_t *all_tot = hist_r + NWW * R;     // [csize][W], row c written by CTA c
    int32_t *misc = all_tot + csize * W;     // [4]  0: bad-index flag, 1: real tokens
    int32_t *scan = misc + 4;                // [36]
    int32_t *codes = scan + 36;              // [NWW][S*k] staged routes

    // every CTA of the cluster must be running before a peer writes into its
    // shared memory: arrive now, wait just before the first remote store
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    for (int i = tid; i < NWW * (E + R); i += blockDim.x) hist_e[i] = 0;
    if (tid < 4) misc[tid] = 0;
    __syncthreads();

    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    const int tps = 32 / k;
    Ranges rg;
    rg.c0 = min(T, crank * p.tpc);
    rg.c1 = min(T, rg.c0 + p.tpc);
    rg.tpw = p.tpw;
    const int nchunks = (p.tpw + S - 1) / S;

    // ---- pass 1: per-walker histograms (shared-memory atomics, any order)
    for (int c = 0; c < nchunks; ++c) {
        stage_chunk(p, idx, rg, c, codes, misc, true);
        const int per_w = S * k;
        for (int i = tid; i < NWW * per_w; i += blockDim.x) {
            const int code = codes[i];
            if (code < 0) continue;
            const int w = i / per_w;
            atomicAdd(&hist_e[w * E + (code & 0xffff)], 1);
            if (code & (1 << 30)) atomicAdd(&hist_r[w * R + ((code >> 16) & 0x3f)], 1);
        }
        __syncthreads();
    }

    // ---- exclusive scan over walkers; push this CTA's totals to every CTA
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    for (int e = tid; e < E + R; e += blockDim.x) {
        int32_t *h = e < E ? hist_e + e : hist_r + (e - E);
        const int stride = e < E ? E : R;
        int run = 0;
        for (int w = 0; w < NWW; ++w) {
            const int v = h[w * stride];
            h[w * stride] = run;
            run += v;
        }
        for (int c = 0; c < csize; ++c) cluster.map_shared_rank(all_tot, c)[crank * W + e] = run;
    }
    if (tid == 0)
        for (int c = 0; c < csize; ++c) {
            int32_t *dst = cluster.map_shared_rank(all_tot, c) + crank * W;
            dst[E + R] = misc[0];
            dst[E + R + 1] = misc[1];
        }
    cluster.sync();  // all totals have arrived in every CTA's shared memory

    // ---- global exclusive scans (local reads only), cursors, CTA 0 writes out
    {
        const int per = (E + blockDim.x - 1) / blockDim.x;
        const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
        int local = 0;
        for (int e = e0; e < e1; ++e)
            for (int c = 0; c < csize; ++c) local += all_tot[c * W + e];
        int total_e;
        int run = block_exclusive_scan(local, scan, &total_e);
        for (int e = e0; e < e1; ++e) {
            int base = 0, tot = 0;
            for (int c = 0; c < csize; ++c) {
                const int v = all_tot[c * W + e];
                base += c < crank ? v : 0;
                tot += v;
            }
            for (int w = 0; w < NWW; ++w) hist_e[w * E + e] += run + base;
            if (crank == 0) {
                p.cnt_e[e] = tot;
                p.off_e[e] = run;
            }
            run += tot;
        }

        const int r = tid;
        int tot_rr = 0, base_r = 0;
        if (r < R)
            for (int c = 0; c < csize; ++c) {
                const int v = all_tot[c * W + E + r];
                base_r += c < crank ? v : 0;
                tot_rr += v;
            }
        int total_r;
        const int off_r = block_exclusive_scan(tot_rr, scan, &total_r);
        if (r < R) {
            for (int w = 0; w < NWW; ++w) hist_r[w * R + r] += off_r + base_r;
            if (crank == 0) {
                p.cnt_r[r] = tot_rr;
                p.off_r[r] = off_r;
            }
        }
        if (tid == 0 && crank == 0) {
            int errc = 0, nr = 0;
            for (int c = 0; c < csize; ++c) {
                errc |= all_tot[c * W + E + R];
                nr += all_tot[c * W + E + R + 1];
            }
            p.off_e[E] = total_e;
            p.off_r[R] = total_r;
            p.totals[0] = total_e;
            p.totals[1] = total_r;
            p.totals[2] = nr;
            p.totals[3] = errc ? (int32_t)EP_DEVERR_BAD_INDEX : 0;
        }
    }
    __syncthreads();  // cursors visible to the walkers

    // ---- pass 2: positions, in (token, slot) order, by the walker warps
    const unsigned lt = lanemask_lt();
    const int tl = lane / k;
    const int j = lane - tl * k;
    for (int c = 0; c < nchunks; ++c) {
        if (nchunks > 1) stage_chunk(p, idx, rg, c, codes, misc, false);
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

size_t layout_smem_bytes(int NWW, int E, int R, int S, int k, int csize)
{
    return sizeof(int32_t) *
           ((size_t)NWW * (E + R) + (size_t)csize * (E + R + 2) + 4 + 36 + (size_t)NWW * S * k);
}

// cudaOccupancyMaxActiveClusters for (cluster size, threads, smem), cached
// per device; 0 means such a cluster cannot be scheduled.
template <typename IdxT>
int max_clusters(int csize, int threads, size_t smem, int dev)
{
    struct Entry {
        int dev, csize, threads;
        size_t smem;
        int result;
    };
    static Entry cache[64];
    static int n_cache = 0;
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].dev == dev && cache[i].csize == csize && cache[i].threads == threads &&
            cache[i].smem == smem)
            return cache[i].result;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, layout_kernel<IdxT>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (n_cache < 64) cache[n_cache++] = Entry{dev, csize, threads, smem, n};
    return n;
}

struct Geometry {
    int csize, threads, nww, tpc, tpw, S;
    size_t smem;
};

// Cluster size, walker warps and staging chunk for a layout problem.  The
// CTA always has 1024 threads: the expert-proportional work (zeroing, scans,
// writing counts and offsets) is spread over all of them, while only the
// walker warps own token ranges.
Geometry plan(int T, int k, int E, int R, int csize)
{
    Geometry g;
    const int tps = 32 / k;
    g.csize = csize;
    g.threads = 1024;
    g.tpc = (T + csize - 1) / csize;
    const int steps = (g.tpc + tps - 1) / tps;
    // about 4 ordered steps per walker: enough walkers to spread the walk,
    // few enough that the per-expert scans over walkers stay short
    int nww = (steps + 3) / 4;
    if (nww > 32) nww = 32;
    if (nww < 1) nww = 1;
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
            return g;
        }
        --nww;
    }
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutParams &p0, cudaStream_t s)
{
    static unsigned attr_set_mask = 0;  // per device (up to 32), set once
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 32 && !(attr_set_mask & (1u << dev))) {
        err = cudaFuncSetAttribute(layout_kernel<IdxT>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (err != cudaSuccess) return err;
        attr_set_mask |= 1u << dev;
    }

    LayoutParams p = p0;
    const long long routes = (long long)p.T * p.k;
    // one CTA up to ~4K routes, then up to an 8-CTA cluster
    int csize = (int)((routes + 4095) / 4096);
    csize = csize < 1 ? 1 : (csize > 8 ? 8 : csize);
    Geometry g = plan(p.T, p.k, p.E, p.R, csize);
    while (g.csize > 1 && max_clusters<IdxT>(g.csize, g.threads, g.smem, dev) == 0)
        g = plan(p.T, p.k, p.E, p.R, g.csize >> 1);
    p.tpc = g.tpc;
    p.tpw = g.tpw;
    p.S = g.S;
    p.nww = g.nww;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g.csize, 1, 1);
    cfg.blockDim = dim3(g.threads, 1, 1);
    cfg.dynamicSmemBytes = g.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g.csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, layout_kernel<IdxT>, p);
}

}  // namespace

cudaError_t launch_layout(const LayoutParams &p, int idx_bits, cudaStream_t s)
{
    return idx_bits == 64 ? launch_layout_t<long long>(p, s) : launch_layout_t<int>(p, s);
}

}  // namespace epx
