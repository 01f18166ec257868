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
// Design (one launch, one thread-block cluster of up to 8 CTAs):
//  * tokens are split into contiguous ranges: CTA c of the cluster, then
//    warp w of the CTA, then steps of floor(32/k) whole tokens, one route per
//    lane, so lane order inside a step is (token, slot) order;
//  * pass 1: warp-aggregated counting -- __match_any_sync groups the lanes of
//    a step by expert (and by (token, rank) to deduplicate ranks) and the
//    group leader adds the group size to the warp's private histogram row in
//    shared memory, so no atomics are needed;
//  * scans: per expert, an exclusive scan over the CTA's warps; the CTA
//    totals are exchanged through distributed shared memory, giving each CTA
//    its base and every CTA the global exclusive scan over experts;
//  * pass 2: the same walk again, each lane taking its expert's warp cursor
//    plus its rank among equal experts in the step (popc of the lower peers).
// Rows therefore come out ordered by token, then slot, inside every expert
// segment and every rank segment, independent of scheduling.
#include <cooperative_groups.h>

#include "epx_internal.cuh"

namespace cg = cooperative_groups;

namespace epx {
namespace {

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

// One step of a warp's walk: lane = route (t0 + lane / k, lane % k).
struct Step {
    bool act;     // lane holds a route of a token in range
    bool valid;   // ... and its expert index is in [0, E)
    bool bad;     // ... or its index is < -1 or >= E
    bool first;   // first valid lane of its (token, rank) pair
    int e, r;     // expert and rank (valid lanes)
    unsigned pe;  // lanes with the same expert
    unsigned pr;  // first-lanes with the same rank
    int nreal;    // tokens of the step with >= 1 valid route (same on all lanes)
};

template <typename IdxT>
__device__ __forceinline__ Step make_step(const IdxT *__restrict__ idx, int t0,
                                          int tend, int k, int E, int epr,
                                          int tps, int lane)
{
    Step s;
    const int tl = lane / k;
    const int j = lane - tl * k;
    const int t = t0 + tl;
    s.act = tl < tps && t < tend;
    long long e = s.act ? (long long)idx[(size_t)t * k + j] : -1;
    s.bad = s.act && (e < -1 || e >= E);
    s.valid = s.act && e >= 0 && e < E;
    s.e = s.valid ? (int)e : -1;
    s.pe = __match_any_sync(kFull, s.e);
    s.r = s.valid ? s.e / epr : 0;
    // (token slot, rank) key: tl < 32 and r < 64
    const unsigned ptr = __match_any_sync(kFull, s.valid ? (tl << 6) | s.r : -1);
    s.first = s.valid && lane == __ffs(ptr) - 1;
    s.pr = __match_any_sync(kFull, s.first ? s.r : -1);
    // real tokens in this step
    const unsigned vm = __ballot_sync(kFull, s.valid);
    const unsigned kmask = k == 32 ? kFull : ((1u << k) - 1u);
    const bool real = lane < tps && ((vm >> (lane * k)) & kmask) != 0u;
    s.nreal = __popc(__ballot_sync(kFull, real));
    return s;
}

template <typename IdxT>
__global__ void __launch_bounds__(1024, 1) layout_kernel(LayoutParams p)
{
    extern __shared__ __align__(16) int32_t smem[];
    const int NW = blockDim.x >> 5;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int E = p.E, R = p.R, k = p.k, T = p.T;
    int32_t *hist_e = smem;              // [NW][E] per-warp counts, then cursors
    int32_t *hist_r = hist_e + NW * E;   // [NW][R]
    int32_t *tot_e = hist_r + NW * R;    // [E]  CTA totals (read by peer CTAs)
    int32_t *tot_r = tot_e + E;          // [R]
    int32_t *misc = tot_r + R;           // [4]  0: bad-index flag, 1: real tokens
    int32_t *scan = misc + 4;            // [34]

    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();
    const int csize = (int)cluster.num_blocks();

    for (int i = tid; i < NW * (E + R); i += blockDim.x) hist_e[i] = 0;
    if (tid < 4) misc[tid] = 0;
    __syncthreads();

    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    const int tps = 32 / k;
    const int c0 = min(T, crank * p.tpc), c1 = min(T, c0 + p.tpc);
    const int w0 = min(c1, c0 + wid * p.tpw), w1 = min(c1, w0 + p.tpw);

    // tokens not sent to a rank keep -1 (pass 2 overwrites the sent pairs)
    for (long long i = (long long)w0 * R + lane; i < (long long)w1 * R; i += 32)
        p.recv_pos[i] = -1;

    // ---- pass 1: warp-private histograms
    bool bad = false;
    int nreal = 0;
    for (int t0 = w0; t0 < w1; t0 += tps) {
        Step s = make_step(idx, t0, w1, k, E, p.epr, tps, lane);
        bad |= s.bad;
        nreal += s.nreal;
        if (s.valid && lane == __ffs(s.pe) - 1) hist_e[wid * E + s.e] += __popc(s.pe);
        if (s.first && lane == __ffs(s.pr) - 1) hist_r[wid * R + s.r] += __popc(s.pr);
        __syncwarp();
    }
    bad = __any_sync(kFull, bad);
    if (lane == 0) {
        if (bad) atomicOr(&misc[0], 1);
        atomicAdd(&misc[1], nreal);
    }
    __syncthreads();

    // ---- exclusive scan over this CTA's warps, per expert / per rank
    for (int e = tid; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < NW; ++w) {
            int v = hist_e[w * E + e];
            hist_e[w * E + e] = run;
            run += v;
        }
        tot_e[e] = run;
    }
    for (int r = tid; r < R; r += blockDim.x) {
        int run = 0;
        for (int w = 0; w < NW; ++w) {
            int v = hist_r[w * R + r];
            hist_r[w * R + r] = run;
            run += v;
        }
        tot_r[r] = run;
    }
    cluster.sync();  // every CTA's totals are now readable by its peers

    // ---- cluster-wide: base of this CTA, global scan over experts / ranks
    {
        const int per = (E + blockDim.x - 1) / blockDim.x;
        const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
        int local = 0;
        for (int e = e0; e < e1; ++e)
            for (int c = 0; c < csize; ++c) local += cluster.map_shared_rank(tot_e, c)[e];
        int total_e;
        int run = block_exclusive_scan(local, scan, &total_e);
        for (int e = e0; e < e1; ++e) {
            int base = 0, tot = 0;
            for (int c = 0; c < csize; ++c) {
                int v = cluster.map_shared_rank(tot_e, c)[e];
                base += c < crank ? v : 0;
                tot += v;
            }
            for (int w = 0; w < NW; ++w) hist_e[w * E + e] += run + base;
            if (crank == 0) {
                p.cnt_e[e] = tot;
                p.off_e[e] = run;
            }
            run += tot;
        }

        const int r = tid;
        int tot_rr = 0, base_r = 0;
        if (r < R) {
            for (int c = 0; c < csize; ++c) {
                int v = cluster.map_shared_rank(tot_r, c)[r];
                base_r += c < crank ? v : 0;
                tot_rr += v;
            }
        }
        int total_r;
        int off_r = block_exclusive_scan(tot_rr, scan, &total_r);
        if (r < R) {
            for (int w = 0; w < NW; ++w) hist_r[w * R + r] += off_r + base_r;
            if (crank == 0) {
                p.cnt_r[r] = tot_rr;
                p.off_r[r] = off_r;
            }
        }
        if (tid == 0) {
            int errc = 0, nr = 0;
            for (int c = 0; c < csize; ++c) {
                const int32_t *m = cluster.map_shared_rank(misc, c);
                errc |= m[0];
                nr += m[1];
            }
            if (crank == 0) {
                p.off_e[E] = total_e;
                p.off_r[R] = total_r;
                p.totals[0] = total_e;
                p.totals[1] = total_r;
                p.totals[2] = nr;
                p.totals[3] = errc ? (int32_t)EP_DEVERR_BAD_INDEX : 0;
            }
        }
    }
    cluster.sync();  // peers are done reading; cursors visible CTA-wide

    // ---- pass 2: positions
    const unsigned lt = lanemask_lt();
    for (int t0 = w0; t0 < w1; t0 += tps) {
        Step s = make_step(idx, t0, w1, k, E, p.epr, tps, lane);
        const int tl = lane / k;
        const int t = t0 + tl;
        int base = s.valid ? hist_e[wid * E + s.e] : 0;
        int base_r = s.first ? hist_r[wid * R + s.r] : 0;
        __syncwarp();
        if (s.valid && lane == __ffs(s.pe) - 1) hist_e[wid * E + s.e] = base + __popc(s.pe);
        if (s.first && lane == __ffs(s.pr) - 1) hist_r[wid * R + s.r] = base_r + __popc(s.pr);
        if (s.act) p.pos[(size_t)t * k + (lane - tl * k)] = s.valid ? base + __popc(s.pe & lt) : -1;
        if (s.first) p.recv_pos[(size_t)t * R + s.r] = base_r + __popc(s.pr & lt);
        __syncwarp();
    }
}

size_t layout_smem_bytes(int NW, int E, int R)
{
    return sizeof(int32_t) * ((size_t)NW * (E + R) + E + R + 4 + 34);
}

// cudaOccupancyMaxActiveClusters for (cluster size, threads, smem), cached
// per device; 0 means such a cluster cannot be scheduled.
template <typename IdxT>
int max_cluster_ok(int csize, int threads, size_t smem, int dev)
{
    struct Entry { int dev, csize, threads; size_t smem; int result; };
    static Entry cache[32];
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
    if (n_cache < 32) cache[n_cache++] = Entry{dev, csize, threads, smem, n};
    return n;
}

template <typename IdxT>
cudaError_t launch_layout_t(const LayoutParams &p0, cudaStream_t s)
{
    static int attr_set_mask = 0;  // per device (up to 32), set once
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 32 && !(attr_set_mask & (1 << dev))) {
        err = cudaFuncSetAttribute(layout_kernel<IdxT>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kMaxDynSmem);
        if (err != cudaSuccess) return err;
        attr_set_mask |= 1 << dev;
    }

    LayoutParams p = p0;
    const int T = p.T, k = p.k, E = p.E, R = p.R;
    const int tps = 32 / k;
    const long long routes = (long long)T * k;
    // one CTA up to ~4K routes, then up to an 8-CTA cluster
    int csize = (int)((routes + 4095) / 4096);
    csize = csize < 1 ? 1 : (csize > 8 ? 8 : csize);
    int nw_max = 32;
    while (nw_max > 1 && layout_smem_bytes(nw_max, E, R) > (size_t)kMaxDynSmem) --nw_max;
    // largest cluster (<= csize) that the device can co-schedule at this size
    while (csize > 1 && max_cluster_ok<IdxT>(csize, nw_max * 32,
                                             layout_smem_bytes(nw_max, E, R), dev) == 0)
        csize >>= 1;
    const int tpc = (T + csize - 1) / csize;
    int steps = (tpc + tps - 1) / tps;
    int NW = steps < 1 ? 1 : (steps > nw_max ? nw_max : steps);
    // the rank scan gives one rank to each thread
    const int nw_ranks = (R + 31) / 32;
    if (NW < nw_ranks) NW = nw_ranks;
    int tpw = (tpc + NW - 1) / NW;
    tpw = ((tpw + tps - 1) / tps) * tps;
    if (tpw < tps) tpw = tps;
    p.tpc = tpc;
    p.tpw = tpw;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize, 1, 1);
    cfg.blockDim = dim3(NW * 32, 1, 1);
    cfg.dynamicSmemBytes = layout_smem_bytes(NW, E, R);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
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
