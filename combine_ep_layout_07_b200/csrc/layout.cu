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
// is off_r[r] + (earlier tokens that reach r).  Both middle terms are prefix
// sums over tokens, computed without any ordering primitive by one of two
// schedules with identical results: the warp-chunk schedule (the default
// wherever its per-warp table fits; described at layout_warp_kernel below)
// and the count-matrix schedule, which handles every valid size:
//  * one launch of one CTA, or of one thread-block cluster of up to 16 CTAs
//    of 1024 threads; CTA c owns a contiguous range of tokens;
//  * build: one thread per token loads its k indices, validates them,
//    computes each route's rank, marks the first route of every
//    (token, rank) pair and counts its column of the matrix in shared
//    memory -- counts are packed two 16-bit rows per 32-bit word, and the
//    count seen before incrementing is the route's rank among equal experts
//    of its own token;
//  * row scan: one thread per matrix row walks its tokens and rewrites the
//    counts as a running prefix (packed 16-bit halves add independently);
//    the row sum is the CTA total;
//  * cluster exchange: each CTA stores its totals into its own row of every
//    peer's totals table (distributed-shared-memory stores); after one
//    cluster barrier each CTA sums the table locally, over all CTAs and over
//    the CTAs below it; a single CTA skips this;
//  * global scan: one packed 64-bit block scan of the (expert, rank) totals
//    gives both exclusive scans, plus this CTA's base per expert / rank;
//  * placement: one thread per four routes, then per four (token, rank)
//    pairs, so the stores of pos / recv_pos are coalesced 16-byte vectors.
// When a CTA's tokens do not fit in shared memory at once, it counts all of
// them first (atomics into its totals) and then builds, scans and places the
// tokens chunk by chunk with a running base per row.
#include <cooperative_groups.h>

#include "epx_internal.cuh"

namespace cg = cooperative_groups;

namespace epx {
namespace {

// route code in shared memory: -1 = no route (or a dropped bad index), else
// expert | (rank among equal experts of the token) << 12
__device__ __forceinline__ int code_e(int c) { return c & 0xfff; }
__device__ __forceinline__ int code_dup(int c) { return (c >> 12) & 0x1f; }

__device__ __forceinline__ int rank_of(int e, float inv_epr)
{
    // exact for e < 2^22: (e + 1/2) / epr is at least 1/(2 epr) away from an
    // integer, far more than the two fp32 roundings can move it
    return __float2int_rd(__fmul_rn(__fadd_rn((float)e, 0.5f), inv_epr));
}

__device__ __forceinline__ int div_small(int i, float inv)
{
    // floor(i / d) for 0 <= i < 2^22 with inv = 1/d (same argument as rank_of)
    return __float2int_rd(__fmul_rn(__fadd_rn((float)i, 0.5f), inv));
}

__device__ __forceinline__ uint32_t half16(uint32_t w, int sh) { return (w >> sh) & 0xffffu; }

struct Smem {
    uint32_t *M;              // [wde + wdr][ld] counts, then in-chunk prefixes (ld odd)
    int32_t *codes;           // [tch][k]
    unsigned long long *hit;  // [tch] ranks each token reaches
    int32_t *tot;             // [E + R] CTA totals / chunk sums
    int32_t *base;            // [E + R] this CTA's first row per expert / rank
    int32_t *all_tot;         // [csize][E + R + 2] every CTA's totals, bad flag, real tokens
                              // (grid schedule: partial column sums)
    int32_t *misc;            // [2] bad flag, real tokens
    int32_t *low;             // grid schedule: [E + R] totals of the CTAs below this one
    unsigned long long *scan; // [34] block-scan scratch
};

// Thread-per-token pass over tokens [t0, t0 + n).  With count_only it adds
// each route into the CTA totals with atomics; otherwise it counts the
// token's matrix column (zeroed beforehand) and records codes and rank masks.
// Returns this thread's number of tokens with a valid route; *bad is set if
// an index < -1 or >= E was seen.
template <typename IdxT>
__device__ int build_tokens(const LayoutParams &p, const IdxT *__restrict__ idx, int t0, int n,
                            const Smem &sm, bool count_only, bool *bad)
{
    const int k = p.k, E = p.E, ld = p.ld;
    int nreal = 0;
    for (int u = threadIdx.x; u < n; u += blockDim.x) {
        const IdxT *row = idx + (size_t)(t0 + u) * k;
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
                    if (count_only) {
                        atomicAdd(&sm.tot[ei], 1);
                        if (first) atomicAdd(&sm.tot[E + r], 1);
                    } else {
                        const int sh = (ei & 1) * 16;
                        uint32_t *cell = sm.M + (size_t)(ei >> 1) * ld + u;
                        const uint32_t w = *cell;
                        *cell = w + (1u << sh);
                        if (first) sm.M[(size_t)(p.wde + (r >> 1)) * ld + u] += 1u << ((r & 1) * 16);
                        code = ei | ((int)half16(w, sh) << 12);
                    }
                }
                if (!count_only) sm.codes[(size_t)u * k + j] = code;
            }
        }
        if (!count_only) sm.hit[u] = mask;
        nreal += mask != 0ull;
    }
    return nreal;
}

// Exclusive prefix over the n tokens of every matrix row: one thread per row,
// walking its tokens eight at a time (loads first, then the rewritten
// prefixes); the row stride is odd, so the 32 rows of a warp sit in 32
// different banks.  The row totals, unpacked, go to tot[E + R].
__device__ void row_scan(const LayoutParams &p, const Smem &sm, int n)
{
    const int wdt = p.wde + p.wdr;
    for (int w = threadIdx.x; w < wdt; w += blockDim.x) {
        uint32_t *row = sm.M + (size_t)w * p.ld;
        uint32_t run = 0;
        for (int c = 0; c < n; c += 8) {
            uint32_t v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = c + i < n ? row[c + i] : 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (c + i < n) row[c + i] = run;
                run += v[i];
            }
        }
        const bool er = w < p.wde;
        const int c0 = er ? 2 * w : 2 * (w - p.wde);
        const int lim = er ? p.E : p.R;
        int32_t *dst = er ? sm.tot : sm.tot + p.E;
        dst[c0] = (int32_t)(run & 0xffffu);
        if (c0 + 1 < lim) dst[c0 + 1] = (int32_t)(run >> 16);
    }
}

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

constexpr int kMaxPer = EPX_MAX_EXPERTS / 1024;  // experts per thread at most

// pos / recv_pos of tokens [t0, t0 + n): one thread per four routes (or per
// route when k is not a multiple of 4), then per four (token, rank) pairs;
// the 16-byte stores are coalesced.
__device__ __forceinline__ int route_pos(const LayoutParams &p, const Smem &sm, int i, int u)
{
    const int c = sm.codes[i];
    if (c < 0) return -1;
    const int e = code_e(c);
    return sm.base[e] +
           (int)half16(sm.M[(size_t)(e >> 1) * p.ld + u], (e & 1) * 16) +
           code_dup(c);
}

__device__ __forceinline__ int pair_pos(const LayoutParams &p, const Smem &sm, int u, int r)
{
    if (!((sm.hit[u] >> r) & 1ull)) return -1;
    return sm.base[p.E + r] +
           (int)half16(sm.M[(size_t)(p.wde + (r >> 1)) * p.ld + u], (r & 1) * 16);
}

__device__ void place_tokens(const LayoutParams &p, const Smem &sm, int t0, int n)
{
    const int k = p.k, R = p.R;
    if ((k & 3) == 0) {
        const int k4 = k >> 2;
        const float inv = 1.0f / (float)k4;
        int4 *dst = reinterpret_cast<int4 *>(p.pos + (size_t)t0 * k);
        for (int i = threadIdx.x; i < n * k4; i += blockDim.x) {
            const int u = div_small(i, inv);
            const int j = 4 * i;
            dst[i] = make_int4(route_pos(p, sm, j, u), route_pos(p, sm, j + 1, u),
                               route_pos(p, sm, j + 2, u), route_pos(p, sm, j + 3, u));
        }
    } else {
        const float inv = 1.0f / (float)k;
        for (int i = threadIdx.x; i < n * k; i += blockDim.x)
            p.pos[(size_t)t0 * k + i] = route_pos(p, sm, i, div_small(i, inv));
    }
    if ((R & 3) == 0) {
        const int r4 = R >> 2;
        const float inv = 1.0f / (float)r4;
        int4 *dst = reinterpret_cast<int4 *>(p.recv_pos + (size_t)t0 * R);
        for (int i = threadIdx.x; i < n * r4; i += blockDim.x) {
            const int u = div_small(i, inv);
            const int r = 4 * (i - u * r4);
            dst[i] = make_int4(pair_pos(p, sm, u, r), pair_pos(p, sm, u, r + 1),
                               pair_pos(p, sm, u, r + 2), pair_pos(p, sm, u, r + 3));
        }
    } else {
        const float inv = 1.0f / (float)R;
        for (int i = threadIdx.x; i < n * R; i += blockDim.x) {
            const int u = div_small(i, inv);
            p.recv_pos[(size_t)t0 * R + i] = pair_pos(p, sm, u, i - u * R);
        }
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

__host__ __device__ size_t matrix_words(int wdt, int ld)
{
    return ((size_t)wdt * ld + 3) & ~(size_t)3;
}

// How CTA totals reach the global scan: one CTA; a thread-block cluster
// (distributed shared memory); a grid (sums already in sm.tot / sm.low).
constexpr int kModeSingle = 0, kModeCluster = 1, kModeGrid = 2;

// Cluster exchange of the CTA totals in sm.tot (and sm.misc), then one packed
// 64-bit block scan: writes cnt / off / totals (CTA 0) and this CTA's first
// row per expert and rank into sm.base.  In grid mode sm.tot already holds
// the grid totals and sm.low the totals of the CTAs below this one, and
// totals[2..3] are left to the grid's last CTA.  Ends without a barrier.
template <int MODE>
__device__ void global_offsets(const LayoutParams &p, const Smem &sm, int crank, int csize)
{
    constexpr bool CLUSTER = MODE == kModeCluster;
    const int tid = threadIdx.x;
    const int E = p.E, R = p.R;
    const int W = E + R + 2;
    // ---- cluster exchange: push this CTA's totals into row crank of every
    // CTA's table (distributed shared memory stores), then read locally
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
        for (int i = tid; i < W; i += blockDim.x) {
            const int v = i < E + R ? sm.tot[i] : sm.misc[i - E - R];
            for (int c = 0; c < csize; ++c)
                cluster.map_shared_rank(sm.all_tot, c)[(size_t)crank * W + i] = v;
        }
        cluster.sync();
    }

    // ---- global exclusive scans (one packed 64-bit block scan), bases
    {
        // this CTA's totals sum over the cluster: all CTAs (glob) and the
        // CTAs below this one (lower), read from the local table
        auto sums = [&](int i, int &g, int &lo) {
            if (MODE == kModeGrid) {
                g = sm.tot[i];
                lo = sm.low[i];
                return;
            }
            if (!CLUSTER) {
                g = sm.tot[i];
                lo = 0;
                return;
            }
            g = 0;
            lo = 0;
            for (int c = 0; c < csize; ++c) {
                const int v = sm.all_tot[(size_t)c * W + i];
                g += v;
                lo += c < crank ? v : 0;
            }
        };
        const int per = (E + (int)blockDim.x - 1) / (int)blockDim.x;
        int glob[kMaxPer], lower[kMaxPer];
        unsigned int contrib_e = 0;
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            const int e = tid * per + q;
            glob[q] = lower[q] = 0;
            if (q < per && e < E) {
                sums(e, glob[q], lower[q]);
                contrib_e += glob[q];
            }
        }
        int glob_r = 0, lower_r = 0;
        if (tid < R) sums(E + tid, glob_r, lower_r);
        unsigned long long total;
        const unsigned long long ex = block_exclusive_scan64(
            ((unsigned long long)contrib_e << 32) | (unsigned)glob_r, sm.scan, &total);
        unsigned int run = (unsigned int)(ex >> 32);
#pragma unroll
        for (int q = 0; q < kMaxPer; ++q) {
            const int e = tid * per + q;
            if (q < per && e < E) {
                sm.base[e] = (int)run + lower[q];
                if (crank == 0) {
                    p.cnt_e[e] = glob[q];
                    p.off_e[e] = (int)run;
                }
                run += glob[q];
            }
        }
        if (tid < R) {
            const int off_r = (int)(unsigned int)(ex & 0xffffffffull);
            sm.base[E + tid] = off_r + lower_r;
            if (crank == 0) {
                p.cnt_r[tid] = glob_r;
                p.off_r[tid] = off_r;
            }
        }
        if (tid == 0 && crank == 0) {
            const int n_route = (int)(total >> 32);
            const int n_recv = (int)(total & 0xffffffffull);
            int errc = sm.misc[0], nr = sm.misc[1];
            if (CLUSTER) {
                errc = 0;
                nr = 0;
                for (int c = 0; c < csize; ++c) {
                    errc |= sm.all_tot[(size_t)c * W + E + R];
                    nr += sm.all_tot[(size_t)c * W + E + R + 1];
                }
            }
            p.off_e[E] = n_route;
            p.off_r[R] = n_recv;
            p.totals[0] = n_route;
            p.totals[1] = n_recv;
            if (MODE != kModeGrid) {
                p.totals[2] = nr;
                p.totals[3] = errc ? (int32_t)EP_DEVERR_BAD_INDEX : 0;
            }
        }
    }
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
    }

    const int W = E + R + 2;
    const int wdt = p.wde + p.wdr;
    Smem sm;
    sm.M = reinterpret_cast<uint32_t *>(smem);
    sm.hit = reinterpret_cast<unsigned long long *>(smem + matrix_words(wdt, p.ld));
    sm.scan = sm.hit + p.tch;
    sm.codes = reinterpret_cast<int32_t *>(sm.scan + 34);
    sm.tot = sm.codes + (size_t)p.tch * p.k;
    sm.base = sm.tot + E + R;
    sm.all_tot = sm.base + E + R;
    sm.misc = sm.all_tot + (size_t)csize * W;

    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    const int c0 = min(T, crank * p.tpc);
    const int nt = min(T, c0 + p.tpc) - c0;
    const int nchunks = (nt + p.tch - 1) / p.tch;
    bool bad = false;
    int nreal = 0;

    // prologue in shared memory only, so it may overlap the previous kernel
    if (tid < 2) sm.misc[tid] = 0;
    if (nchunks <= 1) {
        zero_words(sm.M, wdt * p.ld);
    } else {
        for (int i = tid; i < E + R; i += blockDim.x) sm.tot[i] = 0;
    }
    __syncthreads();
    // peers write into this CTA's shared memory only once every CTA runs
    if (CLUSTER) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    pdl_wait_previous();
    // the dependent grid (normally the dispatch) launches only now, when
    // every kernel before this one has completed: it may then read the
    // batch's inputs (x, topk_idx) before its own wait.  For the grid
    // schedule this also means dependents start only once every CTA of this
    // grid is resident.
    pdl_launch_dependents();

    if (nchunks <= 1) {
        nreal = build_tokens(p, idx, c0, nt, sm, false, &bad);
        __syncthreads();
        row_scan(p, sm, nt);
    } else {
        nreal = build_tokens(p, idx, c0, nt, sm, true, &bad);
    }
    if (__any_sync(kFull, bad) && (tid & 31) == 0) atomicOr(&sm.misc[0], 1);
    if (nreal) atomicAdd(&sm.misc[1], nreal);
    __syncthreads();

    global_offsets<CLUSTER ? kModeCluster : kModeSingle>(p, sm, crank, csize);
    __syncthreads();

    // ---- positions
    if (nchunks <= 1) {
        place_tokens(p, sm, c0, nt);
        return;
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        const int t0 = c0 + ch * p.tch;
        const int n = min(p.tch, c0 + nt - t0);
        zero_words(sm.M, wdt * p.ld);
        __syncthreads();
        bool b2 = false;
        build_tokens(p, idx, t0, n, sm, false, &b2);
        __syncthreads();
        row_scan(p, sm, n);  // tot <- this chunk's row sums
        __syncthreads();
        place_tokens(p, sm, t0, n);
        __syncthreads();
        for (int i = tid; i < E + R; i += blockDim.x) sm.base[i] += sm.tot[i];
        __syncthreads();
    }
}

// ------------------------------------------------------ warp-chunk schedule
//
// A warp takes tpw = floor(32 / k) whole tokens, one lane per route in
// (token, slot) order, so the warp's routes form one chunk of the CTA's
// tokens.  Inside the warp, lanes with equal experts are found with one
// ballot per bit of the expert (match_bits): a route's rank among the warp's
// earlier routes to its expert (from earlier tokens and from earlier slots of
// its own token alike) is the population count of its group below its lane,
// and the group's lowest lane stores the group size into the warp's row of a
// chunk x (expert | rank) count table of 16-bit counts.  The same on the
// rank marks the first route of each (token, rank) pair (no lower lane of
// its token has its rank) and ranks those first routes.  One thread per
// table word (two 16-bit columns) then rewrites its column as an exclusive
// prefix over the chunks, so that
//     pos = base[e] + prefix[chunk][e] + rank in warp
// and the same for recv_pos with the rank columns; base comes from the
// cluster exchange and global scan shared with the count-matrix schedule.
// Each lane keeps its routes in registers (one per pass of the CTA's warps
// over its tokens), so nothing walks the tokens serially.  The CTA has few
// warps (8 or 16, 32 only beyond 64 chunks): the phases are short and
// separated by barriers, and every barrier and every shared-memory phase is
// cheaper with fewer warps.

// Lanes of the warp whose `key` equals this lane's, among `active` lanes;
// `bits` covers every key value.  One ballot per bit (match.any is a slow
// instruction on this part).
__device__ __forceinline__ unsigned match_bits(unsigned key, int bits, unsigned active)
{
    unsigned m = active;
    for (int b = 0; b < bits; ++b) {
        const bool set = (key >> b) & 1u;
        const unsigned bb = __ballot_sync(kFull, set);
        m &= set ? bb : ~bb;
    }
    return m;
}

__host__ __device__ size_t warp_table_words(int nch, int wt)
{
    return ((size_t)nch * wt + 3) & ~(size_t)3;
}

// Per-lane state of the warp-chunk schedule, one entry per pass of the
// CTA's warps over its tokens.
template <int PASSES>
struct WarpRoutes {
    int ex[PASSES];    // expert of the route, -1 for none
    int re_e[PASSES];  // rank among the warp's earlier routes to that expert
    int rk[PASSES];    // rank of the (token, rank) pair this route opens, -1 if none
    int re_r[PASSES];  // rank among the warp's earlier pairs of that rank
    int tl, j;         // token within the warp's chunk, slot
};

// Count phase of the warp-chunk schedule over tokens [c0, c0 + nt) (the
// table `tab` is zero, sm.misc cleared, and the previous kernel waited for):
// fills this CTA's recv_pos rows with -1, matches routes within each warp,
// writes the chunk x (expert | rank) table, turns every column into its
// exclusive prefix over chunks and leaves the CTA totals in sm.tot[E + R],
// the bad-index flag in sm.misc[0] and the real-token count in sm.misc[1].
// Ends with a barrier.
template <typename IdxT, int PASSES>
__device__ __forceinline__ void warp_count(const LayoutParams &p, uint32_t *tab, const Smem &sm,
                                           int c0, int nt, WarpRoutes<PASSES> &wr)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int NW = blockDim.x >> 5;
    const int E = p.E, R = p.R, k = p.k, tpw = p.tpw;
    const int wt = p.tstr >> 1;
    const int nuse = (nt + tpw - 1) / tpw;  // chunks holding tokens
    const IdxT *idx = static_cast<const IdxT *>(p.idx);

    const int tl = div_small(lane, p.inv_k);  // token of this lane within its chunk
    const int j = lane - tl * k;              // slot
    wr.tl = tl;
    wr.j = j;
    const unsigned lt = lanemask_lt();
    IdxT raw[PASSES];
#pragma unroll
    for (int q = 0; q < PASSES; ++q) {
        const int u = (q * NW + wid) * tpw + tl;
        raw[q] = (tl < tpw && u < nt) ? idx[(size_t)(c0 + u) * k + j] : (IdxT)-1;
    }
    // (token, rank) pairs nobody reaches read -1: fill this CTA's rows first
    if ((R & 3) == 0) {
        int4 *dst = reinterpret_cast<int4 *>(p.recv_pos + (size_t)c0 * R);
        for (int i = tid; i < (nt * R) >> 2; i += blockDim.x) dst[i] = make_int4(-1, -1, -1, -1);
    } else {
        for (int i = tid; i < nt * R; i += blockDim.x) p.recv_pos[(size_t)c0 * R + i] = -1;
    }

    bool bad = false;
    int nreal = 0;
    const unsigned kmask = k == 32 ? kFull : ((1u << k) - 1u);
    const unsigned tokmask = tl < tpw ? kmask << (tl * k) : 0u;  // lanes of this lane's token
#pragma unroll
    for (int q = 0; q < PASSES; ++q) {
        const int c = q * NW + wid;
        const long long ev = (long long)raw[q];
        bad |= (ev < -1 || ev >= E);
        const bool v = ev >= 0 && ev < E;
        const int e = v ? (int)ev : 0;
        const int r = v ? rank_of(e, p.inv_epr) : 0;
        const unsigned vb = __ballot_sync(kFull, v);
        const unsigned pe = match_bits((unsigned)e, p.bits_e, vb);
        const unsigned pr = match_bits((unsigned)r, p.bits_r, vb);
        const bool first = v && !(pr & tokmask & lt);
        const unsigned pf = pr & __ballot_sync(kFull, first);
        uint16_t *row = reinterpret_cast<uint16_t *>(tab + (size_t)c * wt);
        if (v && !(pe & lt)) row[e] = (uint16_t)__popc(pe);
        if (first && !(pf & lt)) row[E + r] = (uint16_t)__popc(pf);
        nreal += j == 0 && (vb & tokmask) != 0u;
        wr.ex[q] = v ? e : -1;
        wr.re_e[q] = __popc(pe & lt);
        wr.rk[q] = first ? r : -1;
        wr.re_r[q] = __popc(pf & lt);
    }
    __syncthreads();

    // exclusive prefix of every table column over the chunks (two packed
    // 16-bit columns per word add independently); the sums are the CTA totals
    for (int w = tid; w < wt; w += blockDim.x) {
        uint32_t run = 0;
        for (int c = 0; c < nuse; c += 8) {
            uint32_t v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = c + i < nuse ? tab[(size_t)(c + i) * wt + w] : 0u;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (c + i < nuse) tab[(size_t)(c + i) * wt + w] = run;
                run += v[i];
            }
        }
        if (2 * w < E + R) sm.tot[2 * w] = (int32_t)(run & 0xffffu);
        if (2 * w + 1 < E + R) sm.tot[2 * w + 1] = (int32_t)(run >> 16);
    }
    if (__any_sync(kFull, bad) && lane == 0) atomicOr(&sm.misc[0], 1);
    if (nreal) atomicAdd(&sm.misc[1], nreal);
    __syncthreads();
}

// Placement phase: pos and recv_pos of every route this lane holds, from the
// bases in sm.base, the chunk prefixes in `tab` and the in-warp ranks.
template <int PASSES>
__device__ __forceinline__ void warp_place(const LayoutParams &p, const uint32_t *tab,
                                           const Smem &sm, int c0, int nt,
                                           const WarpRoutes<PASSES> &wr)
{
    const int wid = threadIdx.x >> 5;
    const int NW = blockDim.x >> 5;
    const int E = p.E, R = p.R, k = p.k, tpw = p.tpw;
    const int wt = p.tstr >> 1;
#pragma unroll
    for (int q = 0; q < PASSES; ++q) {
        const int c = q * NW + wid;
        const int u = c * tpw + wr.tl;
        if (wr.tl < tpw && u < nt) {
            const uint16_t *row = reinterpret_cast<const uint16_t *>(tab + (size_t)c * wt);
            const int e = wr.ex[q];
            p.pos[(size_t)(c0 + u) * k + wr.j] =
                e < 0 ? -1 : sm.base[e] + (int)row[e] + wr.re_e[q];
            const int r = wr.rk[q];
            if (r >= 0)
                p.recv_pos[(size_t)(c0 + u) * R + r] =
                    sm.base[E + r] + (int)row[E + r] + wr.re_r[q];
        }
    }
}

template <typename IdxT, bool CLUSTER, int PASSES>
__global__ void __launch_bounds__(1024, 1) layout_warp_kernel(LayoutParams p)
{
    extern __shared__ __align__(16) int32_t smem[];
    const int tid = threadIdx.x;
    const int E = p.E, R = p.R, T = p.T, tpw = p.tpw;

    int crank = 0, csize = 1;
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        crank = (int)cluster.block_rank();
        csize = (int)cluster.num_blocks();
    }
    const int W = E + R + 2;
    const int wt = p.tstr >> 1;  // table row length in 32-bit words
    const int nch_max = (p.tpc + tpw - 1) / tpw;

    uint32_t *tab = reinterpret_cast<uint32_t *>(smem);  // [chunks][wt]
    Smem sm;
    sm.M = nullptr;
    sm.codes = nullptr;
    sm.hit = nullptr;
    sm.low = nullptr;
    sm.scan = reinterpret_cast<unsigned long long *>(smem + warp_table_words(nch_max, wt));
    sm.tot = reinterpret_cast<int32_t *>(sm.scan + 34);
    sm.base = sm.tot + E + R;
    sm.all_tot = sm.base + E + R;
    sm.misc = sm.all_tot + (size_t)csize * W;

    const int c0 = min(T, crank * p.tpc);
    const int nt = min(T, c0 + p.tpc) - c0;
    const int nuse = (nt + tpw - 1) / tpw;  // chunks holding tokens

    // prologue in shared memory only, so it may overlap the previous kernel
    if (tid < 2) sm.misc[tid] = 0;
    zero_words(tab, nuse * wt);
    __syncthreads();
    if (CLUSTER) asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    pdl_wait_previous();
    // the dependent grid (normally the dispatch) launches only now, when
    // every kernel before this one has completed: it may then read the
    // batch's inputs (x, topk_idx) before its own wait.  For the grid
    // schedule this also means dependents start only once every CTA of this
    // grid is resident.
    pdl_launch_dependents();

    WarpRoutes<PASSES> wr;
    warp_count<IdxT, PASSES>(p, tab, sm, c0, nt, wr);
    global_offsets<CLUSTER ? kModeCluster : kModeSingle>(p, sm, crank, csize);
    __syncthreads();
    warp_place<PASSES>(p, tab, sm, c0, nt, wr);
}

// --------------------------------------------------------- grid schedule
//
// For large batches the warp-chunk schedule spreads over many CTAs of one
// ordinary grid -- up to one per SM, each with a few hundred routes -- in
// place of one cluster of at most 16.  CTA totals cannot go through
// distributed shared memory across a grid, so they go through a workspace
// in global memory, with two grid barriers:
//  * count phase as above; the CTA's (expert | rank) totals are stored as
//    one row of packed 16-bit counts; barrier 1;
//  * column scan: CTA b owns the count words b, b + nb, ...; for each, one
//    thread per CTA row loads that row's word, a block scan turns the
//    column into exclusive prefixes over the CTAs, stored in every CTA's
//    prefix row, and the column totals; barrier 2;
//  * every CTA reads its own prefix row and the totals (a few KB), runs the
//    packed global scan and places its routes.
// Each barrier is an arrival counter every CTA adds one to and then waits
// on (bounded: after kGridWaitLimit polls it flags EP_DEVERR_TIMEOUT and goes
// on).  The grid never has more CTAs than SMs, and programmatic launch lets
// dependent grids start only once every CTA of this one has started, so all
// CTAs are resident together.  Bad-index and real-token counts go into two
// more header words; the last CTA to leave writes them to totals[2..3] and
// zeroes the header, so the workspace is clean after every call (its header
// must be zero before the first one).
constexpr int kGridHeader = kGridHeaderWords;  // [0] arrivals 1, [1] departures,
                                               // [2] error bits, [3] real tokens,
                                               // [4] arrivals 2
constexpr long long kGridWaitLimit = 1ll << 21;

__device__ __forceinline__ int ld_acquire_gpu(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// One thread: arrive at the counter and wait (bounded) for all nb CTAs;
// false if the wait gave up (flagged in the header).
__device__ __forceinline__ bool grid_arrive_wait(int32_t *counter, int32_t *flags, int nb)
{
    __threadfence();
    atomicAdd(counter, 1);
    for (long long i = 0; i < kGridWaitLimit; ++i) {
        if (ld_acquire_gpu(counter) >= nb) {
            __threadfence();
            return true;
        }
        __nanosleep(32);
    }
    atomicOr(flags, (int)EP_DEVERR_TIMEOUT);
    return false;
}

constexpr int kGridMaxThreads = 512;

template <typename IdxT, int PASSES>
__global__ void __launch_bounds__(kGridMaxThreads, 1) layout_grid_kernel(LayoutParams p)
{
    // no static shared memory: the dynamic part may take the whole 227 KB
    extern __shared__ __align__(16) int32_t smem[];
    const int tid = threadIdx.x;
    const int E = p.E, R = p.R, T = p.T, tpw = p.tpw;
    const int nb = (int)gridDim.x, b = (int)blockIdx.x;

    const int wt = p.tstr >> 1;
    const int hs = p.hs;                   // count row length in words (multiple of 4)
    const int ps = (E + R + 3) & ~3;       // prefix row length in words
    const int nch_max = (p.tpc + tpw - 1) / tpw;

    uint32_t *tab = reinterpret_cast<uint32_t *>(smem);  // [chunks][wt]
    Smem sm;
    sm.M = nullptr;
    sm.codes = nullptr;
    sm.hit = nullptr;
    sm.all_tot = nullptr;
    sm.scan = reinterpret_cast<unsigned long long *>(smem + warp_table_words(nch_max, wt));
    sm.tot = reinterpret_cast<int32_t *>(sm.scan + 34);
    sm.base = sm.tot + E + R;
    sm.low = sm.base + E + R;
    sm.misc = sm.low + E + R;  // [0] bad flag, [1] real tokens, [2] a barrier gave up
    int *s_fail = sm.misc + 2;

    const int c0 = min(T, b * p.tpc);
    const int nt = min(T, c0 + p.tpc) - c0;
    const int nuse = (nt + tpw - 1) / tpw;

    if (tid < 3) sm.misc[tid] = 0;
    zero_words(tab, nuse * wt);
    __syncthreads();
    pdl_wait_previous();
    // the dependent grid (normally the dispatch) launches only now, when
    // every kernel before this one has completed: it may then read the
    // batch's inputs (x, topk_idx) before its own wait.  For the grid
    // schedule this also means dependents start only once every CTA of this
    // grid is resident.
    pdl_launch_dependents();

    WarpRoutes<PASSES> wr;
    warp_count<IdxT, PASSES>(p, tab, sm, c0, nt, wr);

    int32_t *hdr = p.work;
    uint32_t *rows = reinterpret_cast<uint32_t *>(p.work + kGridHeader);  // [nb][hs]
    uint32_t *pref = rows + (size_t)nb * hs;                               // [nb][ps]
    uint32_t *gtot = pref + (size_t)nb * ps;                               // [ps]

    // ---- this CTA's totals as one row of packed 16-bit counts; barrier 1
    for (int w = tid; w < hs; w += blockDim.x) {
        const uint32_t lo = 2 * w < E + R ? (uint32_t)sm.tot[2 * w] : 0u;
        const uint32_t hi = 2 * w + 1 < E + R ? (uint32_t)sm.tot[2 * w + 1] : 0u;
        rows[(size_t)b * hs + w] = lo | (hi << 16);
    }
    __syncthreads();
    if (tid == 0) {
        if (sm.misc[0]) atomicOr(&hdr[2], (int)EP_DEVERR_BAD_INDEX);
        if (sm.misc[1]) atomicAdd(&hdr[3], sm.misc[1]);
        if (!grid_arrive_wait(&hdr[0], &hdr[2], nb)) *s_fail = 1;
    }
    __syncthreads();

    // ---- column scan of the words this CTA owns, over the CTAs; barrier 2
    for (int w = b; 2 * w < E + R; w += nb) {
        const uint32_t v = tid < nb ? __ldcg(rows + (size_t)tid * hs + w) : 0u;
        unsigned long long total;
        const unsigned long long ex = block_exclusive_scan64(
            ((unsigned long long)(v >> 16) << 32) | (v & 0xffffu), sm.scan, &total);
        if (tid < nb) {
            pref[(size_t)tid * ps + 2 * w] = (uint32_t)(ex & 0xffffffffull);
            if (2 * w + 1 < E + R) pref[(size_t)tid * ps + 2 * w + 1] = (uint32_t)(ex >> 32);
        }
        if (tid == 0) {
            gtot[2 * w] = (uint32_t)(total & 0xffffffffull);
            if (2 * w + 1 < E + R) gtot[2 * w + 1] = (uint32_t)(total >> 32);
        }
        __syncthreads();  // sm.scan is reused by the next word
    }
    __syncthreads();
    if (tid == 0 && !grid_arrive_wait(&hdr[4], &hdr[2], nb)) *s_fail = 1;
    __syncthreads();

    // ---- this CTA's bases: its prefix row and the totals
    for (int c = tid; c < E + R; c += blockDim.x) {
        sm.tot[c] = (int32_t)__ldcg(gtot + c);
        sm.low[c] = (int32_t)__ldcg(pref + (size_t)b * ps + c);
    }
    __syncthreads();
    // this CTA no longer reads the workspace: leave (the last one out
    // publishes the header's counts and zeroes it)
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(&hdr[1], 1) == nb - 1) {
            p.totals[2] = atomicExch(&hdr[3], 0);
            p.totals[3] = atomicExch(&hdr[2], 0);
            atomicExch(&hdr[0], 0);
            atomicExch(&hdr[4], 0);
            atomicExch(&hdr[1], 0);
        }
    }

    global_offsets<kModeGrid>(p, sm, b, nb);
    __syncthreads();
    if (*s_fail) {  // the sums are not trustworthy: no route gets a row
        for (int i = tid; i < nt * p.k; i += blockDim.x) p.pos[(size_t)c0 * p.k + i] = -1;
        return;
    }
    warp_place<PASSES>(p, tab, sm, c0, nt, wr);
}

// ------------------------------------------------------------------- host

struct Geometry {
    int csize, tpc, tch, ld, wde, wdr;
    size_t smem;
};

size_t fixed_bytes(int E, int R, int csize)
{
    // scan scratch, tot, base, the cluster's totals table, misc
    return 34 * 8 +
           sizeof(int32_t) * (2 * (size_t)(E + R) + (size_t)csize * (E + R + 2) + 2) + 16;
}

// Cluster size and chunk width for a layout problem.
Geometry plan(int T, int k, int E, int R, int csize)
{
    Geometry g;
    g.wde = (E + 1) / 2;
    g.wdr = (R + 1) / 2;
    const int wdt = g.wde + g.wdr;
    // the totals table grows with the cluster: shrink the cluster if the
    // fixed part would leave room for fewer than 32 tokens per chunk
    while (csize > 1 && fixed_bytes(E, R, csize) + ((size_t)wdt * 32 + 4) * 4 + 32 * 8 +
                            (size_t)32 * k * 4 > (size_t)kMaxDynSmem)
        csize >>= 1;
    g.csize = csize;
    g.tpc = (T + csize - 1) / csize;
    const size_t fixed = fixed_bytes(E, R, csize);
    // shared memory for a chunk of w tokens: matrix rows of an odd length
    // >= w, rank masks, route codes
    auto bytes = [&](int w) {
        return ((size_t)wdt * (w | 1) + 4) * 4 + (size_t)w * 8 + (size_t)w * k * 4 + fixed;
    };
    // the CTA's tokens in one chunk when they fit: at most one token per
    // thread, 16-bit counts, shared memory
    int tch = g.tpc < 1 ? 1 : g.tpc;
    if (tch > 1024) tch = 1024;
    if (tch > 65535 / k) tch = 65535 / k;
    while (tch > 1 && bytes(tch) > (size_t)kMaxDynSmem) tch = tch > 64 ? tch - 32 : tch - 1;
    g.tch = tch;
    g.ld = tch | 1;
    g.smem = bytes(tch);
    return g;
}

// Warp-chunk geometry: tokens per warp and per CTA, passes, table row
// length, shared memory; false when the table does not fit or more than
// four passes would be needed (the count-matrix schedule covers those).
struct WarpGeometry {
    int csize, tpc, tpw, passes, threads, tstr;
    size_t smem;
};

int bits_for(int n)  // bits of the largest value below n (at least 1)
{
    int b = 1;
    while ((1 << b) < n) ++b;
    return b;
}

bool plan_warp(int T, int k, int E, int R, int csize, WarpGeometry *g)
{
    g->tpw = 32 / k;
    g->tstr = (E + R + 1) & ~1;
    // the global scan gives each thread at most four experts, and one rank
    int min_threads = (E + 3) / 4 > R ? (E + 3) / 4 : R;
    min_threads = ((min_threads + 31) / 32) * 32;
    for (;; csize >>= 1) {
        g->csize = csize;
        g->tpc = (T + csize - 1) / csize;
        const int nch = (g->tpc + g->tpw - 1) / g->tpw;
        // warps (8, 16 or 32): at most two passes up to 16 warps, then at
        // most four (measured: decode's 32 chunks run faster as 16 warps x 2
        // passes than as 8 x 4; prefill's 64 faster as 16 x 4 than 32 x 2)
        int warps = 8;
        while (warps < 16 && nch > 2 * warps) warps *= 2;
        while (warps < 32 && nch > 4 * warps) warps *= 2;
        if (warps * 32 < min_threads) warps = (min_threads + 31) / 32;
        const int passes = (nch + warps - 1) / warps;
        g->threads = warps * 32;
        g->passes = passes <= 1 ? 1 : passes <= 2 ? 2 : 4;
        g->smem = warp_table_words(nch, g->tstr >> 1) * 4 + fixed_bytes(E, R, csize);
        if (passes <= 4 && g->smem <= (size_t)kMaxDynSmem) return true;
        if (csize == 1 || passes > 4) return false;
    }
}

// Grid-schedule geometry: CTAs of ~kGridRoutesPerCta routes (at most one
// per SM), warps and passes as in the warp-chunk schedule; false when fewer
// than two CTAs would be used or shared memory does not suffice.
bool plan_grid(int T, int k, int E, int R, int nsm, WarpGeometry *g, int *hs)
{
    const long long routes = (long long)T * k;
    int nb = grid_max_ctas(routes);
    if (nb > nsm) nb = nsm;
    if (nb < 2) return false;
    g->tpw = 32 / k;
    g->tstr = (E + R + 1) & ~1;
    g->tpc = (T + nb - 1) / nb;
    g->csize = (T + g->tpc - 1) / g->tpc;  // CTAs that hold tokens
    if (g->csize < 2) return false;
    const int nch = (g->tpc + g->tpw - 1) / g->tpw;
    int min_threads = (E + 3) / 4 > R ? (E + 3) / 4 : R;
    min_threads = ((min_threads + 31) / 32) * 32;
    int warps = 8;
    while (warps * 32 < kGridMaxThreads && nch > 4 * warps) warps *= 2;
    if (warps * 32 < min_threads) warps = (min_threads + 31) / 32;
    if (warps * 32 > kGridMaxThreads) return false;
    const int passes = (nch + warps - 1) / warps;
    if (passes > 4) return false;
    g->passes = passes <= 1 ? 1 : passes <= 2 ? 2 : 4;
    g->threads = warps * 32;
    if (g->threads < g->csize) return false;  // the column scan takes one thread per CTA
    *hs = grid_row_words(E, R);
    g->smem = warp_table_words(nch, g->tstr >> 1) * 4 + 34 * 8 +
              sizeof(int32_t) * (3 * (size_t)(E + R) + 3);
    return g->smem <= (size_t)kMaxDynSmem;
}

using LayoutKernel = void (*)(LayoutParams);

template <typename IdxT, bool CLUSTER>
LayoutKernel warp_kernel(int passes)
{
    return passes == 1   ? layout_warp_kernel<IdxT, CLUSTER, 1>
           : passes == 2 ? layout_warp_kernel<IdxT, CLUSTER, 2>
                         : layout_warp_kernel<IdxT, CLUSTER, 4>;
}

// largest number of co-resident clusters of `csize` CTAs of `fn` (0 when a
// cluster of that size with that much shared memory cannot be placed)
int max_clusters(LayoutKernel fn, int csize, int threads, size_t smem, int dev)
{
    struct Entry {
        LayoutKernel fn;
        int dev, csize, threads;
        size_t smem;
        int result;
    };
    static Entry cache[128];
    static int n_cache = 0;
    std::lock_guard<std::mutex> lock(launcher_mutex());
    for (int i = 0; i < n_cache; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev && cache[i].csize == csize &&
            cache[i].threads == threads && cache[i].smem == smem)
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
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (n_cache < 128) cache[n_cache++] = Entry{fn, dev, csize, threads, smem, n};
    return n;
}

template <typename IdxT>
LayoutKernel grid_kernel(int passes)
{
    return passes == 1   ? layout_grid_kernel<IdxT, 1>
           : passes == 2 ? layout_grid_kernel<IdxT, 2>
                         : layout_grid_kernel<IdxT, 4>;
}

template <typename IdxT>
cudaError_t set_attributes_once(int dev)
{
    static std::atomic<unsigned> done{0};  // per device (up to 32)
    if (dev < 32 && (done.load() & (1u << dev))) return cudaSuccess;
    const LayoutKernel single[] = {layout_kernel<IdxT, false>, warp_kernel<IdxT, false>(1),
                                   warp_kernel<IdxT, false>(2), warp_kernel<IdxT, false>(4)};
    const LayoutKernel clustered[] = {layout_kernel<IdxT, true>, warp_kernel<IdxT, true>(1),
                                      warp_kernel<IdxT, true>(2), warp_kernel<IdxT, true>(4)};
    cudaError_t err = cudaSuccess;
    const LayoutKernel grid[] = {grid_kernel<IdxT>(1), grid_kernel<IdxT>(2), grid_kernel<IdxT>(4)};
    for (LayoutKernel fn : grid)
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxDynSmem);
    for (LayoutKernel fn : single)
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxDynSmem);
    for (LayoutKernel fn : clustered) {
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxDynSmem);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    }
    if (err == cudaSuccess && dev < 32) done.fetch_or(1u << dev);
    return err;
}

// variant: 0 = warp chunks where they fit, else the grid schedule where it
// fits, else the count matrix; 1 = warp chunks (cudaErrorNotSupported
// where they do not fit); 2 = count matrix; 3 = grid schedule
// (cudaErrorNotSupported without a workspace or where it does not fit)
template <typename IdxT>
cudaError_t launch_layout_t(const LayoutParams &p0, int variant, cudaStream_t s)
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
    // automatic: the warp-chunk cluster where it fits (measured faster than
    // the grid schedule at 4096 x top-8: its two grid barriers cost more
    // than the cluster's exchange saves), then the grid schedule, then the
    // count matrix
    bool grid = variant == 3;
    if (variant == 0 && p.work) {
        WarpGeometry gw;
        grid = !plan_warp(p.T, p.k, p.E, p.R, csize, &gw);
    }
    if (grid) {
        WarpGeometry g;
        int hs = 0;
        if (p.work && plan_grid(p.T, p.k, p.E, p.R, sm_count(dev), &g, &hs)) {
            p.tpc = g.tpc;
            p.tpw = g.tpw;
            p.tstr = g.tstr;
            p.hs = hs;
            p.inv_k = 1.0f / (float)p.k;
            p.bits_e = bits_for(p.E);
            p.bits_r = bits_for(p.R);
            return launch_pdl(grid_kernel<IdxT>(g.passes), dim3(g.csize), dim3(g.threads),
                              g.smem, s, p);
        }
        if (variant == 3) return cudaErrorNotSupported;
    }

    if (variant != 2) {
        WarpGeometry g;
        bool ok = plan_warp(p.T, p.k, p.E, p.R, csize, &g);
        while (ok && g.csize > 1 &&
               max_clusters(warp_kernel<IdxT, true>(g.passes), g.csize, g.threads, g.smem,
                            dev) == 0)
            ok = plan_warp(p.T, p.k, p.E, p.R, g.csize > 8 ? 8 : g.csize >> 1, &g);
        if (ok) {
            p.tpc = g.tpc;
            p.tpw = g.tpw;
            p.tstr = g.tstr;
            p.inv_k = 1.0f / (float)p.k;
            p.bits_e = bits_for(p.E);
            p.bits_r = bits_for(p.R);
            if (g.csize == 1)
                return launch_pdl(warp_kernel<IdxT, false>(g.passes), dim3(1), dim3(g.threads),
                                  g.smem, s, p);
            return launch_pdl(warp_kernel<IdxT, true>(g.passes), dim3(g.csize), dim3(g.threads),
                              g.smem, s, p, g.csize);
        }
        if (variant == 1) return cudaErrorNotSupported;
    }

    Geometry g = plan(p.T, p.k, p.E, p.R, csize);
    while (g.csize > 1 &&
           max_clusters(layout_kernel<IdxT, true>, g.csize, 1024, g.smem, dev) == 0)
        g = plan(p.T, p.k, p.E, p.R, g.csize > 8 ? 8 : g.csize >> 1);
    p.tpc = g.tpc;
    p.tch = g.tch;
    p.ld = g.ld;
    p.wde = g.wde;
    p.wdr = g.wdr;
    if (g.csize == 1)
        return launch_pdl(layout_kernel<IdxT, false>, dim3(1), dim3(1024), g.smem, s, p);
    return launch_pdl(layout_kernel<IdxT, true>, dim3(g.csize), dim3(1024), g.smem, s, p,
                      g.csize);
}

}  // namespace

cudaError_t launch_layout(const LayoutParams &p, int idx_bits, int variant, cudaStream_t s)
{
    return idx_bits == 64 ? launch_layout_t<long long>(p, variant, s)
                          : launch_layout_t<int>(p, variant, s);
}

}  // namespace epx
