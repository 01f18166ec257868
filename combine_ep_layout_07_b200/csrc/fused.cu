// Routing layout and dispatch + expand in one launch, for small batches.
//
// What is computed is exactly ep_layout followed by ep_dispatch_expand: the
// layout ("handle") of DeepEP issue #760's Reproduction (dispatch returns
// it, combine takes it back) and the copies of DeepEP issue #48 (a token is
// received once per destination rank, then duplicated once per expert).  At
// a handful of tokens -- the regime of the issue #760 report -- the separate
// layout launch is a chain of dependent steps (load, count, exchange, scan,
// place) that the dispatch must wait for; here that chain is removed:
//
//  * CTA (token t, chunk c) first issues every load it needs: its token's
//    k routes, its chunk of x[t] and the routes of the whole batch (read
//    coalesced into a shared-memory table of experts, one row per token,
//    with each token's set of ranks OR-ed together on the way), so the DRAM
//    latency of x overlaps the count;
//  * it derives its own token's rows by counting over all T*k routes.  In
//    (expert, token, slot) order the row of route (t, j) with expert e is
//    the number of valid routes before it:
//        pos[t, j] = #{(t', j') : e' < e, or e' == e and t' < t}
//                  + #{j' < j : e_{t, j'} == e},
//    i.e. the routes of token t' with e' < e + [t' < t], plus the earlier
//    slots of t with the same expert.  Likewise a (token, rank) pair's row
//    is the number of pairs (t', r') with r' < r + [t' < t]:
//    popcount(M' & lowmask(r + [t' < t])) summed over tokens t', M' being
//    t''s set of ranks.  Each thread owns one query (a slot or a rank of
//    token t) and a subset of the tokens, so the count has no cross-lane
//    dependency until one shuffle sum at the end;
//  * warp 0 adds the warps' counts and lists the destination rows; the CTA
//    stores its chunk (staged in shared memory) to every destination row --
//    a long chunk as one TMA bulk store per row, a short one with the (row,
//    vector) pairs spread over all threads so that a chunk of a few vectors
//    still uses the whole CTA; chunk 0 of token t writes pos[t, :] and
//    recv_pos[t, :];
//  * one extra CTA writes what no token CTA owns: the per-expert and per-rank
//    counts and exclusive scans, the totals and the error word.
//
// No CTA waits for another, so there is no grid-wide barrier.  The count
// costs every CTA work in proportion to T*k; measured on B200 the one
// launch is faster than the layout and dispatch kernels from one token up
// to about two thousand routes (EPX_FUSED_AUTO_MIN_ROUTES to
// EPX_FUSED_AUTO_MAX_ROUTES), which is where the automatic choice takes it.
// Rows beyond a caller's capacity are skipped; the summary CTA flags them
// (a row beyond the capacity exists exactly when the total exceeds it).
#include "epx_internal.cuh"

namespace epx {
namespace {

// Threads per CTA.  Measured on B200 (amortised steps, L2 flushed): 256
// against 128 took decode from 20.3 to 20.2 us and DP compact from 20.4 to
// 20.3 us (tiny 6.6 -> 6.7 us); 512 was no better than 128.  The kernel is
// bound by instruction latency (about 11 cycles per issued instruction with
// two warps per scheduler at 128 threads), not by its loads.
#ifndef EPX_FUSED_THREADS
#define EPX_FUSED_THREADS 256
#endif
constexpr int kFusedThreads = EPX_FUSED_THREADS;
// chunks of at least this many 16-byte vectors are stored with TMA bulk
// copies, one per destination row (measured on B200, amortised, against the
// spread register stores: decode -0.08 and -0.06 us, DP compact -0.15 and
// +0.06 us on two boxes, i.e. about even; at 32-vector chunks, low batch
// T = 1, 6.7 -> 6.9 us, so short chunks keep the spread register stores)
constexpr int kBulkMinVectors = 128;
constexpr int kFusedWarps = kFusedThreads / 32;

__device__ __forceinline__ int rank_of_e(int e, float inv_epr)
{
    // floor(e / epr), exact for e < 2^22 ((e + 1/2) / epr is at least
    // 1/(2 epr) away from an integer, more than two fp32 roundings move it)
    return __float2int_rd(__fmul_rn(__fadd_rn((float)e, 0.5f), inv_epr));
}

__device__ __forceinline__ unsigned long long lowmask64(int n)
{
    return n >= 64 ? ~0ull : ((1ull << n) - 1ull);
}

template <typename IdxT>
__device__ __forceinline__ int load_expert(const IdxT *idx, size_t i, int E, bool *bad)
{
    const long long e = (long long)idx[i];
    *bad |= (e < -1 || e >= E);
    return (e >= 0 && e < E) ? (int)e : -1;
}

// ----------------------------------------------------------- summary CTA
// cnt_e / off_e / cnt_r / off_r / totals for the whole batch.  A warp takes
// floor(32 / k) whole tokens per step, one lane per route (one coalesced
// load per lane, the steps independent of each other); the first route of
// every (token, rank) pair -- no lower lane of its token has its rank, found
// with one ballot per bit of the rank -- counts for the rank.  Expert counts
// are 16-bit halves of 32-bit shared words (a count is at most T*k, which the
// launcher keeps below 2^16).
__device__ __forceinline__ unsigned same_key_lanes(unsigned key, int bits, unsigned active)
{
    unsigned m = active;
    for (int b = 0; b < bits; ++b) {
        const bool set = (key >> b) & 1u;
        const unsigned bb = __ballot_sync(kFull, set);
        m &= set ? bb : ~bb;
    }
    return m;
}

template <typename IdxT>
__device__ void summary_cta(const FusedParams &p, uint32_t *smem)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int E = p.E, R = p.R, k = p.k;
    const int wde = (E + 1) >> 1;
    uint32_t *he = smem;                  // [wde] packed 16-bit expert counts
    int *hr = reinterpret_cast<int *>(smem + wde);  // [R] rank counts
    int *misc = hr + R;                   // [0] bad flag, [1] real tokens
    unsigned long long *scan = reinterpret_cast<unsigned long long *>(
        smem + (((size_t)wde + R + 2 + 1) & ~(size_t)1));  // [kFusedWarps + 1]
    for (int i = tid; i < wde; i += kFusedThreads) he[i] = 0u;
    for (int i = tid; i < R; i += kFusedThreads) hr[i] = 0;
    if (tid < 2) misc[tid] = 0;
    __syncthreads();

    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    const int tpw = 32 / k;
    const int tl = lane / k, jl = lane - tl * k;
    const unsigned kmask = k == 32 ? kFull : ((1u << k) - 1u);
    const unsigned tokmask = tl < tpw ? kmask << (tl * k) : 0u;
    const unsigned lt = lanemask_lt();
    int bits_r = 1;
    while ((1 << bits_r) < R) ++bits_r;
    bool bad = false;
    int nreal = 0;
    const int nsteps = (p.T + tpw - 1) / tpw;
    // four steps per iteration: their loads are issued together
    for (int s0 = wid * 4; s0 < nsteps; s0 += kFusedWarps * 4) {
        int ev[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int u = (s0 + a) * tpw + tl;
            ev[a] = (tl < tpw && u < p.T) ? load_expert(idx, (size_t)u * k + jl, E, &bad) : -1;
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int e = ev[a];
            const bool valid = e >= 0;
            const int r = valid ? rank_of_e(e, p.inv_epr) : 0;
            const unsigned vb = __ballot_sync(kFull, valid);
            const unsigned same_r = same_key_lanes((unsigned)r, bits_r, vb) & tokmask;
            if (valid) {
                atomicAdd(&he[e >> 1], 1u << ((e & 1) * 16));
                if (!(same_r & lt)) atomicAdd(&hr[r], 1);
            }
            // the token's first valid route counts it as real
            nreal += valid && !(vb & tokmask & lt);
        }
    }
    if (__any_sync(kFull, bad) && lane == 0) atomicOr(&misc[0], 1);
    const int wr = __reduce_add_sync(kFull, nreal);
    if (lane == 0 && wr) atomicAdd(&misc[1], wr);
    __syncthreads();

    // one packed 64-bit exclusive scan: experts (a contiguous run per
    // thread) in the high half, ranks (one per thread) in the low half
    const int per = (E + kFusedThreads - 1) / kFusedThreads;
    const int e0 = tid * per;
    unsigned int run_e = 0;
    for (int q = 0; q < per; ++q) {
        const int e = e0 + q;
        if (e < E) run_e += (he[e >> 1] >> ((e & 1) * 16)) & 0xffffu;
    }
    const unsigned int cr = tid < R ? (unsigned)hr[tid] : 0u;
    // a rank beyond the first 128 threads cannot occur: R <= 64
    const unsigned long long v = ((unsigned long long)run_e << 32) | cr;
    unsigned long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long n = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) scan[wid] = inc;
    __syncthreads();
    if (tid == 0) {
        unsigned long long s = 0ull;
        for (int w = 0; w < kFusedWarps; ++w) {
            const unsigned long long x = scan[w];
            scan[w] = s;
            s += x;
        }
        scan[kFusedWarps] = s;
    }
    __syncthreads();
    const unsigned long long ex = scan[wid] + inc - v;
    const unsigned long long total = scan[kFusedWarps];
    unsigned int off = (unsigned int)(ex >> 32);
    for (int q = 0; q < per; ++q) {
        const int e = e0 + q;
        if (e < E) {
            const int c = (int)((he[e >> 1] >> ((e & 1) * 16)) & 0xffffu);
            p.cnt_e[e] = c;
            p.off_e[e] = (int)off;
            off += c;
        }
    }
    if (tid < R) {
        p.cnt_r[tid] = (int)cr;
        p.off_r[tid] = (int)(unsigned int)(ex & 0xffffffffull);
    }
    if (tid == 0) {
        const int n_route = (int)(total >> 32);
        const int n_recv = (int)(total & 0xffffffffull);
        p.off_e[E] = n_route;
        p.off_r[R] = n_recv;
        p.totals[0] = n_route;
        p.totals[1] = n_recv;
        p.totals[2] = misc[1];
        int err = misc[0] ? (int)EP_DEVERR_BAD_INDEX : 0;
        if ((int64_t)n_recv > p.recv_cap) err |= (int)EP_DEVERR_RECV_CAP;
        if ((int64_t)n_route > p.exp_cap) err |= (int)EP_DEVERR_EXP_CAP;
        p.totals[3] = err;
    }
}

// ------------------------------------------------------------ token CTAs
//
// Counting: the batch's experts sit in a shared-memory table, one row of
// KM entries per token (INT_MAX for no route), next to each token's set of
// ranks.  Thread (query j, subset s) -- j = tid mod KM, s = tid div KM --
// visits the tokens u = s, s + S, ... (S = threads / KM) and counts, for slot j of its
// own token (expert e_j), the routes of u with expert below e_j + [u < t],
// and for the j-th rank r_j of its own token whether u reaches a rank below
// r_j + [u < t].  Lanes of a warp with the same j are summed by shuffles,
// the warps by warp 0.  Rows are read by all KM threads of a subset at once
// (a shared-memory broadcast); nothing in the count waits on another lane.

template <typename IdxT, int KM, int VPT>
__global__ void __launch_bounds__(kFusedThreads) layout_dispatch_kernel(FusedParams p)
{
    extern __shared__ __align__(16) uint32_t fsmem[];
    __shared__ int s_part[kFusedWarps][64];  // per warp: [0, 32) slot counts, [32, 64) rank counts
    __shared__ int s_rrow[32];
    __shared__ int s_rq[64];                 // the token's ranks in increasing order
    __shared__ uint4 *s_dst[64];
    __shared__ int s_n;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    if (blockIdx.x == 0) {
        summary_cta<IdxT>(p, fsmem);
        return;
    }
    const int b = (int)blockIdx.x - 1;
    const int t = b / p.chunks;
    const int c = b - t * p.chunks;
    const int k = p.k, E = p.E, R = p.R, T = p.T;
    const IdxT *idx = static_cast<const IdxT *>(p.idx);
    // shared memory: the chunk of x[t] [vpc], the experts [T][KM], the rank sets [T]
    uint4 *s_x = reinterpret_cast<uint4 *>(fsmem);
    int *s_e = reinterpret_cast<int *>(s_x + p.vpc);
    unsigned long long *s_m = reinterpret_cast<unsigned long long *>(s_e + T * KM);

    // every load is issued before anything waits on one: this token's
    // routes (one per lane; every warp reads them, so no barrier), its chunk
    // of x[t] and the batch's routes (coalesced, eight per thread at a time)
    long long own = -1;
    if (lane < k) own = (long long)idx[(size_t)t * k + lane];
    const int v0 = c * p.vpc;
    const int nv = min(p.V, v0 + p.vpc) - v0;
    const uint4 *src = p.x + (size_t)t * p.V + v0;
    uint4 val[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int v = tid + u * kFusedThreads;
        if (v < nv) val[u] = ld_nc_v4(src + v);
    }
    // the table: expert of route i = u k + j at s_e[u KM + j] (INT_MAX for
    // no route), and token u's set of ranks.  When k divides 32 a token's
    // routes sit in k aligned lanes of one warp load, and an OR over those
    // lanes (shuffles) gives the set; otherwise each route ORs its rank bit
    // in with a 32-bit shared atomic (64-bit ones were measured slow)
    const bool seg = (32 % k) == 0;
    if (!seg)
        for (int u = tid; u < T; u += kFusedThreads) s_m[u] = 0ull;
    const int nk = T * k;
    for (int i0 = 0; i0 < nk; i0 += 8 * kFusedThreads) {
        long long ev[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int i = i0 + a * kFusedThreads + tid;
            ev[a] = i < nk ? (long long)idx[i] : -1;
        }
        if (!seg && i0 == 0) __syncthreads();  // s_m zeroed (the loads are in flight)
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            if (i0 + a * kFusedThreads >= nk) break;  // the same for every thread
            const int i = i0 + a * kFusedThreads + tid;
            const bool ok = i < nk && ev[a] >= 0 && ev[a] < E;
            const int r = ok ? rank_of_e((int)ev[a], p.inv_epr) : 0;
            // i = u k + j; (i + 1/2) / k is at least 1/(2k) from an integer,
            // far more than the fp32 roundings move it
            const int u = __float2int_rd(__fmul_rn(__fadd_rn((float)i, 0.5f), p.inv_k));
            const int jj = i - u * k;
            if (i < nk) s_e[u * KM + jj] = ok ? (int)ev[a] : 0x7fffffff;
            if (seg) {
                unsigned long long m = ok ? 1ull << r : 0ull;
                for (int off = 1; off < k; off <<= 1) m |= __shfl_xor_sync(kFull, m, off);
                if (i < nk && jj == 0) s_m[u] = m;
            } else if (ok) {
                atomicOr(reinterpret_cast<unsigned int *>(&s_m[u]) + (r >> 5), 1u << (r & 31));
            }
        }
    }
    const int e_mine = (own >= 0 && own < E) ? (int)own : -1;
    const int r_mine = e_mine >= 0 ? rank_of_e(e_mine, p.inv_epr) : -1;
    const unsigned m_lo = __reduce_or_sync(kFull, r_mine >= 0 && r_mine < 32 ? 1u << r_mine : 0u);
    const unsigned m_hi = __reduce_or_sync(kFull, r_mine >= 32 ? 1u << (r_mine - 32) : 0u);
    const unsigned long long m_own = ((unsigned long long)m_hi << 32) | m_lo;
    if (m_own == 0ull) {  // no valid route: nothing to copy, rows of -1
        if (c == 0) {
            for (int j = tid; j < k; j += kFusedThreads) p.pos[(size_t)t * k + j] = -1;
            for (int r = tid; r < R; r += kFusedThreads) p.recv_pos[(size_t)t * R + r] = -1;
        }
        return;
    }
    for (int r = tid; r < R; r += kFusedThreads)
        if ((m_own >> r) & 1ull) s_rq[__popcll((long long)(m_own & lowmask64(r)))] = r;
    __syncthreads();  // s_e, s_m, s_rq complete

    // this thread's queries: slot j of token t (expert eq, -1 for none) and
    // the j-th smallest rank of token t (rq, -1 for none)
    const int j = tid & (KM - 1);
    const int sub = tid / KM;
    constexpr int kSubsets = kFusedThreads / KM;
    int eq = -1;
    if (j < k) {
        const int e = s_e[t * KM + j];
        eq = e == 0x7fffffff ? -1 : e;
    }
    const int nr = __popcll((long long)m_own);
    const int rq = j < nr ? s_rq[j] : -1;
    int n_slot = 0, n_rank = 0;
#pragma unroll 2
    for (int u = sub; u < T; u += kSubsets) {
        const int bt = u < t;
        const int thr = eq + bt;  // eq = -1: no valid expert is below -1 + bt
        const int4 *row = reinterpret_cast<const int4 *>(s_e + u * KM);
#pragma unroll
        for (int q = 0; q < KM / 4; ++q) {
            const int4 w = row[q];
            // entries beyond k are never written: mask them by index
            n_slot += (4 * q + 0 < k && w.x < thr) + (4 * q + 1 < k && w.y < thr) +
                      (4 * q + 2 < k && w.z < thr) + (4 * q + 3 < k && w.w < thr);
        }
        if (rq >= 0) n_rank += __popcll((long long)(s_m[u] & lowmask64(rq + bt)));
    }
#pragma unroll
    for (int off = KM; off < 32; off <<= 1) {
        n_slot += __shfl_xor_sync(kFull, n_slot, off);
        n_rank += __shfl_xor_sync(kFull, n_rank, off);
    }
    if (lane < KM) {
        s_part[wid][lane] = n_slot;
        s_part[wid][32 + lane] = n_rank;
    }
    // the chunk of x into shared memory, for the stores below
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const int v = tid + u * kFusedThreads;
        if (v < nv) s_x[v] = val[u];
    }
    // long chunks go out through the TMA engine, which reads them from
    // shared memory: order these writes for it
    const bool bulk = nv >= kBulkMinVectors;
    if (bulk) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    // warp 0: rows of the token's routes and pairs, destination list
    if (wid == 0) {
        const unsigned lt = lanemask_lt();
        int dup = 0;  // earlier slots of this token with the same expert
        {
            const int4 *row = reinterpret_cast<const int4 *>(s_e + t * KM);
#pragma unroll
            for (int q = 0; q < KM / 4; ++q) {
                const int4 w = row[q];
                dup += (4 * q + 0 < lane && w.x == e_mine) + (4 * q + 1 < lane && w.y == e_mine) +
                       (4 * q + 2 < lane && w.z == e_mine) + (4 * q + 3 < lane && w.w == e_mine);
            }
        }
        int row = -1;
        if (lane < k && e_mine >= 0) {
            row = dup;
            for (int w = 0; w < kFusedWarps; ++w) row += s_part[w][lane];
        }
        int rrow = -1;
        if (lane < nr) {
            rrow = 0;
            for (int w = 0; w < kFusedWarps; ++w) rrow += s_part[w][32 + lane];
            s_rrow[lane] = rrow;
        }
        const bool ok_e = row >= 0 && (int64_t)row < p.exp_cap;
        const unsigned me = __ballot_sync(kFull, ok_e);
        if (ok_e) s_dst[__popc(me & lt)] = p.expanded + (size_t)row * p.V + v0;
        const int ne = __popc(me);
        const bool ok_r = rrow >= 0 && (int64_t)rrow < p.recv_cap;
        const unsigned mr = __ballot_sync(kFull, ok_r);
        if (ok_r) s_dst[ne + __popc(mr & lt)] = p.recv + (size_t)rrow * p.V + v0;
        if (lane == 0) s_n = ne + __popc(mr);
        if (c == 0 && lane < k) p.pos[(size_t)t * k + lane] = row;
        __syncwarp();
        if (c == 0) {
            for (int r = lane; r < R; r += 32) {
                int v = -1;
                if ((m_own >> r) & 1ull) v = s_rrow[__popcll((long long)(m_own & lowmask64(r)))];
                p.recv_pos[(size_t)t * R + r] = v;
            }
        }
    }
    __syncthreads();

    // the stores: a long chunk as one TMA bulk store per destination row
    // (one thread each); a short one as items q = (destination i, vector v),
    // q = i nv + v, spread over all threads (a few tokens' rows still use the
    // whole CTA)
    if (bulk) {
        if (tid < s_n) {
            const uint32_t src_s = (uint32_t)__cvta_generic_to_shared(s_x);
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                             s_dst[tid]),
                         "r"(src_s), "r"((unsigned)nv * 16u)
                         : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            // the chunk must stay in shared memory until the engine has read it
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
        return;
    }
    const int items = s_n * nv;
    if (items > 0) {
        int i = tid / nv, v = tid - (tid / nv) * nv;
        const int si = kFusedThreads / nv, sv = kFusedThreads - si * nv;
        for (int q = tid; q < items; q += kFusedThreads) {
            st_v4(s_dst[i] + v, s_x[v]);
            v += sv;
            i += si;
            if (v >= nv) {
                v -= nv;
                ++i;
            }
        }
    }
}

}  // namespace

namespace {

template <typename K>
cudaError_t launch_smem(K kernel, const FusedParams &p, dim3 grid, size_t smem, cudaStream_t s)
{
    // above the default 48 KB (one route per token at the largest batches)
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kernel, grid, dim3(kFusedThreads), smem, s, p);
}

template <typename IdxT, int KM>
cudaError_t launch_km(const FusedParams &p, int vpt, dim3 grid, size_t smem, cudaStream_t s)
{
    switch (vpt) {
    case 1: return launch_smem(layout_dispatch_kernel<IdxT, KM, 1>, p, grid, smem, s);
    case 2: return launch_smem(layout_dispatch_kernel<IdxT, KM, 2>, p, grid, smem, s);
    default: return launch_smem(layout_dispatch_kernel<IdxT, KM, 4>, p, grid, smem, s);
    }
}

template <typename IdxT>
cudaError_t launch_t(const FusedParams &p, int vpt, dim3 grid, size_t smem, cudaStream_t s)
{
    if (p.k <= 4) return launch_km<IdxT, 4>(p, vpt, grid, smem, s);
    if (p.k <= 8) return launch_km<IdxT, 8>(p, vpt, grid, smem, s);
    if (p.k <= 16) return launch_km<IdxT, 16>(p, vpt, grid, smem, s);
    return launch_km<IdxT, 32>(p, vpt, grid, smem, s);
}

}  // namespace

// Target CTAs per SM.  Every CTA counts over all routes, so fewer, wider
// chunks cost less count work in total; measured on B200 (amortised steps):
// decode 20.3 us at 1 CTA per SM against 20.7 at 2 and 21.0 at 4, DP
// compact 20.4 / 20.6 / 20.9 us, tiny unchanged.
#ifndef EPX_FUSED_CTAS_PER_SM
#define EPX_FUSED_CTAS_PER_SM 1
#endif

cudaError_t launch_layout_dispatch(const FusedParams &p0, int idx_bits, cudaStream_t s)
{
    FusedParams p = p0;
    // per-CTA counting reads every route: small batches only (this also keeps
    // the summary CTA's 16-bit expert counts below 2^16)
    if ((long long)p.T * p.k > kFusedMaxRoutes) return cudaErrorNotSupported;
    const int nsm = current_sm_count();
    int chunks = 1, vpt = 1;
    if (p.T > 0) {
        // about EPX_FUSED_CTAS_PER_SM CTAs per SM, chunks of >= 32 vectors,
        // at most four vectors per thread
        chunks = (EPX_FUSED_CTAS_PER_SM * nsm + p.T - 1) / p.T;
        const int max_chunks = (p.V + 31) / 32;
        if (chunks > max_chunks) chunks = max_chunks;
        const int min_chunks = (p.V + 4 * kFusedThreads - 1) / (4 * kFusedThreads);
        if (chunks < min_chunks) chunks = min_chunks;
        if (chunks < 1) chunks = 1;
        p.vpc = (p.V + chunks - 1) / chunks;
        chunks = (p.V + p.vpc - 1) / p.vpc;
        vpt = (p.vpc + kFusedThreads - 1) / kFusedThreads;
        vpt = vpt <= 1 ? 1 : vpt <= 2 ? 2 : 4;
    }
    p.chunks = chunks;
    const long long ctas = 1 + (long long)p.T * chunks;
    if (ctas > 0x7fffffffLL) return cudaErrorNotSupported;
    // summary CTA: packed expert counts, rank counts, flags, scan scratch;
    // token CTAs: the chunk of x, the batch's experts (rows padded to KM
    // entries) and rank sets
    const size_t km = p.k <= 4 ? 4 : p.k <= 8 ? 8 : p.k <= 16 ? 16 : 32;
    const size_t smem_sum = (((size_t)(p.E + 1) / 2 + p.R + 2 + 1) & ~(size_t)1) * 4 +
                            (kFusedWarps + 1) * 8;
    const size_t smem_tok = (size_t)p.vpc * 16 + (size_t)p.T * km * 4 + (size_t)p.T * 8;
    const size_t smem = smem_sum > smem_tok ? smem_sum : smem_tok;
    p.early_pdl = early_trigger(ctas);
    const dim3 grid((unsigned)ctas);
    return idx_bits == 64 ? launch_t<long long>(p, vpt, grid, smem, s)
                          : launch_t<int>(p, vpt, grid, smem, s);
}

}  // namespace epx
