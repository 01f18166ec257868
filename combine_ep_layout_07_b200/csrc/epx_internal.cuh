// Internal declarations shared by the CUDA translation units of libepx.
// Not part of the public ABI (that is include/epx.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "epx.h"

namespace epx {

constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------ parameters

struct LayoutParams {
    const void *idx;
    int T, k, E, R;
    float inv_epr;  // 1.0f / (E / R): rank of expert e = floor((e + 0.5) * inv_epr)
    int tpc;        // tokens per CTA of the cluster
    int tch;        // tokens per chunk (columns of the count matrix)
    int ld;         // count-matrix row length in words: odd, >= tch
    int wde, wdr;   // count-matrix rows (two 16-bit counts per 32-bit word) for experts / ranks
    int tpw;        // warp-chunk schedule: whole tokens per warp, floor(32 / k)
    int tstr;       // warp-chunk schedule: table row length in 16-bit counts (even, >= E + R)
    float inv_k;    // 1.0f / k
    int bits_e, bits_r;  // bits of the largest expert / rank
    int hs;              // grid schedule: workspace row length in words
    int32_t *cnt_e, *off_e, *cnt_r, *off_r, *pos, *recv_pos, *totals;
    int32_t *work;       // grid schedule workspace (header + one row per CTA), or null
};

// Grid schedule of the layout: one CTA per this many routes, at most
// kGridMaxCtas CTAs (and never more than the SMs).  Its workspace holds a
// header of barrier words, one row of packed 16-bit (expert | rank) counts
// per CTA, one row of 32-bit exclusive prefixes per CTA, and the totals.
constexpr int kGridRoutesPerCta = 256;
constexpr int kGridMaxCtas = 256;
constexpr int kGridHeaderWords = 16;

inline int grid_row_words(int E, int R) { return (((E + R + 1) / 2) + 3) & ~3; }
inline int grid_prefix_words(int E, int R) { return (E + R + 3) & ~3; }

inline int grid_max_ctas(long long routes)
{
    long long n = (routes + kGridRoutesPerCta - 1) / kGridRoutesPerCta;
    return (int)(n < kGridMaxCtas ? n : kGridMaxCtas);
}

inline size_t grid_work_bytes(int T, int k, int E, int R)
{
    const size_t nb = (size_t)grid_max_ctas((long long)T * k);
    return sizeof(int32_t) * ((size_t)kGridHeaderWords + nb * grid_row_words(E, R) +
                              (nb + 1) * grid_prefix_words(E, R));
}


struct DispatchParams {
    const uint4 *x;
    const int32_t *pos;
    const int32_t *recv_pos;
    int T, k, R;
    int V;    // 16-byte vectors per row (H / 8)
    int vpc;  // vectors per CTA chunk
    uint4 *recv;
    int64_t recv_cap;
    uint4 *expanded;
    int64_t exp_cap;
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
    long long first_wait_limit;  // bulk engine: polls allowed by a CTA's first bounded wait
    // both engines: the previous kernel is this library's layout kernel,
    // launched for the same batch: it lets this grid start only once every
    // kernel before it has completed, so x and topk_idx (which the layout
    // does not write) may be read before this kernel's wait
    int prefetch;
    const void *idx;  // topk_idx [T, k], idx_bits wide (prefetch only)
    int idx_bits, E;
};

// layout + dispatch/expand in one launch (small batches)
struct FusedParams {
    const void *idx;
    const uint4 *x;
    int T, k, E, R;
    int V;       // 16-byte vectors per row (H / 8)
    int vpc;     // vectors per CTA chunk
    int chunks;  // CTAs per token
    float inv_epr;
    float inv_k;  // 1.0f / k: token of flat route i = floor((i + 0.5) * inv_k)
    uint4 *recv;
    int64_t recv_cap;
    uint4 *expanded;
    int64_t exp_cap;
    int32_t *cnt_e, *off_e, *cnt_r, *off_r, *pos, *recv_pos, *totals;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

// the one-launch layout + dispatch handles at most this many routes (T*k)
constexpr int kFusedMaxRoutes = EPX_FUSED_MAX_ROUTES;
// ... and is the automatic choice in this range of routes
constexpr int kFusedAutoMinRoutes = EPX_FUSED_AUTO_MIN_ROUTES;
constexpr int kFusedAutoMaxRoutes = EPX_FUSED_AUTO_MAX_ROUTES;

// routing that travels with each row of a multi-GPU dispatch
struct MetaParams {
    const void *idx;
    const float *w;
    const int32_t *recv_pos;
    int T, k, E, R;
    float inv_epr;
    int32_t *meta_idx;  // [rows, k]
    float *meta_w;      // [rows, k]
    int64_t rows;
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

struct CombineParams {
    const uint4 *y;
    const float *w;
    const int32_t *pos;
    int T, k;
    int V;
    int vpc;
    int64_t y_rows;
    uint4 *out;
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

struct LocalParams {
    const uint4 *y;
    const float *w;
    const int32_t *pos;
    const int32_t *recv_pos;
    const int32_t *off_e;
    int T, k, R, epr;
    int V, vpc;
    int64_t y_rows;
    void *partial;    // [part_cap, H] fp32 or bf16, receive layout
    int64_t part_cap;
    int part_bits;    // 32 or 16
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

// A peer's buffers as the kernels see them (ep_peer_rows_t, in device form).
struct PeerRows {
    uint4 *rows;
    int32_t *meta_idx;
    float *meta_w;
    int64_t row0, cap, first, count;
};

// local reduce whose partial rows go to other ranks' buffers
struct LocalP2PParams : LocalParams {
    int n_peer;
    PeerRows peer[EPX_MAX_RANKS];
};

// dispatch whose rows go straight into the receiving ranks' buffers
struct P2PDispatchParams {
    const uint4 *x;
    const int32_t *recv_pos;
    const int32_t *off_r;
    const void *idx;  // topk_idx [T, k], idx_bits wide
    const float *w;   // topk_weights [T, k]
    int idx_bits;
    int T, k, E, R;
    int V, vpc;
    float inv_epr;
    int32_t *err;
    int early_pdl;
    PeerRows peer[EPX_MAX_RANKS];
};

struct EpilogueParams {
    const void *partial;
    int part_bits;
    const int32_t *recv_pos;
    const uint4 *residual;  // bf16 [T, H] or nullptr
    int T, R, V, vpc;
    int64_t part_cap;
    uint4 *out;
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

struct IndexParams {
    const int32_t *pos;
    const int32_t *recv_pos;
    const int32_t *off_e;
    int T, k, R, epr;
    int32_t *src;   // [rows] recv row serving each expanded row
    int64_t rows;
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

struct GatherParams {
    const uint4 *recv;
    int64_t recv_rows;
    const int32_t *src;
    const int32_t *off_e;
    const int32_t *totals;
    int E, V, vpc;
    int64_t rows;
    uint4 *y;
    int32_t *err;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

struct StandinParams {
    const uint4 *ex;
    const int32_t *off_e;
    const int32_t *totals;
    int E, V, vpc;
    int64_t rows;
    uint4 *y;
    int early_pdl;  // trigger dependents at start (grid fits in one wave)
};

// ------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; arguments are already
// validated by the C-ABI layer.

cudaError_t launch_layout(const LayoutParams &p, int idx_bits, int variant, cudaStream_t s);
cudaError_t launch_dispatch(const DispatchParams &p, int variant, cudaStream_t s);
cudaError_t launch_standin(const StandinParams &p, cudaStream_t s);
// cudaErrorNotSupported when T*k > kFusedMaxRoutes
cudaError_t launch_layout_dispatch(const FusedParams &p, int idx_bits, cudaStream_t s);
cudaError_t launch_combine(const CombineParams &p, int variant, cudaStream_t s);
cudaError_t launch_route_meta(const MetaParams &p, int idx_bits, cudaStream_t s);
cudaError_t launch_local_reduce(const LocalParams &p, cudaStream_t s);
cudaError_t launch_local_reduce_p2p(const LocalP2PParams &p, cudaStream_t s);
cudaError_t launch_dispatch_p2p(const P2PDispatchParams &p, cudaStream_t s);
cudaError_t launch_epilogue(const EpilogueParams &p, cudaStream_t s);
cudaError_t launch_expand_index(const IndexParams &p, cudaStream_t s);
cudaError_t launch_standin_gather(const GatherParams &p, cudaStream_t s);

// Test setting: polls allowed by the first bounded wait of every CTA of the
// bulk copy engine (< 0: the normal limit).  Set by
// ep_debug_dispatch_first_wait_limit.
extern std::atomic<long long> dispatch_first_wait_limit;

// ------------------------------------------------- host-side caches
// Launchers may be called from several host threads at once.

// guards the launchers' small lookup tables
inline std::mutex &launcher_mutex()
{
    static std::mutex m;
    return m;
}

// multiprocessor count of device `dev`, queried once per device
inline int sm_count(int dev)
{
    static std::atomic<int> cache[64];
    int n = 0;
    if (dev >= 0 && dev < 64) n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

inline int current_sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return sm_count(dev);
}

// Programmatic-launch trigger policy: a grid that fits in about one wave
// lets its dependents launch at once (their launch hides behind this grid);
// a multi-wave grid triggers only after each CTA's main work, so waiting
// dependent CTAs do not sit on the SMs through its later waves.  per_sm is
// how many of the grid's CTAs count as one wave's share of an SM (8 for
// 128-thread CTAs; more for smaller CTAs that shared memory does not limit).
inline int early_trigger(long long ctas, int per_sm = 8)
{
    return ctas <= (long long)per_sm * current_sm_count();
}

// maximum dynamic shared memory per block that the layout kernel may use
constexpr int kMaxDynSmem = 227 * 1024;

// Launch `kernel` on `s` with programmatic stream serialisation (the kernel
// may begin while its predecessor in the stream finishes; it synchronises
// with pdl_wait_previous) and, when cluster > 1, a 1-D cluster.
template <typename Params>
cudaError_t launch_pdl(void (*kernel)(Params), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, const Params &p, int cluster = 1)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

// ----------------------------------------------------- device utilities

// Programmatic dependent launch.  Every kernel of the path lets the next one
// in its stream start launching early (its launch and prologue overlap this
// kernel: at once for one-wave grids, after the main work otherwise), and
// waits for the previous one to finish -- with its memory visible -- before
// it touches any global memory.  Without the launch attribute both are
// no-ops.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait_previous()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// 16-byte read-only load that does not allocate in L1 (each source vector is
// read by exactly one thread).
__device__ __forceinline__ uint4 ld_nc_v4(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 16-byte load of data written by an earlier kernel (plain global load).
__device__ __forceinline__ uint4 ld_v4(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(uint4 *p, const uint4 &v)
{
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// streaming (evict-first) store for write-once outputs
__device__ __forceinline__ void st_cs_v4(uint4 *p, const uint4 &v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

}  // namespace epx
