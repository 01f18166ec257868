// C ABI of libepx: argument validation, layout carving and launches.
// The operations themselves are documented in include/epx.h.
#include <string.h>

#include "epx_internal.cuh"

using namespace epx;

namespace {

inline cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool sizes_ok(int32_t T, int32_t k, int32_t E, int32_t R)
{
    if (T < 0 || k < 1 || E < 1 || R < 1) return false;
    if (k > EPX_MAX_TOPK || R > EPX_MAX_RANKS || E > EPX_MAX_EXPERTS) return false;
    if (E % R != 0) return false;
    if ((int64_t)T * k > INT32_MAX || (int64_t)T * R > INT32_MAX) return false;
    return true;
}

bool layout_ok(const ep_layout_t *L)
{
    if (!L) return false;
    if (!sizes_ok(L->T, L->k, L->E, L->R)) return false;
    if (L->idx_bits != 32 && L->idx_bits != 64) return false;
    return L->cnt_e && L->off_e && L->cnt_r && L->off_r && L->pos && L->recv_pos && L->totals &&
           L->work;
}

ep_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

// peers[0..R) into device form; false if an entry is malformed
bool peers_in(const ep_peer_rows_t *peers, int R, int64_t row_align, PeerRows *out,
                     bool meta)
{
    for (int r = 0; r < R; ++r) {
        const ep_peer_rows_t &e = peers[r];
        if (e.cap < 0 || e.row0 < 0 || e.first < 0 || e.count < 0) return false;
        if (e.cap > 0 && !e.rows) return false;
        if (!aligned(e.rows, (size_t)row_align)) return false;
        if (meta && ((e.meta_idx && !aligned(e.meta_idx, 4)) || (e.meta_w && !aligned(e.meta_w, 4))))
            return false;
        out[r].rows = static_cast<uint4 *>(e.rows);
        out[r].meta_idx = meta ? e.meta_idx : nullptr;
        out[r].meta_w = meta ? e.meta_w : nullptr;
        out[r].row0 = e.row0;
        out[r].cap = e.cap;
        out[r].first = e.first;
        out[r].count = e.count;
    }
    return true;
}

}  // namespace

extern "C" {

int32_t ep_abi_version(void) { return EPX_ABI_VERSION; }

const char *ep_status_str(ep_status_t s)
{
    switch (s) {
    case EP_OK: return "EP_OK";
    case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG: invalid argument";
    case EP_ERR_MISALIGNED: return "EP_ERR_MISALIGNED: buffer not 16-byte aligned";
    case EP_ERR_CAPACITY: return "EP_ERR_CAPACITY: a destination row exceeded a capacity";
    case EP_ERR_BAD_INDEX: return "EP_ERR_BAD_INDEX: a topk index < -1 or >= E was dropped";
    case EP_ERR_CUDA: return "EP_ERR_CUDA: CUDA runtime error";
    case EP_ERR_UNSUPPORTED: return "EP_ERR_UNSUPPORTED: size beyond a library limit";
    }
    return "EP_ERR_UNKNOWN";
}

size_t ep_layout_bytes(int32_t T, int32_t k, int32_t E, int32_t R)
{
    if (!sizes_ok(T, k, E, R)) return 0;
    size_t n = 0;
    n += round_up(sizeof(int32_t) * (size_t)E, 16);
    n += round_up(sizeof(int32_t) * ((size_t)E + 1), 16);
    n += round_up(sizeof(int32_t) * (size_t)R, 16);
    n += round_up(sizeof(int32_t) * ((size_t)R + 1), 16);
    n += round_up(sizeof(int32_t) * (size_t)T * k, 16);
    n += round_up(sizeof(int32_t) * (size_t)T * R, 16);
    n += round_up(sizeof(int32_t) * 4, 16);
    n += round_up(grid_work_bytes(T, k, E, R), 16);
    return n;
}

ep_status_t ep_layout_init(ep_layout_t *L, int32_t T, int32_t k, int32_t E, int32_t R,
                           int32_t idx_bits, void *dev_mem, size_t bytes)
{
    if (!L || !dev_mem) return EP_ERR_INVALID_ARG;
    if (T < 0 || k < 1 || E < 1 || R < 1 || E % R != 0) return EP_ERR_INVALID_ARG;
    if (k > EPX_MAX_TOPK || R > EPX_MAX_RANKS || E > EPX_MAX_EXPERTS) return EP_ERR_UNSUPPORTED;
    if (!sizes_ok(T, k, E, R)) return EP_ERR_INVALID_ARG;
    if (idx_bits != 32 && idx_bits != 64) return EP_ERR_INVALID_ARG;
    if (!aligned(dev_mem, 16)) return EP_ERR_MISALIGNED;
    if (bytes < ep_layout_bytes(T, k, E, R)) return EP_ERR_INVALID_ARG;
    char *p = static_cast<char *>(dev_mem);
    auto take = [&](size_t n) {
        int32_t *r = reinterpret_cast<int32_t *>(p);
        p += round_up(sizeof(int32_t) * n, 16);
        return r;
    };
    ep_layout_t l;
    memset(&l, 0, sizeof l);
    l.T = T;
    l.k = k;
    l.E = E;
    l.R = R;
    l.idx_bits = idx_bits;
    l.cnt_e = take((size_t)E);
    l.off_e = take((size_t)E + 1);
    l.cnt_r = take((size_t)R);
    l.off_r = take((size_t)R + 1);
    l.pos = take((size_t)T * k);
    l.recv_pos = take((size_t)T * R);
    l.totals = take(4);
    l.work = reinterpret_cast<int32_t *>(p);
    *L = l;
    return EP_OK;
}

ep_status_t ep_layout_variant(const void *topk_idx, const ep_layout_t *L, int32_t variant,
                              void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (variant < 0 || variant > 3) return EP_ERR_INVALID_ARG;
    if (L->T > 0 && !topk_idx) return EP_ERR_INVALID_ARG;
    if (topk_idx && !aligned(topk_idx, (size_t)L->idx_bits / 8)) return EP_ERR_MISALIGNED;
    LayoutParams p;
    memset(&p, 0, sizeof p);
    p.idx = topk_idx;
    p.T = L->T;
    p.k = L->k;
    p.E = L->E;
    p.R = L->R;
    p.inv_epr = 1.0f / (float)(L->E / L->R);
    p.cnt_e = L->cnt_e;
    p.off_e = L->off_e;
    p.cnt_r = L->cnt_r;
    p.off_r = L->off_r;
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.totals = L->totals;
    p.work = L->work;
    const cudaError_t e = launch_layout(p, L->idx_bits, variant, as_stream(stream));
    return e == cudaErrorNotSupported ? EP_ERR_UNSUPPORTED : from_cuda(e);
}

ep_status_t ep_layout(const void *topk_idx, const ep_layout_t *L, void *stream)
{
    return ep_layout_variant(topk_idx, L, 0, stream);
}

}  // extern "C"

namespace {

// Dispatch + expand; topk_idx non-null means the previous kernel on the
// stream is this library's layout kernel for the same batch (see
// DispatchParams::prefetch).
ep_status_t dispatch_expand_impl(const void *x, int32_t H, const ep_layout_t *L, void *recv,
                                 int64_t recv_cap, void *expanded, int64_t exp_cap,
                                 int32_t variant, const void *topk_idx, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || recv_cap < 0 || exp_cap < 0) return EP_ERR_INVALID_ARG;
    if (variant < 0 || variant > 2) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    // recv may be NULL with recv_cap 0: expanded rows only
    if (!x || !expanded || (!recv && recv_cap != 0)) return EP_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(recv, 16) || !aligned(expanded, 16)) return EP_ERR_MISALIGNED;
    DispatchParams p;
    memset(&p, 0, sizeof p);
    p.x = static_cast<const uint4 *>(x);
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.T = L->T;
    p.k = L->k;
    p.R = L->R;
    p.V = H / 8;
    p.recv = static_cast<uint4 *>(recv);
    p.recv_cap = recv_cap;
    p.expanded = static_cast<uint4 *>(expanded);
    p.exp_cap = exp_cap;
    p.err = L->totals + 3;
    p.prefetch = topk_idx != nullptr;
    p.idx = topk_idx;
    p.idx_bits = L->idx_bits;
    p.E = L->E;
    return from_cuda(launch_dispatch(p, variant, as_stream(stream)));
}

}  // namespace

extern "C" {

ep_status_t ep_dispatch_expand_variant(const void *x, int32_t H, const ep_layout_t *L,
                                       void *recv, int64_t recv_cap, void *expanded,
                                       int64_t exp_cap, int32_t variant, void *stream)
{
    return dispatch_expand_impl(x, H, L, recv, recv_cap, expanded, exp_cap, variant, nullptr,
                                stream);
}

ep_status_t ep_dispatch_expand(const void *x, int32_t H, const ep_layout_t *L, void *recv,
                               int64_t recv_cap, void *expanded, int64_t exp_cap, void *stream)
{
    return ep_dispatch_expand_variant(x, H, L, recv, recv_cap, expanded, exp_cap, 0, stream);
}

ep_status_t ep_layout_dispatch_expand_variant(const void *topk_idx, const ep_layout_t *L,
                                              const void *x, int32_t H, void *recv,
                                              int64_t recv_cap, void *expanded, int64_t exp_cap,
                                              int32_t variant, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || recv_cap < 0 || exp_cap < 0) return EP_ERR_INVALID_ARG;
    if (variant < 0 || variant > 2) return EP_ERR_INVALID_ARG;
    if (L->T > 0 && (!topk_idx || !x || !recv || !expanded)) return EP_ERR_INVALID_ARG;
    if (topk_idx && !aligned(topk_idx, (size_t)L->idx_bits / 8)) return EP_ERR_MISALIGNED;
    if (L->T > 0 && (!aligned(x, 16) || !aligned(recv, 16) || !aligned(expanded, 16)))
        return EP_ERR_MISALIGNED;
    const long long routes = (long long)L->T * L->k;
    // automatic: one launch where it was measured faster on B200 (while each
    // CTA's count over all routes stays cheap), else the layout and dispatch
    // kernels
    const bool automatic = variant == 0;
    if (automatic)
        variant = routes >= kFusedAutoMinRoutes && routes <= kFusedAutoMaxRoutes ? 1 : 2;
    if (variant == 1 && routes > kFusedMaxRoutes) {
        if (!automatic) return EP_ERR_UNSUPPORTED;
        variant = 2;
    }
    if (variant == 2) {
        ep_status_t st = ep_layout(topk_idx, L, stream);
        if (st != EP_OK || L->T == 0) return st;
        // the layout kernel just launched lets the dispatch read x early
        return dispatch_expand_impl(x, H, L, recv, recv_cap, expanded, exp_cap, 0, topk_idx,
                                    stream);
    }
    FusedParams p;
    memset(&p, 0, sizeof p);
    p.idx = topk_idx;
    p.x = static_cast<const uint4 *>(x);
    p.T = L->T;
    p.k = L->k;
    p.E = L->E;
    p.R = L->R;
    p.V = H / 8;
    p.inv_epr = 1.0f / (float)(L->E / L->R);
    p.inv_k = 1.0f / (float)L->k;
    p.recv = static_cast<uint4 *>(recv);
    p.recv_cap = recv_cap;
    p.expanded = static_cast<uint4 *>(expanded);
    p.exp_cap = exp_cap;
    p.cnt_e = L->cnt_e;
    p.off_e = L->off_e;
    p.cnt_r = L->cnt_r;
    p.off_r = L->off_r;
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.totals = L->totals;
    const cudaError_t e = launch_layout_dispatch(p, L->idx_bits, as_stream(stream));
    if (e == cudaErrorNotSupported) {  // checked before launching anything
        if (!automatic) return EP_ERR_UNSUPPORTED;
        const ep_status_t st = ep_layout(topk_idx, L, stream);
        if (st != EP_OK || L->T == 0) return st;
        return dispatch_expand_impl(x, H, L, recv, recv_cap, expanded, exp_cap, 0, topk_idx,
                                    stream);
    }
    return from_cuda(e);
}

ep_status_t ep_layout_dispatch_expand(const void *topk_idx, const ep_layout_t *L, const void *x,
                                      int32_t H, void *recv, int64_t recv_cap, void *expanded,
                                      int64_t exp_cap, void *stream)
{
    return ep_layout_dispatch_expand_variant(topk_idx, L, x, H, recv, recv_cap, expanded, exp_cap,
                                             0, stream);
}

ep_status_t ep_dispatch(const void *x, int32_t H, const ep_layout_t *L, void *recv,
                        int64_t recv_cap, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || recv_cap < 0) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!x || !recv) return EP_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(recv, 16)) return EP_ERR_MISALIGNED;
    DispatchParams p;
    memset(&p, 0, sizeof p);
    p.x = static_cast<const uint4 *>(x);
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.T = L->T;
    p.k = L->k;
    p.R = L->R;
    p.V = H / 8;
    p.recv = static_cast<uint4 *>(recv);
    p.recv_cap = recv_cap;
    p.expanded = nullptr;  // no expanded copy
    p.exp_cap = 0;
    p.err = L->totals + 3;
    return from_cuda(launch_dispatch(p, 0, as_stream(stream)));
}

ep_status_t ep_route_meta(const void *topk_idx, const float *topk_weights, const ep_layout_t *L,
                          int32_t *meta_idx, float *meta_w, int64_t rows, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (rows < 0) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!topk_idx || !topk_weights || !meta_idx || !meta_w) return EP_ERR_INVALID_ARG;
    if (!aligned(topk_idx, (size_t)L->idx_bits / 8) || !aligned(topk_weights, 4) ||
        !aligned(meta_idx, 4) || !aligned(meta_w, 4))
        return EP_ERR_MISALIGNED;
    MetaParams p;
    memset(&p, 0, sizeof p);
    p.idx = topk_idx;
    p.w = topk_weights;
    p.recv_pos = L->recv_pos;
    p.T = L->T;
    p.k = L->k;
    p.E = L->E;
    p.R = L->R;
    p.inv_epr = 1.0f / (float)(L->E / L->R);
    p.meta_idx = meta_idx;
    p.meta_w = meta_w;
    p.rows = rows;
    p.err = L->totals + 3;
    return from_cuda(launch_route_meta(p, L->idx_bits, as_stream(stream)));
}

ep_status_t ep_dispatch_p2p(const void *x, int32_t H, const ep_layout_t *L, const void *topk_idx,
                            const float *topk_weights, const ep_peer_rows_t *peers, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!x || !topk_idx || !topk_weights || !peers) return EP_ERR_INVALID_ARG;
    if (!aligned(x, 16)) return EP_ERR_MISALIGNED;
    if (!aligned(topk_idx, (size_t)L->idx_bits / 8) || !aligned(topk_weights, 4))
        return EP_ERR_MISALIGNED;
    P2PDispatchParams p;
    memset(&p, 0, sizeof p);
    if (!peers_in(peers, L->R, 16, p.peer, true)) return EP_ERR_INVALID_ARG;
    p.x = static_cast<const uint4 *>(x);
    p.recv_pos = L->recv_pos;
    p.off_r = L->off_r;
    p.idx = topk_idx;
    p.w = topk_weights;
    p.idx_bits = L->idx_bits;
    p.T = L->T;
    p.k = L->k;
    p.E = L->E;
    p.R = L->R;
    p.V = H / 8;
    p.inv_epr = 1.0f / (float)(L->E / L->R);
    p.err = L->totals + 3;
    return from_cuda(launch_dispatch_p2p(p, as_stream(stream)));
}

ep_status_t ep_combine_local_reduce_p2p(const void *expert_out, const float *topk_weights,
                                        int32_t H, const ep_layout_t *L, int32_t partial_bits,
                                        int64_t y_rows, const ep_peer_rows_t *peers, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || y_rows < 0) return EP_ERR_INVALID_ARG;
    if (partial_bits != 32 && partial_bits != 16) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!expert_out || !topk_weights || !peers) return EP_ERR_INVALID_ARG;
    if (!aligned(expert_out, 16) || !aligned(topk_weights, 4)) return EP_ERR_MISALIGNED;
    LocalP2PParams p;
    memset(&p, 0, sizeof p);
    if (!peers_in(peers, L->R, 16, p.peer, false)) return EP_ERR_INVALID_ARG;
    p.n_peer = L->R;
    p.y = static_cast<const uint4 *>(expert_out);
    p.w = topk_weights;
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.off_e = L->off_e;
    p.T = L->T;
    p.k = L->k;
    p.R = L->R;
    p.epr = L->E / L->R;
    p.V = H / 8;
    p.y_rows = y_rows;
    p.partial = nullptr;
    p.part_cap = INT64_MAX;  // the peers' caps are checked per row
    p.part_bits = partial_bits;
    p.err = L->totals + 3;
    return from_cuda(launch_local_reduce_p2p(p, as_stream(stream)));
}

ep_status_t ep_ipc_malloc(size_t bytes, void **dev_ptr, void *handle)
{
    if (!dev_ptr || !handle || bytes == 0) return EP_ERR_INVALID_ARG;
    *dev_ptr = nullptr;
    void *ptr = nullptr;
    if (cudaMalloc(&ptr, bytes) != cudaSuccess) return EP_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, ptr) != cudaSuccess) {
        cudaFree(ptr);
        return EP_ERR_CUDA;
    }
    static_assert(sizeof(cudaIpcMemHandle_t) <= EPX_IPC_HANDLE_BYTES, "IPC handle size");
    memset(handle, 0, EPX_IPC_HANDLE_BYTES);
    memcpy(handle, &h, sizeof h);
    *dev_ptr = ptr;
    return EP_OK;
}

ep_status_t ep_ipc_free(void *dev_ptr)
{
    if (!dev_ptr) return EP_ERR_INVALID_ARG;
    return from_cuda(cudaFree(dev_ptr));
}

ep_status_t ep_ipc_open(const void *handle, void **dev_ptr)
{
    if (!handle || !dev_ptr) return EP_ERR_INVALID_ARG;
    *dev_ptr = nullptr;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof h);
    void *ptr = nullptr;
    if (cudaIpcOpenMemHandle(&ptr, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return EP_ERR_CUDA;
    *dev_ptr = ptr;
    return EP_OK;
}

ep_status_t ep_ipc_close(void *dev_ptr)
{
    if (!dev_ptr) return EP_ERR_INVALID_ARG;
    return from_cuda(cudaIpcCloseMemHandle(dev_ptr));
}

ep_status_t ep_expand_index(const ep_layout_t *L, int32_t *src_row, int64_t rows, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (rows < 0) return EP_ERR_INVALID_ARG;
    if (L->T == 0 || rows == 0) return EP_OK;
    if (!src_row) return EP_ERR_INVALID_ARG;
    if (!aligned(src_row, 4)) return EP_ERR_MISALIGNED;
    IndexParams p;
    memset(&p, 0, sizeof p);
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.off_e = L->off_e;
    p.T = L->T;
    p.k = L->k;
    p.R = L->R;
    p.epr = L->E / L->R;
    p.src = src_row;
    p.rows = rows;
    p.err = L->totals + 3;
    return from_cuda(launch_expand_index(p, as_stream(stream)));
}

ep_status_t ep_standin_expert_gather(const void *recv, int64_t recv_rows, int32_t H,
                                     const ep_layout_t *L, const int32_t *src_row, void *y,
                                     int64_t rows, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || rows < 0 || recv_rows < 0) return EP_ERR_INVALID_ARG;
    if (rows == 0 || L->T == 0) return EP_OK;
    if (!recv || !src_row || !y) return EP_ERR_INVALID_ARG;
    if (!aligned(recv, 16) || !aligned(y, 16) || !aligned(src_row, 4)) return EP_ERR_MISALIGNED;
    GatherParams p;
    memset(&p, 0, sizeof p);
    p.recv = static_cast<const uint4 *>(recv);
    p.recv_rows = recv_rows;
    p.src = src_row;
    p.off_e = L->off_e;
    p.totals = L->totals;
    p.E = L->E;
    p.V = H / 8;
    const int64_t cap = (int64_t)L->T * L->k;
    p.rows = rows < cap ? rows : cap;
    p.y = static_cast<uint4 *>(y);
    p.err = L->totals + 3;
    return from_cuda(launch_standin_gather(p, as_stream(stream)));
}

ep_status_t ep_standin_expert(const void *expanded, int32_t H, const ep_layout_t *L, void *y,
                              int64_t rows, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || rows < 0) return EP_ERR_INVALID_ARG;
    if (rows == 0 || L->T == 0) return EP_OK;
    if (!expanded || !y) return EP_ERR_INVALID_ARG;
    if (!aligned(expanded, 16) || !aligned(y, 16)) return EP_ERR_MISALIGNED;
    StandinParams p;
    memset(&p, 0, sizeof p);
    p.ex = static_cast<const uint4 *>(expanded);
    p.off_e = L->off_e;
    p.totals = L->totals;
    p.E = L->E;
    p.V = H / 8;
    const int64_t cap = (int64_t)L->T * L->k;
    p.rows = rows < cap ? rows : cap;
    p.y = static_cast<uint4 *>(y);
    return from_cuda(launch_standin(p, as_stream(stream)));
}

ep_status_t ep_combine_reduce_variant(const void *expert_out, const float *topk_weights,
                                      int32_t H, const ep_layout_t *L, void *out,
                                      int64_t y_rows, int32_t variant, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || y_rows < 0) return EP_ERR_INVALID_ARG;
    if (variant < 0 || variant > 2) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!expert_out || !topk_weights || !out) return EP_ERR_INVALID_ARG;
    if (!aligned(expert_out, 16) || !aligned(out, 16)) return EP_ERR_MISALIGNED;
    if (!aligned(topk_weights, 4)) return EP_ERR_MISALIGNED;
    CombineParams p;
    memset(&p, 0, sizeof p);
    p.y = static_cast<const uint4 *>(expert_out);
    p.w = topk_weights;
    p.pos = L->pos;
    p.T = L->T;
    p.k = L->k;
    p.V = H / 8;
    p.y_rows = y_rows;
    p.out = static_cast<uint4 *>(out);
    p.err = L->totals + 3;
    return from_cuda(launch_combine(p, variant, as_stream(stream)));
}

ep_status_t ep_combine_reduce(const void *expert_out, const float *topk_weights, int32_t H,
                              const ep_layout_t *L, void *out, int64_t y_rows, void *stream)
{
    return ep_combine_reduce_variant(expert_out, topk_weights, H, L, out, y_rows, 0, stream);
}

ep_status_t ep_combine_local_reduce(const void *expert_out, const float *topk_weights, int32_t H,
                                    const ep_layout_t *L, void *partial, int64_t partial_cap,
                                    int32_t partial_bits, int64_t y_rows, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || y_rows < 0 || partial_cap < 0) return EP_ERR_INVALID_ARG;
    if (partial_bits != 32 && partial_bits != 16) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!expert_out || !topk_weights || !partial) return EP_ERR_INVALID_ARG;
    if (!aligned(expert_out, 16) || !aligned(partial, 16)) return EP_ERR_MISALIGNED;
    if (!aligned(topk_weights, 4)) return EP_ERR_MISALIGNED;
    LocalParams p;
    memset(&p, 0, sizeof p);
    p.y = static_cast<const uint4 *>(expert_out);
    p.w = topk_weights;
    p.pos = L->pos;
    p.recv_pos = L->recv_pos;
    p.off_e = L->off_e;
    p.T = L->T;
    p.k = L->k;
    p.R = L->R;
    p.epr = L->E / L->R;
    p.V = H / 8;
    p.y_rows = y_rows;
    p.partial = partial;
    p.part_cap = partial_cap;
    p.part_bits = partial_bits;
    p.err = L->totals + 3;
    return from_cuda(launch_local_reduce(p, as_stream(stream)));
}

ep_status_t ep_combine_epilogue(const void *partial, int32_t partial_bits, int32_t H,
                                const ep_layout_t *L, int64_t partial_cap, const void *residual,
                                void *out, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    if (H <= 0 || H % 8 != 0 || partial_cap < 0) return EP_ERR_INVALID_ARG;
    if (partial_bits != 32 && partial_bits != 16) return EP_ERR_INVALID_ARG;
    if (L->T == 0) return EP_OK;
    if (!partial || !out) return EP_ERR_INVALID_ARG;
    if (!aligned(partial, 16) || !aligned(out, 16)) return EP_ERR_MISALIGNED;
    if (residual && !aligned(residual, 16)) return EP_ERR_MISALIGNED;
    EpilogueParams p;
    memset(&p, 0, sizeof p);
    p.partial = partial;
    p.part_bits = partial_bits;
    p.recv_pos = L->recv_pos;
    p.residual = static_cast<const uint4 *>(residual);
    p.T = L->T;
    p.R = L->R;
    p.V = H / 8;
    p.part_cap = partial_cap;
    p.out = static_cast<uint4 *>(out);
    p.err = L->totals + 3;
    return from_cuda(launch_epilogue(p, as_stream(stream)));
}

ep_status_t ep_layout_read_totals(const ep_layout_t *L, int64_t *n_route, int64_t *n_recv,
                                  int64_t *t_real, int32_t *dev_err, void *stream)
{
    if (!layout_ok(L)) return EP_ERR_INVALID_ARG;
    int32_t h[4] = {0, 0, 0, 0};
    cudaStream_t s = as_stream(stream);
    cudaError_t e = cudaMemcpyAsync(h, L->totals, sizeof h, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return EP_ERR_CUDA;
    if (n_route) *n_route = h[0];
    if (n_recv) *n_recv = h[1];
    if (t_real) *t_real = h[2];
    if (dev_err) *dev_err = h[3];
    if (h[3] & (int32_t)EP_DEVERR_BAD_INDEX) return EP_ERR_BAD_INDEX;
    if (h[3] & (int32_t)(EP_DEVERR_RECV_CAP | EP_DEVERR_EXP_CAP | EP_DEVERR_Y_ROWS))
        return EP_ERR_CAPACITY;
    if (h[3] & (int32_t)EP_DEVERR_TIMEOUT) return EP_ERR_CUDA;
    return EP_OK;
}

// ------------------------------------------------------- host round trip

namespace {

struct RoundtripCarve {
    size_t x, idx, w, lay, recv, exp, y, out, total;
};

bool roundtrip_carve(int32_t T, int32_t H, int32_t k, int32_t E, int32_t R, int32_t idx_bits,
                     RoundtripCarve *c)
{
    if (!sizes_ok(T, k, E, R) || H <= 0 || H % 8 != 0) return false;
    if (idx_bits != 32 && idx_bits != 64) return false;
    const size_t row = (size_t)H * 2;
    const size_t cap_recv = (size_t)T * (k < R ? k : R);
    const size_t cap_exp = (size_t)T * k;
    size_t off = 0;
    auto take = [&](size_t n) {
        size_t r = off;
        off += round_up(n ? n : 1, 256);
        return r;
    };
    c->x = take((size_t)T * row);
    c->idx = take((size_t)T * k * (idx_bits / 8));
    c->w = take((size_t)T * k * 4);
    c->lay = take(ep_layout_bytes(T, k, E, R));
    c->recv = take(cap_recv * row);
    c->exp = take(cap_exp * row);
    c->y = take(cap_exp * row);
    c->out = take((size_t)T * row);
    c->total = off;
    return true;
}

}  // namespace

size_t ep_roundtrip_device_bytes(int32_t T, int32_t H, int32_t k, int32_t E, int32_t R,
                                 int32_t idx_bits)
{
    RoundtripCarve c;
    return roundtrip_carve(T, H, k, E, R, idx_bits, &c) ? c.total : 0;
}

ep_status_t ep_roundtrip_host(const void *x_host, const void *topk_idx_host,
                              const float *topk_weights_host, int32_t T, int32_t H, int32_t k,
                              int32_t E, int32_t R, int32_t idx_bits, void *dev_mem, size_t bytes,
                              void *out_host, int32_t *dev_err_host, void *stream)
{
    RoundtripCarve c;
    if (!roundtrip_carve(T, H, k, E, R, idx_bits, &c)) return EP_ERR_INVALID_ARG;
    if (!dev_mem || bytes < c.total) return EP_ERR_INVALID_ARG;
    if (!aligned(dev_mem, 256)) return EP_ERR_MISALIGNED;
    if (T > 0 && (!x_host || !topk_idx_host || !topk_weights_host || !out_host))
        return EP_ERR_INVALID_ARG;
    char *d = static_cast<char *>(dev_mem);
    cudaStream_t s = as_stream(stream);
    const size_t row = (size_t)H * 2;
    const int64_t cap_recv = (int64_t)T * (k < R ? k : R);
    const int64_t cap_exp = (int64_t)T * k;
    ep_layout_t L;
    ep_status_t st = ep_layout_init(&L, T, k, E, R, idx_bits, d + c.lay, ep_layout_bytes(T, k, E, R));
    if (st != EP_OK) return st;
    // the grid layout's barrier words must start at zero (the scratch may
    // hold anything from an earlier call)
    if (cudaMemsetAsync(L.work, 0, sizeof(int32_t) * kGridHeaderWords, s) != cudaSuccess)
        return EP_ERR_CUDA;
    if (T > 0) {
        cudaError_t e;
        e = cudaMemcpyAsync(d + c.x, x_host, (size_t)T * row, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return EP_ERR_CUDA;
        e = cudaMemcpyAsync(d + c.idx, topk_idx_host, (size_t)T * k * (idx_bits / 8),
                            cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return EP_ERR_CUDA;
        e = cudaMemcpyAsync(d + c.w, topk_weights_host, (size_t)T * k * 4, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return EP_ERR_CUDA;
    }
    st = ep_layout_dispatch_expand(d + c.idx, &L, d + c.x, H, d + c.recv, cap_recv, d + c.exp,
                                   cap_exp, stream);
    if (st != EP_OK) return st;
    if (T > 0) {
        st = ep_standin_expert(d + c.exp, H, &L, d + c.y, cap_exp, stream);
        if (st != EP_OK) return st;
        st = ep_combine_reduce(d + c.y, reinterpret_cast<const float *>(d + c.w), H, &L,
                               d + c.out, cap_exp, stream);
        if (st != EP_OK) return st;
        const cudaError_t e =
            cudaMemcpyAsync(out_host, d + c.out, (size_t)T * row, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return EP_ERR_CUDA;
    }
    // the layout's device error word (dropped routes / rows) for the caller
    if (dev_err_host &&
        cudaMemcpyAsync(dev_err_host, L.totals + 3, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess)
        return EP_ERR_CUDA;
    return EP_OK;
}

void ep_debug_dispatch_first_wait_limit(int64_t limit)
{
    dispatch_first_wait_limit.store(limit, std::memory_order_relaxed);
}

}  // extern "C"
