/*
 * epx -- MoE token dispatch and combine on one B200 (sm_100a).
 *
 * C ABI of libepx.so.  Every pointer documented as "device" is caller-owned
 * device memory; the library allocates and frees memory only in
 * ep_ipc_malloc / ep_ipc_free (memory other processes map).  Every call is
 * asynchronous on the given CUDA stream (`stream` is a cudaStream_t passed as
 * void*, NULL = the legacy default stream) except ep_layout_read_totals,
 * which synchronises that stream.
 *
 * Pipeline, as the pages state the problem (DeepEP issue #48 "How to apply
 * Moe MLP to recv_x returned by dispatch when num_expert_per_rank > 1";
 * DeepEP issue #760 "[Performance] DeepEP V2 combine epilogue low batch
 * performance", section "Reproduction"):
 *
 *   ep_layout          topk_idx            -> routing layout ("handle")
 *   ep_dispatch_expand x, layout           -> recv (one row per token and
 *                                             destination rank), expanded
 *                                             (one row per valid route,
 *                                             expert-contiguous)
 *   (expert FFN on expanded rows; ep_standin_expert is a deterministic
 *    stand-in for tests and benchmarks)
 *   ep_combine_reduce  expert_out, topk_weights, layout -> out
 *
 * Logical ranks: experts live on ranks in contiguous blocks of E/R
 * (expert e on rank e / (E/R)), as in the issue #760 reproduction's
 * local_experts.  On one GPU all ranks are partitions of buffers on that
 * GPU; with one process per GPU, ep_dispatch_p2p and
 * ep_combine_local_reduce_p2p (below) store rows into the other ranks'
 * buffers directly.
 *
 * Ordering: inside an expert's segment of `expanded` and inside a rank's
 * segment of `recv`, rows are ordered by token, then by top-k slot.  The
 * result is deterministic and identical from run to run.
 *
 * Errors: arguments are validated on the host before anything is launched
 * (EP_ERR_INVALID_ARG / EP_ERR_MISALIGNED; nothing is written).  Problems only
 * the device can see -- an index < -1 or >= E, a destination row beyond a
 * caller's capacity -- never trap: the offending route or row is skipped, a
 * bit is set in the layout's device error word (totals[3]) and
 * ep_layout_read_totals reports it.  A failed launch returns EP_ERR_CUDA.
 */
#ifndef EPX_H
#define EPX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EPX_ABI_VERSION 3

#define EPX_MAX_TOPK 32      /* k <= 32: one warp holds a token's routes      */
#define EPX_MAX_RANKS 64     /* R <= 64: a token's rank set fits in 64 bits   */
#define EPX_MAX_EXPERTS 4096 /* E <= 4096: per-warp expert histograms in smem */

typedef enum ep_status {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1, /* bad size / null pointer / E % R != 0 ...       */
    EP_ERR_MISALIGNED = 2,  /* a row buffer is not 16-byte aligned            */
    EP_ERR_CAPACITY = 3,    /* device: a destination row exceeded a capacity  */
    EP_ERR_BAD_INDEX = 4,   /* device: a topk index < -1 or >= E was skipped  */
    EP_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed           */
    EP_ERR_UNSUPPORTED = 6  /* size beyond a documented limit (EPX_MAX_*, or  */
                            /* of a schedule chosen by a *_variant call)      */
} ep_status_t;

/* bits of the device error word, totals[3] */
#define EP_DEVERR_BAD_INDEX 0x1u
#define EP_DEVERR_RECV_CAP 0x2u
#define EP_DEVERR_EXP_CAP 0x4u
#define EP_DEVERR_Y_ROWS 0x8u
#define EP_DEVERR_TIMEOUT 0x10u /* a bounded wait on an async copy gave up */

/*
 * Routing layout ("handle" in the pages' dispatch/combine API).  Plain data;
 * every array is device memory inside one caller-owned block carved by
 * ep_layout_init.  All int32.
 *   cnt_e[E]      valid routes per expert
 *   off_e[E+1]    exclusive scan of cnt_e (expert e's rows in `expanded`
 *                 are [off_e[e], off_e[e+1]))
 *   cnt_r[R]      tokens received by rank r (a token counts once per rank)
 *   off_r[R+1]    exclusive scan of cnt_r (rank r's rows in `recv`)
 *   pos[T*k]      row of route (t, j) in `expanded`, -1 for no route
 *   recv_pos[T*R] row of token t in `recv` for rank r, -1 if not sent
 *   totals[4]     N_route = off_e[E], N_recv = off_r[R],
 *                 T_real = rows with >= 1 valid route, device error word
 *   work          workspace of the grid layout schedule: a header of
 *                 barrier words, then one row of counts per CTA.  The
 *                 header must be zero before the first ep_layout call on
 *                 the block (allocate it zeroed, or cudaMemset the block
 *                 once); every call leaves it zero again.
 */
typedef struct ep_layout {
    int32_t T, k, E, R;
    int32_t idx_bits; /* 32 or 64: width of the topk_idx elements */
    int32_t reserved;
    int32_t *cnt_e;
    int32_t *off_e;
    int32_t *cnt_r;
    int32_t *off_r;
    int32_t *pos;
    int32_t *recv_pos;
    int32_t *totals;
    int32_t *work;
} ep_layout_t;

/* ABI version of the loaded library (EPX_ABI_VERSION at build time). */
int32_t ep_abi_version(void);

/* Human-readable name of a status code; never NULL. */
const char *ep_status_str(ep_status_t status);

/* Device bytes ep_layout_init needs for a layout of these sizes; 0 if the
 * sizes are invalid or unsupported. */
size_t ep_layout_bytes(int32_t T, int32_t k, int32_t E, int32_t R);

/*
 * Fill *L by carving `dev_mem` (device, >= ep_layout_bytes(...) bytes,
 * 16-byte aligned).  Host-only: launches nothing, touches no device memory.
 * Requires T >= 0, 1 <= k <= EPX_MAX_TOPK, 1 <= R <= EPX_MAX_RANKS,
 * 1 <= E <= EPX_MAX_EXPERTS, E % R == 0, idx_bits in {32, 64}.
 */
ep_status_t ep_layout_init(ep_layout_t *L, int32_t T, int32_t k, int32_t E,
                           int32_t R, int32_t idx_bits, void *dev_mem,
                           size_t bytes);

/*
 * Routing layout from topk_idx (device, [T, k] row-major, int32 or int64 as
 * L->idx_bits says; -1 = no route).  Overwrites every array of *L, including
 * totals[3] (the error word is reset here).  Indices < -1 or >= E are
 * dropped and flagged EP_DEVERR_BAD_INDEX.  One launch: for up to a few
 * thousand routes one thread-block cluster whose CTAs share their counts
 * through distributed shared memory; for large batches a grid of up to one
 * CTA per SM whose CTAs share their counts through L->work behind one grid
 * barrier (a bounded wait: if it gives up, EP_DEVERR_TIMEOUT is set and
 * every pos of the CTA is -1).  Two calls on one layout block must not
 * overlap on the GPU.
 */
ep_status_t ep_layout(const void *topk_idx, const ep_layout_t *L, void *stream);

/* Same, choosing the schedule: 0 = automatic, 1 = warp chunks (each warp
 * takes whole tokens, one lane per route, and finds the lanes that share an
 * expert or a rank with one warp ballot per bit of the key;
 * EP_ERR_UNSUPPORTED when its per-warp count table does not
 * fit in shared memory or the CTA's tokens need more than four passes of
 * its warps), 2 = count matrix (one thread per token; any valid size),
 * 3 = grid of up to one CTA per SM (EP_ERR_UNSUPPORTED below two CTAs or
 * where its tables do not fit in shared memory).  Results are identical. */
ep_status_t ep_layout_variant(const void *topk_idx, const ep_layout_t *L,
                              int32_t variant, void *stream);

/*
 * Layout and dispatch + expand in one call: the same results as ep_layout
 * followed by ep_dispatch_expand with the same arguments (every array of *L,
 * recv, expanded and the error word).  For small batches (T*k up to
 * EPX_FUSED_MAX_ROUTES) it can run as ONE launch: every CTA derives its own
 * token's rows by counting over all routes (the batch's experts in a
 * shared-memory table, one thread per query of the token: a slot or a rank)
 * while its chunk of x is in flight, so nothing waits for a separate layout
 * kernel.  Otherwise it runs the layout
 * kernel and the dispatch kernel back to back; since the layout kernel lets
 * its successor start only once every earlier kernel on the stream has
 * completed, the dispatch launched here reads topk_idx and its first chunk
 * of x (for a token with a route) before waiting for the layout, so the
 * DRAM latency of x overlaps the layout.  variant: 0 = automatic (one
 * launch where it was measured faster, see EPX_FUSED_AUTO_MIN_ROUTES; else
 * two), 1 = one launch (EP_ERR_UNSUPPORTED beyond EPX_FUSED_MAX_ROUTES),
 * 2 = the two kernels.  Rows beyond a capacity are skipped and flagged
 * (EP_DEVERR_RECV_CAP / EP_DEVERR_EXP_CAP) as in ep_dispatch_expand.
 */
#define EPX_FUSED_MAX_ROUTES 4096
/* variant 0 takes one launch for T*k in [MIN, MAX]: measured on B200 it is
 * faster from one token (16 routes: 7.7 against 8.6 us per step) to 2048
 * routes; above that every CTA's count over all routes outweighs the launch
 * saved (2560 routes: 42.8 against 42.0 us) */
#define EPX_FUSED_AUTO_MIN_ROUTES 1
#define EPX_FUSED_AUTO_MAX_ROUTES 2048
ep_status_t ep_layout_dispatch_expand(const void *topk_idx, const ep_layout_t *L,
                                      const void *x, int32_t H, void *recv,
                                      int64_t recv_cap, void *expanded,
                                      int64_t exp_cap, void *stream);
ep_status_t ep_layout_dispatch_expand_variant(const void *topk_idx,
                                              const ep_layout_t *L, const void *x,
                                              int32_t H, void *recv,
                                              int64_t recv_cap, void *expanded,
                                              int64_t exp_cap, int32_t variant,
                                              void *stream);

/*
 * Dispatch + expand.  x: device bf16 [T, H] row-major (16-byte aligned,
 * H % 8 == 0).  Each token with >= 1 valid route is read once and written
 *   recv[recv_pos[t, r]]  = x[t] for every rank r it reaches, and
 *   expanded[pos[t, j]]   = x[t] for every valid route j.
 * recv: device bf16 [recv_cap, H]; expanded: device bf16 [exp_cap, H].
 * Worst-case capacities T*min(k, R) and T*k never overflow; a smaller
 * capacity is allowed, and rows beyond it are skipped and flagged.
 * Rows past N_recv / N_route are left untouched.  recv may be NULL with
 * recv_cap 0: only the expanded rows are written (the receiving side of a
 * multi-GPU dispatch, whose rows arrived already).
 */
ep_status_t ep_dispatch_expand(const void *x, int32_t H, const ep_layout_t *L,
                               void *recv, int64_t recv_cap, void *expanded,
                               int64_t exp_cap, void *stream);

/* Same, choosing the copy engine: 0 = automatic, 1 = 16-byte vector
 * loads/stores through registers, 2 = TMA bulk copies staged in shared
 * memory.  Results are identical. */
ep_status_t ep_dispatch_expand_variant(const void *x, int32_t H,
                                       const ep_layout_t *L, void *recv,
                                       int64_t recv_cap, void *expanded,
                                       int64_t exp_cap, int32_t variant,
                                       void *stream);

/*
 * Dispatch only (the pages' do_expand=False: DeepEP issue #760,
 * Reproduction): recv[recv_pos[t, r]] = x[t] for every rank r the token
 * reaches, and no expanded copy -- the VRAM side of the expand tradeoff
 * (DeepEP issue #48, answer on VRAM vs performance).  Arguments as in
 * ep_dispatch_expand.
 */
ep_status_t ep_dispatch(const void *x, int32_t H, const ep_layout_t *L, void *recv,
                        int64_t recv_cap, void *stream);

/*
 * Routing that travels with each sent row of a multi-GPU dispatch (one rank
 * per GPU, rank r owning experts [r*E/R, (r+1)*E/R)): a token goes once to
 * every rank that owns one of its experts together with its top-k routing
 * (DeepEP issue #48, question), and that rank expands it per local expert
 * and reduces the outputs before the combine travels back (issue #48,
 * answer on the reduction before the combine all2all).  For every
 * (token t, rank r) pair of the layout, row q = recv_pos[t, r] gets
 *   meta_idx[q, j] = topk_idx[t, j] if expert topk_idx[t, j] is on rank r,
 *                    else -1,
 *   meta_w[q, j]   = topk_weights[t, j] if so, else 0,
 * so the rows sent to rank r, with these as their routing, form a batch
 * whose routes all stay on rank r.  topk_idx: device [T, k] (L->idx_bits
 * wide); topk_weights: device fp32 [T, k]; meta_idx: device int32
 * [rows, k]; meta_w: device fp32 [rows, k]; rows >= N_recv (worst case
 * T*min(k, R)); a row >= rows is skipped and flagged EP_DEVERR_RECV_CAP.
 */
ep_status_t ep_route_meta(const void *topk_idx, const float *topk_weights,
                          const ep_layout_t *L, int32_t *meta_idx, float *meta_w,
                          int64_t rows, void *stream);

/*
 * Gather index for a consumer that reads the received rows directly:
 *   src_row[pos[t, j]] = recv_pos[t, rank(e_j)]   for every valid route,
 * i.e. the recv row that holds expanded row p's data.  src_row: device int32
 * [rows], rows >= N_route (worst case T*k); entries past N_route untouched;
 * a pos >= rows is skipped and flagged (EP_DEVERR_EXP_CAP).
 */
ep_status_t ep_expand_index(const ep_layout_t *L, int32_t *src_row, int64_t rows,
                            void *stream);

/*
 * The stand-in expert of ep_standin_expert reading recv[src_row[p]] in place
 * of expanded[p] (identical results, no expanded buffer): the pattern of a
 * grouped consumer of a dispatch without expand.  recv: device bf16
 * [recv_rows, H]; src_row from ep_expand_index; y: device bf16 [rows, H].
 */
ep_status_t ep_standin_expert_gather(const void *recv, int64_t recv_rows, int32_t H,
                                     const ep_layout_t *L, const int32_t *src_row,
                                     void *y, int64_t rows, void *stream);

/*
 * Deterministic stand-in for the expert FFN (test and benchmark helper):
 * y[p] = bf16_rn(float(expanded[p]) * (1 + e/E)) in IEEE fp32 for every row
 * p < N_route of expert e's segment.  expanded, y: device bf16 [rows, H],
 * rows >= N_route (rows beyond N_route are untouched).
 */
ep_status_t ep_standin_expert(const void *expanded, int32_t H,
                              const ep_layout_t *L, void *y, int64_t rows,
                              void *stream);

/*
 * Combine reduce.  expert_out: device bf16 [y_rows, H], row pos[t, j] holds
 * expert idx[t, j]'s output for token t.  topk_weights: device fp32 [T, k].
 *   out[t, h] = bf16_rn( sum over valid j in k order of
 *                        topk_weights[t, j] * expert_out[pos[t, j], h] )
 * accumulated in fp32; weights are used as given (no renormalisation);
 * a token with no valid route gives a row of +0.  out: device bf16 [T, H].
 * Work is split over the hidden dimension across CTAs when T is small, so
 * that a handful of tokens still spreads over all SMs.
 */
ep_status_t ep_combine_reduce(const void *expert_out, const float *topk_weights,
                              int32_t H, const ep_layout_t *L, void *out,
                              int64_t y_rows, void *stream);

/* Same, choosing the schedule: 0 = automatic, 1 = one warp per output token
 * (the DeepEP V2 epilogue's schedule, kept as a baseline), 2 = hidden
 * dimension split across CTAs.  Results are identical. */
ep_status_t ep_combine_reduce_variant(const void *expert_out,
                                      const float *topk_weights, int32_t H,
                                      const ep_layout_t *L, void *out,
                                      int64_t y_rows, int32_t variant,
                                      void *stream);

/*
 * Two-stage combine, first stage: the local reduce a rank runs before the
 * combine all2all (DeepEP issue #48, answer on the reduction kernel before
 * the combine all2all).  For every (token t, rank r) pair of the layout:
 *   partial[recv_pos[t, r], h] = sum over valid j whose expert lives on r,
 *                                in k order, of topk_weights[t, j] *
 *                                expert_out[pos[t, j], h]
 * accumulated in fp32 and stored as fp32 (partial_bits 32) or bf16 (16).
 * partial: device [partial_cap, H] in the receive layout (rank r's rows are
 * [off_r[r], off_r[r+1])); worst case partial_cap = T*min(k, R).  These rows
 * are what a consumer that takes over the epilogue receives (the "skip the
 * epilogue" option of DeepEP issue #760).  expert_out / topk_weights as in
 * ep_combine_reduce.
 */
ep_status_t ep_combine_local_reduce(const void *expert_out, const float *topk_weights,
                                    int32_t H, const ep_layout_t *L, void *partial,
                                    int64_t partial_cap, int32_t partial_bits,
                                    int64_t y_rows, void *stream);

/*
 * Two-stage combine, second stage: the combine epilogue (DeepEP issue #760,
 * combine_reduce_epilogue).  For every token:
 *   out[t, h] = bf16_rn( residual[t, h] + sum over ranks r with
 *                        recv_pos[t, r] >= 0, in rank order, of
 *                        partial[recv_pos[t, r], h] )
 * in fp32; residual (device bf16 [T, H], 16-byte aligned) may be NULL, which
 * drops that term -- the residual add is the downstream fusion the issue's
 * second proposal asks for.  out: device bf16 [T, H].
 */
ep_status_t ep_combine_epilogue(const void *partial, int32_t partial_bits, int32_t H,
                                const ep_layout_t *L, int64_t partial_cap,
                                const void *residual, void *out, void *stream);

/*
 * Copy the layout's totals to the host and synchronise `stream`.  Any
 * pointer may be NULL.  Returns EP_ERR_BAD_INDEX or EP_ERR_CAPACITY when
 * the device error word has the matching bit set (the totals are still
 * written), EP_ERR_CUDA if the copy or an earlier launch failed.
 */
ep_status_t ep_layout_read_totals(const ep_layout_t *L, int64_t *n_route,
                                  int64_t *n_recv, int64_t *t_real,
                                  int32_t *dev_err, void *stream);

/*
 * End-to-end pass from host buffers: copies x (bf16 [T, H]), topk_idx
 * ([T, k], idx_bits wide) and topk_weights (fp32 [T, k]) from host memory
 * (pinned for asynchronous copies), runs layout, dispatch/expand, the
 * stand-in expert and combine on the device, and copies out (bf16 [T, H])
 * back to host memory.  dev_mem: caller-owned device scratch of at least
 * ep_roundtrip_device_bytes(...) bytes, 256-byte aligned.  dev_err_host
 * (host, may be NULL) receives the layout's device error word (EP_DEVERR_*
 * bits; nonzero when a route or a row was dropped, e.g. an index >= E) --
 * the status returned here only covers what the host can check before the
 * work runs.  Asynchronous: the caller synchronises `stream` before reading
 * out_host or *dev_err_host.
 */
size_t ep_roundtrip_device_bytes(int32_t T, int32_t H, int32_t k, int32_t E,
                                 int32_t R, int32_t idx_bits);
ep_status_t ep_roundtrip_host(const void *x_host, const void *topk_idx_host,
                              const float *topk_weights_host, int32_t T,
                              int32_t H, int32_t k, int32_t E, int32_t R,
                              int32_t idx_bits, void *dev_mem, size_t bytes,
                              void *out_host, int32_t *dev_err_host,
                              void *stream);

/*
 * Host round trip that allocates nothing.  The pages have no counterpart:
 * this entry point serves callers that cannot allocate device memory when
 * they need a pass -- code running while another component owns the device
 * allocator (a caching allocator or a pool fixed at start-up), plugins
 * loaded into a host that forbids allocation after initialisation, latency
 * paths that cannot afford an allocation's implicit synchronisation.
 *
 * Same arguments and result as ep_roundtrip_host (including the optional
 * dev_err_host error word), minus dev_mem/bytes: the
 * device scratch is a fixed array of EPX_NOALLOC_SCRATCH_BYTES inside this
 * library, which every GPU that loads the library holds until the process
 * exits.  Sizes whose ep_roundtrip_device_bytes(...) exceeds it return
 * EP_ERR_UNSUPPORTED and launch nothing (64 MiB covers, for example,
 * 128 tokens of hidden 7168 with top-8, or 8 tokens of hidden 3584 with
 * top-16).  No cudaMalloc, cudaFree or other allocating call is made.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the
 * life of the process; make that first call before any stream capture.
 * cudaDeviceReset destroys the context that address belongs to, so this
 * entry point must not be used in a process after a device reset.  All calls share the array and it keeps the
 * last call's contents (nothing in it needs to start at zero); calls whose
 * device work overlaps -- on different streams or from different host
 * threads -- race on it, so order them on one stream or synchronise.
 */
#define EPX_NOALLOC_SCRATCH_BYTES (64u << 20)
ep_status_t ep_roundtrip_host_noalloc(const void *x_host, const void *topk_idx_host,
                                      const float *topk_weights_host, int32_t T,
                                      int32_t H, int32_t k, int32_t E, int32_t R,
                                      int32_t idx_bits, void *out_host,
                                      int32_t *dev_err_host, void *stream);

/* ------------------------------------------------------------------------
 * Multi-GPU expert parallelism over peer memory (one process per GPU, rank r
 * owning experts [r*E/R, (r+1)*E/R)): a token crosses to every rank that owns
 * one of its experts exactly once, with its routing (DeepEP issue #48,
 * question: token A on rank 0 "dispatched only once" to rank 1 for experts M
 * and N), and the per-rank partial sums travel back (issue #48, answer on the
 * reduction before the combine all2all).  The kernels below store those rows
 * straight into the other GPUs' buffers (plain 16-byte stores through device
 * pointers that map a peer's memory into this process, e.g. from
 * ep_ipc_open; never a TMA copy): the placement of each row and the
 * transfer are one kernel, in place of a dispatch kernel followed by an
 * all-to-all.  The caller orders the ranks around them: all ranks' stores
 * must have completed before a receiver reads its buffers (e.g. a one-word
 * collective on every rank's stream after the kernel).  Nothing here waits
 * on another GPU, so a rank that fails cannot leave a kernel spinning.
 *
 * One entry per peer (index = rank), host array of L->R entries:
 */
typedef struct {
    void *rows;         /* device pointer (mapped peer memory or local): bf16
                           [cap, H] rows for the dispatch, fp32 or bf16
                           [cap, H] partial rows for the combine; 16-byte
                           aligned */
    int32_t *meta_idx;  /* dispatch: int32 [cap, k] routes kept on that rank
                           (NULL: not written); combine: unused */
    float *meta_w;      /* dispatch: fp32 [cap, k] their weights (NULL: not
                           written); combine: unused */
    int64_t row0;       /* first row this rank writes there */
    int64_t cap;        /* rows the buffers hold; a row >= cap is skipped and
                           flagged EP_DEVERR_RECV_CAP */
    int64_t first;      /* combine: first local partial row that goes there */
    int64_t count;      /* combine: partial rows that go there */
} ep_peer_rows_t;

/*
 * Dispatch to peers: for every token t with a route on rank r (recv_pos[t,
 * r] >= 0 in the layout *L of this rank's batch over R ranks), the row
 *   q = peers[r].row0 + (recv_pos[t, r] - off_r[r])
 * of rank r's buffers gets
 *   rows[q]        = x[t]                           (bf16 [H]),
 *   meta_idx[q, j] = topk_idx[t, j] if expert topk_idx[t, j] is on rank r,
 *                    else -1,          meta_w[q, j] = its weight, else 0,
 * i.e. what ep_dispatch + ep_route_meta would write into this rank's send
 * buffer, stored instead at this source's place in the receiver's buffer
 * (peers[r].row0 = the rows rank r receives from lower ranks).  Per rank r
 * the received rows are then ordered by source rank, then by the source's
 * token order.  x: device bf16 [T, H]; topk_idx / topk_weights as in
 * ep_route_meta; the layout must come from ep_layout (or
 * ep_layout_dispatch_expand) of the same topk_idx with R = the number of
 * ranks.  The kernel ends with a system-scope fence.
 */
ep_status_t ep_dispatch_p2p(const void *x, int32_t H, const ep_layout_t *L,
                            const void *topk_idx, const float *topk_weights,
                            const ep_peer_rows_t *peers, void *stream);

/*
 * Local reduce to peers: ep_combine_local_reduce of the receiving rank, with
 * each partial row stored at its source instead of locally: partial row d
 * (in the receive layout of *L) with peers[s].first <= d < peers[s].first +
 * peers[s].count goes to row peers[s].row0 + (d - peers[s].first) of
 * peers[s].rows.  Arithmetic identical to ep_combine_local_reduce (fp32
 * sums in k order, stored fp32 or bf16); a row that falls in no entry's
 * range, or beyond its cap, is skipped and flagged EP_DEVERR_RECV_CAP.
 * For the source, its partial rows then sit in its own receive layout, so
 * ep_combine_epilogue applies unchanged.  The kernel ends with a
 * system-scope fence.
 */
ep_status_t ep_combine_local_reduce_p2p(const void *expert_out, const float *topk_weights,
                                        int32_t H, const ep_layout_t *L,
                                        int32_t partial_bits, int64_t y_rows,
                                        const ep_peer_rows_t *peers, void *stream);

/*
 * Device memory other processes can map (cudaIpcGetMemHandle /
 * cudaIpcOpenMemHandle on an allocation of this library's own, so the
 * handle covers exactly the buffer).  ep_ipc_malloc: bytes of device memory
 * on the current device, its pointer in *dev_ptr and its handle in
 * handle[0..EPX_IPC_HANDLE_BYTES).  ep_ipc_open: maps another process's
 * handle into this one (peer access must be possible; the same process
 * cannot open its own handle), pointer in *dev_ptr.  ep_ipc_close /
 * ep_ipc_free undo them.  Errors: EP_ERR_INVALID_ARG, EP_ERR_CUDA.
 */
#define EPX_IPC_HANDLE_BYTES 64
ep_status_t ep_ipc_malloc(size_t bytes, void **dev_ptr, void *handle);
ep_status_t ep_ipc_free(void *dev_ptr);
ep_status_t ep_ipc_open(const void *handle, void **dev_ptr);
ep_status_t ep_ipc_close(void *dev_ptr);

/*
 * Measurement helper: the latency floor of a step of this path.  Launches
 * n_kernels (1..64) one-warp kernels on `stream`, chained like the path's
 * kernels (programmatic dependent launch), each loading one word of `buf`
 * after its predecessor has finished and storing one word -- the skeleton
 * of the low-batch step (launches, hand-offs, one DRAM round trip per
 * kernel) with no work in it.  buf: device int32, at least
 * 64 * (2 * n_kernels + 2) words, 16-byte aligned; its contents are
 * irrelevant and get overwritten.
 */
ep_status_t ep_latency_floor(int32_t *buf, int64_t buf_words, int32_t n_kernels,
                             void *stream);

/*
 * Test setting (not needed by any caller of the path): the number of polls
 * the first bounded wait of every CTA of the bulk copy engine
 * (ep_dispatch_expand_variant(..., 2, ...)) may take before it gives up,
 * for later launches from this process; negative restores the normal limit.
 * With 0 every CTA gives up at once: it flags EP_DEVERR_TIMEOUT, waits
 * (bounded) for its copy in flight, and leaves its rows unwritten, so
 * ep_layout_read_totals returns EP_ERR_CUDA -- the path that a copy which
 * never completes would take, exercised without a stuck copy.
 */
void ep_debug_dispatch_first_wait_limit(int64_t limit);

#ifdef __cplusplus
}
#endif

#endif /* EPX_H */
