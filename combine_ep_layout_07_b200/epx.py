"""Thin ctypes binding of libepx.so (the C ABI declared in include/epx.h).

Argument marshalling only: torch provides device memory and the current CUDA
stream, every step of the path runs in the library's CUDA kernels.  There is
no CPU fallback: if libepx.so is missing or no CUDA device is present, every
call raises.

Functions mirror the C entry points:

    lay = layout(topk_idx, num_experts, num_ranks)
    recv, expanded = dispatch_expand(x, lay)
    y = standin_expert(expanded, lay)                 # test / bench helper
    out = combine_reduce(y, topk_weights, lay)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "EpxError", "Layout", "lib", "layout", "dispatch_expand", "standin_expert",
    "combine_reduce", "combine_local_reduce", "combine_epilogue", "read_totals",
    "dispatch", "expand_index", "standin_expert_gather", "layout_dispatch_expand",
    "latency_floor", "route_meta", "PeerRows", "dispatch_p2p", "combine_local_reduce_p2p",
    "ipc_malloc", "ipc_free", "ipc_open", "ipc_close", "tensor_at", "IPC_HANDLE_BYTES",
    "roundtrip_host", "roundtrip_device_bytes",
    "roundtrip_host_noalloc", "NOALLOC_SCRATCH_BYTES", "debug_dispatch_first_wait_limit",
    "LIB_PATH", "MAX_TOPK", "MAX_RANKS", "MAX_EXPERTS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libepx.so")
MAX_TOPK, MAX_RANKS, MAX_EXPERTS = 32, 64, 4096
NOALLOC_SCRATCH_BYTES = 64 << 20  # EPX_NOALLOC_SCRATCH_BYTES
FUSED_MAX_ROUTES = 4096           # EPX_FUSED_MAX_ROUTES
FUSED_AUTO_MIN_ROUTES = 1         # EPX_FUSED_AUTO_MIN_ROUTES
FUSED_AUTO_MAX_ROUTES = 2048      # EPX_FUSED_AUTO_MAX_ROUTES

EP_OK = 0
_STATUS = {0: "EP_OK", 1: "EP_ERR_INVALID_ARG", 2: "EP_ERR_MISALIGNED", 3: "EP_ERR_CAPACITY",
           4: "EP_ERR_BAD_INDEX", 5: "EP_ERR_CUDA", 6: "EP_ERR_UNSUPPORTED"}


class EpxError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        msg = lib().ep_status_str(int(status)).decode() if _lib is not None else _STATUS.get(status)
        super().__init__(f"{what}: {msg}")


class _LayoutC(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("k", ctypes.c_int32), ("E", ctypes.c_int32),
                ("R", ctypes.c_int32), ("idx_bits", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("cnt_e", ctypes.c_void_p), ("off_e", ctypes.c_void_p),
                ("cnt_r", ctypes.c_void_p), ("off_r", ctypes.c_void_p),
                ("pos", ctypes.c_void_p), ("recv_pos", ctypes.c_void_p),
                ("totals", ctypes.c_void_p), ("work", ctypes.c_void_p)]


class _PeerRowsC(ctypes.Structure):
    """ep_peer_rows_t."""
    _fields_ = [("rows", ctypes.c_void_p), ("meta_idx", ctypes.c_void_p),
                ("meta_w", ctypes.c_void_p), ("row0", ctypes.c_int64), ("cap", ctypes.c_int64),
                ("first", ctypes.c_int64), ("count", ctypes.c_int64)]


IPC_HANDLE_BYTES = 64             # EPX_IPC_HANDLE_BYTES

_lib = None


def lib():
    """Load libepx.so once; raise if it is missing (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libepx.so not built ({LIB_PATH}); run `python -m combine_ep_layout_07_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    LP = ctypes.POINTER(_LayoutC)
    sig = {
        "ep_abi_version": ([], I32),
        "ep_status_str": ([I32], ctypes.c_char_p),
        "ep_layout_bytes": ([I32, I32, I32, I32], SZ),
        "ep_layout_init": ([LP, I32, I32, I32, I32, I32, P, SZ], I32),
        "ep_layout": ([P, LP, P], I32),
        "ep_layout_variant": ([P, LP, I32, P], I32),
        "ep_dispatch_expand": ([P, I32, LP, P, I64, P, I64, P], I32),
        "ep_dispatch_expand_variant": ([P, I32, LP, P, I64, P, I64, I32, P], I32),
        "ep_standin_expert": ([P, I32, LP, P, I64, P], I32),
        "ep_combine_reduce": ([P, P, I32, LP, P, I64, P], I32),
        "ep_combine_reduce_variant": ([P, P, I32, LP, P, I64, I32, P], I32),
        "ep_dispatch": ([P, I32, LP, P, I64, P], I32),
        "ep_expand_index": ([LP, P, I64, P], I32),
        "ep_standin_expert_gather": ([P, I64, I32, LP, P, P, I64, P], I32),
        "ep_combine_local_reduce": ([P, P, I32, LP, P, I64, I32, I64, P], I32),
        "ep_combine_epilogue": ([P, I32, I32, LP, I64, P, P, P], I32),
        "ep_layout_read_totals": ([LP, ctypes.POINTER(I64), ctypes.POINTER(I64),
                                   ctypes.POINTER(I64), ctypes.POINTER(I32), P], I32),
        "ep_roundtrip_device_bytes": ([I32, I32, I32, I32, I32, I32], SZ),
        "ep_roundtrip_host": ([P, P, P, I32, I32, I32, I32, I32, I32, P, SZ, P,
                               ctypes.POINTER(I32), P], I32),
        "ep_roundtrip_host_noalloc": ([P, P, P, I32, I32, I32, I32, I32, I32, P,
                                       ctypes.POINTER(I32), P], I32),
        "ep_debug_dispatch_first_wait_limit": ([I64], None),
        "ep_layout_dispatch_expand": ([P, LP, P, I32, P, I64, P, I64, P], I32),
        "ep_layout_dispatch_expand_variant": ([P, LP, P, I32, P, I64, P, I64, I32, P], I32),
        "ep_latency_floor": ([P, I64, I32, P], I32),
        "ep_route_meta": ([P, P, LP, P, P, I64, P], I32),
        "ep_dispatch_p2p": ([P, I32, LP, P, P, ctypes.POINTER(_PeerRowsC), P], I32),
        "ep_combine_local_reduce_p2p": ([P, P, I32, LP, I32, I64, ctypes.POINTER(_PeerRowsC),
                                         P], I32),
        "ep_ipc_malloc": ([SZ, ctypes.POINTER(P), P], I32),
        "ep_ipc_free": ([P], I32),
        "ep_ipc_open": ([P, ctypes.POINTER(P)], I32),
        "ep_ipc_close": ([P], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _check(status: int, what: str):
    if status != EP_OK:
        raise EpxError(status, what)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise TypeError(f"{name} has dtype {t.dtype}")
    return t.data_ptr() if t.numel() else None


class Layout:
    """Routing layout ("handle"): owns one device block holding every array."""

    def __init__(self, T: int, k: int, E: int, R: int, idx_bits: int = 64, device=None):
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        nbytes = lib().ep_layout_bytes(T, k, E, R)
        if nbytes == 0:
            raise EpxError(6 if (k > MAX_TOPK or R > MAX_RANKS or E > MAX_EXPERTS) else 1,
                           f"ep_layout_bytes(T={T}, k={k}, E={E}, R={R})")
        # zeroed: the grid layout schedule's barrier words start at zero
        self.mem = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.c = _LayoutC()
        _check(lib().ep_layout_init(ctypes.byref(self.c), T, k, E, R, idx_bits,
                                    self.mem.data_ptr(), nbytes), "ep_layout_init")
        self.T, self.k, self.E, self.R, self.idx_bits = T, k, E, R, idx_bits
        base = self.mem.data_ptr()

        def view(ptr, n):
            off = ptr - base
            return self.mem[off:off + 4 * n].view(torch.int32)

        self.cnt_e = view(self.c.cnt_e, E)
        self.off_e = view(self.c.off_e, E + 1)
        self.cnt_r = view(self.c.cnt_r, R)
        self.off_r = view(self.c.off_r, R + 1)
        self.pos = view(self.c.pos, T * k).view(T, k)
        self.recv_pos = view(self.c.recv_pos, T * R).view(T, R)
        self.totals = view(self.c.totals, 4)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    @property
    def recv_cap(self) -> int:
        return self.T * min(self.k, self.R)

    @property
    def exp_cap(self) -> int:
        return self.T * self.k


def layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, out: Layout = None,
           variant: int = 0, stream=None) -> Layout:
    """ep_layout: routing layout of topk_idx (int32 or int64 [T, k], -1 = none).
    variant: 0 automatic, 1 warp chunks, 2 count matrix, 3 grid of up to one
    CTA per SM (same results)."""
    if topk_idx.dim() != 2:
        raise ValueError("topk_idx must be [T, k]")
    T, k = topk_idx.shape
    bits = {torch.int64: 64, torch.int32: 32}.get(topk_idx.dtype)
    if bits is None:
        raise TypeError("topk_idx must be int32 or int64")
    ptr = _dev(topk_idx, "topk_idx")
    lay = out if out is not None else Layout(T, k, num_experts, num_ranks, bits,
                                             device=topk_idx.device)
    if (lay.T, lay.k, lay.E, lay.R, lay.idx_bits) != (T, k, num_experts, num_ranks, bits):
        raise ValueError("layout buffer does not match the sizes")
    _check(lib().ep_layout_variant(ptr, lay.ref, variant, _stream(stream)), "ep_layout")
    return lay


def dispatch_expand(x: torch.Tensor, lay: Layout, recv: torch.Tensor = None,
                    expanded: torch.Tensor = None, variant: int = 0, stream=None,
                    expand_only: bool = False):
    """ep_dispatch_expand: returns (recv [T*min(k,R), H], expanded [T*k, H]) bf16;
    rows past N_recv / N_route are left as allocated.  expand_only: no recv
    copy (recv is None in the result)."""
    if x.dim() != 2 or x.shape[0] != lay.T:
        raise ValueError("x must be [T, H]")
    H = x.shape[1]
    xp = _dev(x, "x", torch.bfloat16)
    if recv is None and not expand_only:
        recv = torch.empty((lay.recv_cap, H), dtype=torch.bfloat16, device=x.device)
    if expanded is None:
        expanded = torch.empty((lay.exp_cap, H), dtype=torch.bfloat16, device=x.device)
    for name, t in (("recv", recv), ("expanded", expanded)):
        if t is not None and (t.dim() != 2 or t.shape[1] != H):
            raise ValueError(f"{name} must be [rows, {H}]")
    _check(lib().ep_dispatch_expand_variant(
        xp, H, lay.ref, None if recv is None else _dev(recv, "recv", torch.bfloat16),
        0 if recv is None else recv.shape[0],
        _dev(expanded, "expanded", torch.bfloat16), expanded.shape[0], variant,
        _stream(stream)), "ep_dispatch_expand")
    return recv, expanded


def layout_dispatch_expand(topk_idx: torch.Tensor, x: torch.Tensor, num_experts: int,
                           num_ranks: int, out: Layout = None, recv: torch.Tensor = None,
                           expanded: torch.Tensor = None, variant: int = 0, stream=None):
    """ep_layout_dispatch_expand: layout + dispatch/expand in one call (one
    launch for small batches).  Returns (layout, recv, expanded); the same
    results as layout() followed by dispatch_expand().
    variant: 0 automatic, 1 one launch, 2 two launches."""
    if topk_idx.dim() != 2:
        raise ValueError("topk_idx must be [T, k]")
    T, k = topk_idx.shape
    bits = {torch.int64: 64, torch.int32: 32}.get(topk_idx.dtype)
    if bits is None:
        raise TypeError("topk_idx must be int32 or int64")
    if x.dim() != 2 or x.shape[0] != T:
        raise ValueError("x must be [T, H]")
    H = x.shape[1]
    lay = out if out is not None else Layout(T, k, num_experts, num_ranks, bits,
                                             device=topk_idx.device)
    if (lay.T, lay.k, lay.E, lay.R, lay.idx_bits) != (T, k, num_experts, num_ranks, bits):
        raise ValueError("layout buffer does not match the sizes")
    if recv is None:
        recv = torch.empty((lay.recv_cap, H), dtype=torch.bfloat16, device=x.device)
    if expanded is None:
        expanded = torch.empty((lay.exp_cap, H), dtype=torch.bfloat16, device=x.device)
    for name, t in (("recv", recv), ("expanded", expanded)):
        if t.dim() != 2 or t.shape[1] != H:
            raise ValueError(f"{name} must be [rows, {H}]")
    _check(lib().ep_layout_dispatch_expand_variant(
        _dev(topk_idx, "topk_idx"), lay.ref, _dev(x, "x", torch.bfloat16), H,
        _dev(recv, "recv", torch.bfloat16), recv.shape[0],
        _dev(expanded, "expanded", torch.bfloat16), expanded.shape[0], variant,
        _stream(stream)), "ep_layout_dispatch_expand")
    return lay, recv, expanded


def route_meta(topk_idx: torch.Tensor, topk_weights: torch.Tensor, lay: Layout,
               meta_idx: torch.Tensor = None, meta_w: torch.Tensor = None, stream=None):
    """ep_route_meta: per sent row (recv_pos order), the token's routes kept on
    the destination rank (int32 expert ids, -1 elsewhere) and their weights
    (0 elsewhere).  Returns (meta_idx [rows, k] int32, meta_w [rows, k] fp32)."""
    if topk_idx.shape != (lay.T, lay.k) or topk_weights.shape != (lay.T, lay.k):
        raise ValueError("topk_idx and topk_weights must be [T, k]")
    dev = topk_idx.device
    if meta_idx is None:
        meta_idx = torch.empty((lay.recv_cap, lay.k), dtype=torch.int32, device=dev)
    if meta_w is None:
        meta_w = torch.empty((lay.recv_cap, lay.k), dtype=torch.float32, device=dev)
    if meta_idx.shape[1:] != (lay.k,) or meta_w.shape != meta_idx.shape:
        raise ValueError("meta buffers must be [rows, k]")
    _check(lib().ep_route_meta(_dev(topk_idx, "topk_idx", (torch.int32, torch.int64)),
                               _dev(topk_weights, "topk_weights", torch.float32), lay.ref,
                               _dev(meta_idx, "meta_idx", torch.int32),
                               _dev(meta_w, "meta_w", torch.float32), meta_idx.shape[0],
                               _stream(stream)), "ep_route_meta")
    return meta_idx, meta_w


class PeerRows:
    """One peer's buffers for ep_dispatch_p2p / ep_combine_local_reduce_p2p:
    `rows` (and, for the dispatch, `meta_idx` / `meta_w`) as CUDA tensors or
    raw device pointers (ints, e.g. from ipc_open), the first row this rank
    writes there (`row0`), the rows the buffers hold (`cap`) and, for the
    combine, the local partial rows [first, first + count) that go there."""

    def __init__(self, rows, cap: int, row0: int = 0, meta_idx=None, meta_w=None,
                 first: int = 0, count: int = 0):
        self.rows, self.cap, self.row0 = rows, int(cap), int(row0)
        self.meta_idx, self.meta_w = meta_idx, meta_w
        self.first, self.count = int(first), int(count)


def _ptr(v, name):
    if v is None:
        return None
    if isinstance(v, torch.Tensor):
        return _dev(v, name)
    return int(v)


def _peers_c(peers, R: int):
    if len(peers) != R:
        raise ValueError(f"{len(peers)} peer entries for {R} ranks")
    arr = (_PeerRowsC * R)()
    for r, e in enumerate(peers):
        arr[r].rows = _ptr(e.rows, f"peers[{r}].rows")
        arr[r].meta_idx = _ptr(e.meta_idx, f"peers[{r}].meta_idx")
        arr[r].meta_w = _ptr(e.meta_w, f"peers[{r}].meta_w")
        arr[r].row0, arr[r].cap = e.row0, e.cap
        arr[r].first, arr[r].count = e.first, e.count
    return arr


def dispatch_p2p(x: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                 lay: Layout, peers, stream=None) -> None:
    """ep_dispatch_p2p: every (token, rank) row of this rank's layout stored,
    with its routing kept on that rank, at peers[r].row0 + (recv_pos[t, r] -
    off_r[r]) of rank r's buffers."""
    if x.dim() != 2 or x.shape[0] != lay.T:
        raise ValueError("x must be [T, H]")
    if topk_idx.shape != (lay.T, lay.k) or topk_weights.shape != (lay.T, lay.k):
        raise ValueError("topk_idx and topk_weights must be [T, k]")
    arr = _peers_c(peers, lay.R)
    _check(lib().ep_dispatch_p2p(_dev(x, "x", torch.bfloat16), x.shape[1], lay.ref,
                                 _dev(topk_idx, "topk_idx", (torch.int32, torch.int64)),
                                 _dev(topk_weights, "topk_weights", torch.float32), arr,
                                 _stream(stream)), "ep_dispatch_p2p")


def combine_local_reduce_p2p(expert_out: torch.Tensor, topk_weights: torch.Tensor, lay: Layout,
                             peers, partial_dtype=torch.float32, stream=None) -> None:
    """ep_combine_local_reduce_p2p: the local reduce of ep_combine_local_reduce
    with partial row d stored at row peers[s].row0 + (d - peers[s].first) of
    peers[s].rows for the entry whose [first, first + count) holds d."""
    if topk_weights.shape != (lay.T, lay.k):
        raise ValueError("topk_weights must be [T, k]")
    bits = {torch.float32: 32, torch.bfloat16: 16}[partial_dtype]
    arr = _peers_c(peers, lay.R)
    _check(lib().ep_combine_local_reduce_p2p(
        _dev(expert_out, "expert_out", torch.bfloat16),
        _dev(topk_weights, "topk_weights", torch.float32), expert_out.shape[1], lay.ref, bits,
        expert_out.shape[0], arr, _stream(stream)), "ep_combine_local_reduce_p2p")


def ipc_malloc(nbytes: int):
    """ep_ipc_malloc: (device pointer, handle bytes) of a new allocation."""
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().ep_ipc_malloc(nbytes, ctypes.byref(ptr), handle), "ep_ipc_malloc")
    return ptr.value, handle.raw


def ipc_free(ptr: int) -> None:
    _check(lib().ep_ipc_free(ptr), "ep_ipc_free")


def ipc_open(handle: bytes) -> int:
    """ep_ipc_open: another process's allocation mapped into this one."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("IPC handle must be IPC_HANDLE_BYTES long")
    ptr = ctypes.c_void_p()
    _check(lib().ep_ipc_open(handle, ctypes.byref(ptr)), "ep_ipc_open")
    return ptr.value


def ipc_close(ptr: int) -> None:
    _check(lib().ep_ipc_close(ptr), "ep_ipc_close")


class _DevArray:
    """A raw device pointer with shape and dtype, for torch.as_tensor (bf16
    travels as int16 and is viewed back)."""

    _TYPESTR = {torch.bfloat16: "<i2", torch.float32: "<f4", torch.int32: "<i4"}

    def __init__(self, ptr: int, shape, dtype):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": self._TYPESTR[dtype],
                                         "data": (int(ptr), False), "version": 3}


def tensor_at(ptr: int, shape, dtype, device) -> torch.Tensor:
    """A tensor view of device memory at `ptr` (not owned: the caller keeps
    the allocation alive)."""
    raw = torch.as_tensor(_DevArray(ptr, shape, dtype), device=device)
    return raw.view(torch.bfloat16) if dtype == torch.bfloat16 else raw


def latency_floor(buf: torch.Tensor, n_kernels: int = 3, stream=None) -> None:
    """ep_latency_floor: n chained one-warp kernels, one dependent load each."""
    _check(lib().ep_latency_floor(_dev(buf, "buf", torch.int32), buf.numel(), n_kernels,
                                  _stream(stream)), "ep_latency_floor")


def dispatch(x: torch.Tensor, lay: Layout, recv: torch.Tensor = None, stream=None):
    """ep_dispatch: recv rows only (no expanded copy); returns recv [T*min(k,R), H]."""
    if x.dim() != 2 or x.shape[0] != lay.T:
        raise ValueError("x must be [T, H]")
    H = x.shape[1]
    if recv is None:
        recv = torch.empty((lay.recv_cap, H), dtype=torch.bfloat16, device=x.device)
    _check(lib().ep_dispatch(_dev(x, "x", torch.bfloat16), H, lay.ref,
                             _dev(recv, "recv", torch.bfloat16), recv.shape[0], _stream(stream)),
           "ep_dispatch")
    return recv


def expand_index(lay: Layout, src: torch.Tensor = None, stream=None):
    """ep_expand_index: int32 [T*k] recv row serving each expanded row."""
    if src is None:
        src = torch.empty((lay.exp_cap,), dtype=torch.int32, device=lay.mem.device)
    _check(lib().ep_expand_index(lay.ref, _dev(src, "src", torch.int32), src.shape[0],
                                 _stream(stream)), "ep_expand_index")
    return src


def standin_expert_gather(recv: torch.Tensor, lay: Layout, src: torch.Tensor,
                          y: torch.Tensor = None, stream=None):
    """ep_standin_expert_gather: the stand-in expert reading recv[src[p]]."""
    H = recv.shape[1]
    if y is None:
        y = torch.empty((lay.exp_cap, H), dtype=torch.bfloat16, device=recv.device)
    _check(lib().ep_standin_expert_gather(_dev(recv, "recv", torch.bfloat16), recv.shape[0], H,
                                          lay.ref, _dev(src, "src", torch.int32),
                                          _dev(y, "y", torch.bfloat16),
                                          min(src.shape[0], y.shape[0]), _stream(stream)),
           "ep_standin_expert_gather")
    return y


def standin_expert(expanded: torch.Tensor, lay: Layout, y: torch.Tensor = None, stream=None):
    """ep_standin_expert: y[p] = bf16(float(expanded[p]) * (1 + e/E)) for p < N_route."""
    H = expanded.shape[1]
    if y is None:
        y = torch.empty_like(expanded)
    _check(lib().ep_standin_expert(_dev(expanded, "expanded", torch.bfloat16), H, lay.ref,
                                   _dev(y, "y", torch.bfloat16),
                                   min(expanded.shape[0], y.shape[0]), _stream(stream)),
           "ep_standin_expert")
    return y


def combine_reduce(expert_out: torch.Tensor, topk_weights: torch.Tensor, lay: Layout,
                   out: torch.Tensor = None, variant: int = 0, stream=None):
    """ep_combine_reduce: out[t] = bf16(sum_j w[t,j] * expert_out[pos[t,j]])."""
    H = expert_out.shape[1]
    if topk_weights.shape != (lay.T, lay.k):
        raise ValueError("topk_weights must be [T, k]")
    if out is None:
        out = torch.empty((lay.T, H), dtype=torch.bfloat16, device=expert_out.device)
    _check(lib().ep_combine_reduce_variant(
        _dev(expert_out, "expert_out", torch.bfloat16), _dev(topk_weights, "topk_weights",
                                                              torch.float32),
        H, lay.ref, _dev(out, "out", torch.bfloat16), expert_out.shape[0], variant,
        _stream(stream)), "ep_combine_reduce")
    return out


def combine_local_reduce(expert_out: torch.Tensor, topk_weights: torch.Tensor, lay: Layout,
                         partial: torch.Tensor = None, partial_dtype=torch.float32,
                         stream=None):
    """ep_combine_local_reduce: one partial row per (token, rank) in the
    receive layout, [T*min(k,R), H] fp32 or bf16 (rows past N_recv untouched)."""
    H = expert_out.shape[1]
    if topk_weights.shape != (lay.T, lay.k):
        raise ValueError("topk_weights must be [T, k]")
    if partial is None:
        partial = torch.empty((lay.recv_cap, H), dtype=partial_dtype, device=expert_out.device)
    bits = {torch.float32: 32, torch.bfloat16: 16}[partial.dtype]
    _check(lib().ep_combine_local_reduce(
        _dev(expert_out, "expert_out", torch.bfloat16),
        _dev(topk_weights, "topk_weights", torch.float32), H, lay.ref,
        _dev(partial, "partial"), partial.shape[0], bits, expert_out.shape[0],
        _stream(stream)), "ep_combine_local_reduce")
    return partial


def combine_epilogue(partial: torch.Tensor, lay: Layout, residual: torch.Tensor = None,
                     out: torch.Tensor = None, stream=None):
    """ep_combine_epilogue: out[t] = bf16(residual[t] + sum of t's partial rows)."""
    H = partial.shape[1]
    bits = {torch.float32: 32, torch.bfloat16: 16}[partial.dtype]
    if out is None:
        out = torch.empty((lay.T, H), dtype=torch.bfloat16, device=partial.device)
    res = None if residual is None else _dev(residual, "residual", torch.bfloat16)
    _check(lib().ep_combine_epilogue(_dev(partial, "partial"), bits, H, lay.ref,
                                     partial.shape[0], res, _dev(out, "out", torch.bfloat16),
                                     _stream(stream)), "ep_combine_epilogue")
    return out


def read_totals(lay: Layout, stream=None, raise_on_error: bool = True) -> dict:
    """ep_layout_read_totals (synchronises the stream)."""
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    e = ctypes.c_int32()
    st = lib().ep_layout_read_totals(lay.ref, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c),
                                     ctypes.byref(e), _stream(stream))
    if raise_on_error:
        _check(st, "ep_layout_read_totals")
    return dict(N_route=a.value, N_recv=b.value, T_real=c.value, dev_err=e.value, status=st)


def roundtrip_device_bytes(T, H, k, E, R, idx_bits=64) -> int:
    return int(lib().ep_roundtrip_device_bytes(T, H, k, E, R, idx_bits))


def _host_roundtrip_args(x_host, idx_host, w_host, out_host):
    """Shapes and dtypes of the host buffers of a round trip (the C call
    trusts them: out_host receives T*H bf16 values)."""
    for name, t in (("x_host", x_host), ("idx_host", idx_host), ("w_host", w_host),
                    ("out_host", out_host)):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
    if x_host.dim() != 2 or x_host.dtype != torch.bfloat16:
        raise TypeError("x_host must be bf16 [T, H]")
    T, H = x_host.shape
    if idx_host.dim() != 2 or idx_host.shape[0] != T:
        raise ValueError("idx_host must be [T, k]")
    bits = {torch.int64: 64, torch.int32: 32}.get(idx_host.dtype)
    if bits is None:
        raise TypeError("idx_host must be int32 or int64")
    k = idx_host.shape[1]
    if w_host.dtype != torch.float32 or tuple(w_host.shape) != (T, k):
        raise TypeError("w_host must be float32 [T, k]")
    if out_host.dtype != torch.bfloat16 or tuple(out_host.shape) != (T, H):
        raise TypeError("out_host must be bf16 [T, H]")
    return T, H, k, bits


def roundtrip_host(x_host: torch.Tensor, idx_host: torch.Tensor, w_host: torch.Tensor,
                   E: int, R: int, dev_mem: torch.Tensor, out_host: torch.Tensor, stream=None,
                   dev_err=None):
    """ep_roundtrip_host: host buffers in, host buffer out (asynchronous).
    dev_err: optional ctypes.c_int32 that receives the layout's device error
    word once the stream has synchronised."""
    T, H, k, bits = _host_roundtrip_args(x_host, idx_host, w_host, out_host)
    if not dev_mem.is_cuda:
        raise ValueError("dev_mem must be a CUDA tensor")
    _check(lib().ep_roundtrip_host(x_host.data_ptr(), idx_host.data_ptr(), w_host.data_ptr(),
                                   T, H, k, E, R, bits, dev_mem.data_ptr(),
                                   dev_mem.numel() * dev_mem.element_size(),
                                   out_host.data_ptr(),
                                   None if dev_err is None else ctypes.byref(dev_err),
                                   _stream(stream)), "ep_roundtrip_host")
    return out_host


def roundtrip_host_noalloc(x_host: torch.Tensor, idx_host: torch.Tensor, w_host: torch.Tensor,
                           E: int, R: int, out_host: torch.Tensor, stream=None, dev_err=None):
    """ep_roundtrip_host_noalloc: like roundtrip_host, for callers that cannot
    allocate device memory -- the device scratch is the library's fixed
    NOALLOC_SCRATCH_BYTES array (asynchronous; calls that overlap on the GPU
    race on that array)."""
    T, H, k, bits = _host_roundtrip_args(x_host, idx_host, w_host, out_host)
    _check(lib().ep_roundtrip_host_noalloc(x_host.data_ptr(), idx_host.data_ptr(),
                                           w_host.data_ptr(), T, H, k, E, R, bits,
                                           out_host.data_ptr(),
                                           None if dev_err is None else ctypes.byref(dev_err),
                                           _stream(stream)),
           "ep_roundtrip_host_noalloc")
    return out_host


def debug_dispatch_first_wait_limit(limit: int) -> None:
    """ep_debug_dispatch_first_wait_limit (test setting; negative = normal)."""
    lib().ep_debug_dispatch_first_wait_limit(int(limit))
