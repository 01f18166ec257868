"""Host-only checks of the C ABI: the library loads without a GPU, exports
every function include/epx.h declares, and validates arguments on the host
(no compute call is made here)."""
import ctypes
import os
import re

import pytest

from combine_ep_layout_07_b200 import build as epx_build
from combine_ep_layout_07_b200 import epx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "epx.h")


@pytest.fixture(scope="module")
def lib():
    epx_build.build()
    return epx.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(ep_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_path():
    names = declared_functions()
    for must in ("ep_layout", "ep_dispatch_expand", "ep_combine_reduce", "ep_layout_init",
                 "ep_layout_bytes", "ep_layout_read_totals", "ep_standin_expert",
                 "ep_status_str", "ep_roundtrip_host"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.ep_abi_version() == 3


def test_status_strings(lib):
    for code in range(7):
        s = lib.ep_status_str(code).decode()
        assert s.startswith("EP_")
    assert lib.ep_status_str(99).decode() == "EP_ERR_UNKNOWN"


def test_layout_bytes_and_init_validate_on_host(lib):
    assert lib.ep_layout_bytes(128, 8, 256, 16) > 0
    assert lib.ep_layout_bytes(128, 8, 250, 16) == 0      # E % R != 0
    assert lib.ep_layout_bytes(128, 33, 256, 16) == 0     # k > 32
    assert lib.ep_layout_bytes(128, 8, 256, 128) == 0     # R > 64
    assert lib.ep_layout_bytes(128, 8, 8192, 16) == 0     # E > 4096
    assert lib.ep_layout_bytes(-1, 8, 256, 16) == 0
    c = epx._LayoutC()
    fake = 0x10000  # never dereferenced: init only carves pointers
    n = lib.ep_layout_bytes(128, 8, 256, 16)
    assert lib.ep_layout_init(ctypes.byref(c), 128, 8, 256, 16, 64, fake, n) == 0
    assert c.T == 128 and c.k == 8 and c.E == 256 and c.R == 16 and c.idx_bits == 64
    ptrs = [c.cnt_e, c.off_e, c.cnt_r, c.off_r, c.pos, c.recv_pos, c.totals]
    assert all(p % 16 == 0 for p in ptrs)
    assert ptrs == sorted(ptrs) and ptrs[-1] + 16 <= fake + n
    assert c.pos - c.off_r >= 4 * 17 and c.recv_pos - c.pos >= 4 * 128 * 8
    assert lib.ep_layout_init(ctypes.byref(c), 128, 8, 256, 16, 64, fake, n - 1) == 1
    assert lib.ep_layout_init(ctypes.byref(c), 128, 8, 256, 16, 16, fake, n) == 1
    assert lib.ep_layout_init(ctypes.byref(c), 128, 8, 250, 16, 64, fake, n) == 1
    assert lib.ep_layout_init(ctypes.byref(c), 128, 40, 256, 16, 64, fake, 1 << 30) == 6
    assert lib.ep_layout_init(ctypes.byref(c), 128, 8, 256, 16, 64, fake + 4, n) == 2
    assert lib.ep_layout_init(None, 128, 8, 256, 16, 64, fake, n) == 1


def test_calls_reject_bad_arguments_before_launching(lib):
    # a NULL layout or an invalid one returns before any CUDA call
    assert lib.ep_layout(None, None, None) == 1
    bad = epx._LayoutC()
    assert lib.ep_layout(None, ctypes.byref(bad), None) == 1
    assert lib.ep_dispatch_expand(None, 64, ctypes.byref(bad), None, 0, None, 0, None) == 1
    assert lib.ep_combine_reduce(None, None, 64, ctypes.byref(bad), None, 0, None) == 1
    c = epx._LayoutC()
    fake = 0x10000
    n = lib.ep_layout_bytes(4, 2, 4, 2)
    assert lib.ep_layout_init(ctypes.byref(c), 4, 2, 4, 2, 64, fake, n) == 0
    # H % 8 != 0, negative capacity, unknown variant
    assert lib.ep_dispatch_expand(fake, 12, ctypes.byref(c), fake, 8, fake, 8, None) == 1
    assert lib.ep_dispatch_expand(fake, 16, ctypes.byref(c), fake, -1, fake, 8, None) == 1
    assert lib.ep_dispatch_expand_variant(fake, 16, ctypes.byref(c), fake, 8, fake, 8, 7,
                                          None) == 1
    # 16-byte alignment of row buffers
    assert lib.ep_dispatch_expand(fake + 2, 16, ctypes.byref(c), fake, 8, fake, 8, None) == 2
    assert lib.ep_combine_reduce(fake + 8, fake, 16, ctypes.byref(c), fake, 8, None) == 2
    assert lib.ep_combine_reduce(fake, fake + 2, 16, ctypes.byref(c), fake, 8, None) == 2
    assert lib.ep_standin_expert(fake, 16, ctypes.byref(c), fake + 4, 8, None) == 2
    # misaligned 64-bit indices
    assert lib.ep_layout(fake + 4, ctypes.byref(c), None) == 2
    # unknown layout schedule or combine schedule
    assert lib.ep_layout_variant(fake, ctypes.byref(c), 4, None) == 1
    assert lib.ep_layout_variant(fake, ctypes.byref(c), -1, None) == 1
    assert lib.ep_layout_variant(fake + 4, ctypes.byref(c), 1, None) == 2
    assert lib.ep_combine_reduce_variant(fake, fake, 16, ctypes.byref(c), fake, 8, 3, None) == 1


def test_roundtrip_sizes(lib):
    n = lib.ep_roundtrip_device_bytes(128, 7168, 8, 256, 16, 64)
    row = 7168 * 2
    assert n >= 128 * row * (1 + 8 + 8 + 1) + 128 * 8 * row
    assert lib.ep_roundtrip_device_bytes(128, 7167, 8, 256, 16, 64) == 0
    assert lib.ep_roundtrip_host(None, None, None, 128, 7168, 8, 256, 16, 64, None, 0, None,
                                 None, None) == 1


def test_host_roundtrip_binding_checks_buffers():
    """The binding rejects host buffers of the wrong dtype or shape before
    calling the library (which trusts them: it copies T*H values back)."""
    import torch
    T, H, k = 4, 16, 2
    x = torch.zeros((T, H), dtype=torch.bfloat16)
    i = torch.zeros((T, k), dtype=torch.int64)
    w = torch.zeros((T, k), dtype=torch.float32)
    out = torch.zeros((T, H), dtype=torch.bfloat16)
    bad = [
        (x.float(), i, w, out),                      # x not bf16
        (x, i.float(), w, out),                      # indices not integer
        (x, i, w.double(), out),                     # weights not fp32
        (x, i, w[:, :1].contiguous(), out),          # weights not [T, k]
        (x, i, w, out[:2].contiguous()),             # out too small
        (x, i, w, out.float()),                      # out not bf16
        (x, i[:3].contiguous(), w, out),             # indices not [T, k]
    ]
    for args in bad:
        with pytest.raises((TypeError, ValueError)):
            epx._host_roundtrip_args(*args)
    assert epx._host_roundtrip_args(x, i, w, out) == (T, H, k, 64)


def test_binding_constants_mirror_the_header():
    src = open(HEADER).read()
    val = lambda name: int(re.search(r"#define %s \(?(\d+)" % name, src).group(1))  # noqa: E731
    assert epx.MAX_TOPK == val("EPX_MAX_TOPK")
    assert epx.MAX_RANKS == val("EPX_MAX_RANKS")
    assert epx.MAX_EXPERTS == val("EPX_MAX_EXPERTS")
    assert epx.FUSED_MAX_ROUTES == val("EPX_FUSED_MAX_ROUTES")
    assert epx.FUSED_AUTO_MIN_ROUTES == val("EPX_FUSED_AUTO_MIN_ROUTES")
    assert epx.FUSED_AUTO_MAX_ROUTES == val("EPX_FUSED_AUTO_MAX_ROUTES")
    assert epx.NOALLOC_SCRATCH_BYTES == val("EPX_NOALLOC_SCRATCH_BYTES") << 20


def test_one_launch_call_validates_on_host(lib):
    c = epx._LayoutC()
    fake = 0x10000
    n = lib.ep_layout_bytes(4, 2, 4, 2)
    assert lib.ep_layout_init(ctypes.byref(c), 4, 2, 4, 2, 64, fake, n) == 0
    f = lib.ep_layout_dispatch_expand_variant
    assert f(fake, ctypes.byref(c), fake, 16, fake, 8, fake, 8, 3, None) == 1    # variant
    assert f(fake, ctypes.byref(c), fake, 12, fake, 8, fake, 8, 0, None) == 1    # H % 8
    assert f(fake, ctypes.byref(c), fake + 2, 16, fake, 8, fake, 8, 0, None) == 2
    assert f(fake + 4, ctypes.byref(c), fake, 16, fake, 8, fake, 8, 0, None) == 2
    assert f(None, ctypes.byref(c), fake, 16, fake, 8, fake, 8, 0, None) == 1
    assert f(fake, None, fake, 16, fake, 8, fake, 8, 0, None) == 1
    assert lib.ep_latency_floor(None, 0, 3, None) == 1
    assert lib.ep_latency_floor(fake, 64, 3, None) == 1                            # too small
    assert lib.ep_latency_floor(fake + 4, 64 * 8, 3, None) == 2


def test_peer_memory_calls_validate_on_host(lib):
    """ep_dispatch_p2p / ep_combine_local_reduce_p2p / ep_ipc_* reject bad
    arguments before touching the GPU."""
    c = epx._LayoutC()
    fake = 0x10000
    n = lib.ep_layout_bytes(4, 2, 4, 2)
    assert lib.ep_layout_init(ctypes.byref(c), 4, 2, 4, 2, 64, fake, n) == 0
    peers = (epx._PeerRowsC * 2)()
    for r in range(2):
        peers[r].rows, peers[r].cap = fake, 8
    d = lib.ep_dispatch_p2p
    assert d(fake, 16, ctypes.byref(c), fake, fake, None, None) == 1          # no peers
    assert d(fake, 12, ctypes.byref(c), fake, fake, peers, None) == 1         # H % 8
    assert d(fake + 2, 16, ctypes.byref(c), fake, fake, peers, None) == 2     # x alignment
    assert d(fake, 16, ctypes.byref(c), fake + 4, fake, peers, None) == 2     # idx alignment
    peers[1].cap = -1
    assert d(fake, 16, ctypes.byref(c), fake, fake, peers, None) == 1         # bad entry
    peers[1].cap, peers[1].rows = 8, fake + 8
    assert d(fake, 16, ctypes.byref(c), fake, fake, peers, None) == 1         # rows alignment
    peers[1].rows = None
    assert d(fake, 16, ctypes.byref(c), fake, fake, peers, None) == 1         # rows missing
    peers[1].rows = fake
    cl = lib.ep_combine_local_reduce_p2p
    assert cl(fake, fake, 16, ctypes.byref(c), 8, 16, peers, None) == 1       # partial bits
    assert cl(fake, fake, 16, ctypes.byref(c), 32, 16, None, None) == 1       # no peers
    assert cl(fake + 2, fake, 16, ctypes.byref(c), 32, 16, peers, None) == 2
    ptr = ctypes.c_void_p()
    h = ctypes.create_string_buffer(epx.IPC_HANDLE_BYTES)
    assert lib.ep_ipc_malloc(0, ctypes.byref(ptr), h) == 1
    assert lib.ep_ipc_malloc(16, None, h) == 1
    assert lib.ep_ipc_free(None) == 1
    assert lib.ep_ipc_open(None, ctypes.byref(ptr)) == 1
    assert lib.ep_ipc_close(None) == 1
    src = open(HEADER).read()
    assert int(re.search(r"#define EPX_IPC_HANDLE_BYTES (\d+)", src).group(1)) == \
        epx.IPC_HANDLE_BYTES
    assert ctypes.sizeof(epx._PeerRowsC) == 56


def test_layout_block_holds_the_grid_workspace(lib):
    """ep_layout_bytes covers the grid schedule's workspace after the
    totals: a 16-word header, one row of packed counts and one row of
    32-bit prefixes per CTA (one CTA per 256 routes, at most 256 CTAs), and
    the totals row."""
    c = epx._LayoutC()
    fake = 0x100000
    for (T, k, E, R) in [(4096, 8, 256, 16), (1, 1, 1, 1), (128, 32, 4096, 64), (70000, 8, 256, 16)]:
        n = lib.ep_layout_bytes(T, k, E, R)
        assert lib.ep_layout_init(ctypes.byref(c), T, k, E, R, 64, fake, n) == 0
        assert c.work > c.totals and c.work % 16 == 0
        nb = min(-(-(T * k) // 256), 256)
        rows = ((E + R + 1) // 2 + 3) // 4 * 4
        pref = (E + R + 3) // 4 * 4
        need = 4 * (16 + nb * rows + (nb + 1) * pref)
        assert c.work + need <= fake + n