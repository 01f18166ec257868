"""CPU oracle for MoE token dispatch and combine -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it; the arithmetic lives in ``epx_oracle.c`` (plain C,
built by the host compiler) and is documented there with the passages of the
pages it follows.

Python here only builds the C file and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "epx_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libepx_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no nvcc, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.orc_layout.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, P]
    lib.orc_layout.restype = I
    lib.orc_dispatch_expand.argtypes = [P, I, I, I, I, I, P, I, P, P, P, P]
    lib.orc_dispatch_expand.restype = None
    lib.orc_standin.argtypes = [P, I, I, P, P]
    lib.orc_standin.restype = None
    lib.orc_combine.argtypes = [P, P, P, I, I, I, P, P]
    lib.orc_combine.restype = None
    lib.orc_combine_local.argtypes = [P, P, P, I, P, P, I, I, I, I, I, I, P]
    lib.orc_combine_local.restype = None
    lib.orc_combine_epilogue.argtypes = [P, I, P, P, I, I, I, P]
    lib.orc_combine_epilogue.restype = None
    lib.orc_expand_index.argtypes = [P, I, P, P, I, I, I, I, P]
    lib.orc_expand_index.restype = None
    lib.orc_bf16_from_double.argtypes = [ctypes.c_double]
    lib.orc_bf16_from_double.restype = ctypes.c_uint16
    lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_double.restype = ctypes.c_double
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def bf16_from_double(v: float) -> int:
    return int(_load().orc_bf16_from_double(float(v)))


def bf16_to_double(b: int) -> float:
    return float(_load().orc_bf16_to_double(int(b) & 0xFFFF))


def layout(topk_idx: np.ndarray, E: int, R: int) -> dict:
    """Routing layout; ``topk_idx`` is int32 or int64 ``[T, k]``."""
    idx = np.ascontiguousarray(topk_idx)
    if idx.dtype == np.int64:
        bits = 64
    elif idx.dtype == np.int32:
        bits = 32
    else:
        raise TypeError(idx.dtype)
    T, k = idx.shape
    out = dict(
        cnt_e=np.zeros(E, np.int32), off_e=np.zeros(E + 1, np.int32),
        cnt_r=np.zeros(R, np.int32), off_r=np.zeros(R + 1, np.int32),
        pos=np.zeros(T * k, np.int32), recv_pos=np.zeros(T * R, np.int32),
        totals=np.zeros(4, np.int64))
    rc = _load().orc_layout(_p(idx), bits, T, k, E, R, _p(out["cnt_e"]),
                            _p(out["off_e"]), _p(out["cnt_r"]), _p(out["off_r"]),
                            _p(out["pos"]), _p(out["recv_pos"]), _p(out["totals"]))
    if rc != 0:
        raise ValueError(f"orc_layout rejected the arguments (rc={rc})")
    out["pos"] = out["pos"].reshape(T, k)
    out["recv_pos"] = out["recv_pos"].reshape(T, R)
    out["N_route"], out["N_recv"], out["T_real"], out["n_bad"] = (
        int(v) for v in out["totals"])
    out.update(T=T, k=k, E=E, R=R, idx=idx)
    return out


def dispatch_expand(x: np.ndarray, lay: dict):
    """Returns (recv [N_recv, H], expanded [N_route, H]) as uint16 bf16 bits."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T, H = x.shape
    assert T == lay["T"]
    idx = lay["idx"]
    recv = np.zeros((max(lay["N_recv"], 1), H), np.uint16)
    expanded = np.zeros((max(lay["N_route"], 1), H), np.uint16)
    _load().orc_dispatch_expand(_p(x), T, H, lay["k"], lay["E"], lay["R"], _p(idx),
                                64 if idx.dtype == np.int64 else 32,
                                _p(lay["pos"]), _p(lay["recv_pos"]), _p(recv),
                                _p(expanded))
    return recv[:lay["N_recv"]], expanded[:lay["N_route"]]


def standin(expanded: np.ndarray, lay: dict) -> np.ndarray:
    """Stand-in expert output for the expert-contiguous rows."""
    ex = np.ascontiguousarray(expanded, dtype=np.uint16)
    n, H = ex.shape
    assert n == lay["N_route"]
    y = np.zeros((max(n, 1), H), np.uint16)
    _load().orc_standin(_p(ex if n else np.zeros((1, H), np.uint16)), H, lay["E"],
                        _p(lay["off_e"]), _p(y))
    return y[:n]


def combine(y: np.ndarray, topk_weights: np.ndarray, lay: dict, exact: bool = False):
    """Weighted combine; returns out [T, H] bf16 bits (and the double sums)."""
    T, k = lay["T"], lay["k"]
    y = np.ascontiguousarray(y, dtype=np.uint16)
    H = y.shape[1]
    if y.shape[0] == 0:
        y = np.zeros((1, H), np.uint16)
    w = np.ascontiguousarray(topk_weights, dtype=np.float32)
    assert w.shape == (T, k)
    out = np.zeros((T, H), np.uint16)
    ex = np.zeros((T, H), np.float64) if exact else None
    _load().orc_combine(_p(y), _p(w), _p(lay["pos"]), T, k, H, _p(out),
                        _p(ex) if exact else None)
    return (out, ex) if exact else out


def run_all(wl: dict, idx_dtype=np.int64) -> dict:
    """Whole path on one workload: layout, dispatch/expand, stand-in, combine."""
    lay = layout(wl["topk_idx"].astype(idx_dtype), wl["E"], wl["R"])
    recv, expanded = dispatch_expand(wl["x"], lay)
    y = standin(expanded, lay)
    out = combine(y, wl["topk_weights"], lay)
    return dict(layout=lay, recv=recv, expanded=expanded, y=y, out=out)


def combine_local(y: np.ndarray, topk_weights: np.ndarray, lay: dict, part_bits: int = 32):
    """Per-(token, rank) partial rows in the receive layout: float32 or bf16
    bits (uint16), shape [N_recv, H]."""
    T, k = lay["T"], lay["k"]
    y = np.ascontiguousarray(y, dtype=np.uint16)
    H = y.shape[1]
    if y.shape[0] == 0:
        y = np.zeros((1, H), np.uint16)
    w = np.ascontiguousarray(topk_weights, dtype=np.float32)
    idx = lay["idx"]
    n = max(lay["N_recv"], 1)
    part = np.zeros((n, H), np.float32 if part_bits == 32 else np.uint16)
    _load().orc_combine_local(_p(y), _p(w), _p(idx), 64 if idx.dtype == np.int64 else 32,
                              _p(lay["pos"]), _p(lay["recv_pos"]), T, k, lay["E"], lay["R"], H,
                              part_bits, _p(part))
    return part[:lay["N_recv"]]


def combine_epilogue(partial: np.ndarray, lay: dict, residual: np.ndarray = None):
    """Sum of each token's partial rows (rank order) plus an optional bf16
    residual row, rounded to bf16 bits [T, H]."""
    T, R = lay["T"], lay["R"]
    part_bits = 32 if partial.dtype == np.float32 else 16
    H = partial.shape[1]
    part = np.ascontiguousarray(partial)
    if part.shape[0] == 0:
        part = np.zeros((1, H), part.dtype)
    res = None if residual is None else np.ascontiguousarray(residual, dtype=np.uint16)
    out = np.zeros((T, H), np.uint16)
    _load().orc_combine_epilogue(_p(part), part_bits, _p(lay["recv_pos"]),
                                 _p(res) if res is not None else None, T, R, H, _p(out))
    return out


def expand_index(lay: dict) -> np.ndarray:
    """Row of `recv` that serves each expert-contiguous row, int32 [N_route]."""
    idx = lay["idx"]
    src = np.full(max(lay["N_route"], 1), -1, np.int32)
    _load().orc_expand_index(_p(idx), 64 if idx.dtype == np.int64 else 32, _p(lay["pos"]),
                             _p(lay["recv_pos"]), lay["T"], lay["k"], lay["E"], lay["R"],
                             _p(src))
    return src[:lay["N_route"]]
