"""The oracle: a plain single-threaded CPU statement of the MoE route -> layout
-> dispatch -> combine path, written in C (``moe_oracle.c``) and called here
through ctypes on numpy arrays.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the ``smoke()`` check
of ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
It shares no code with the CUDA package ``combine_moe_route_08_b200``.

What each function follows is stated in ``moe_oracle.c`` (page title and
section of the two Perplexity posts, the DeepSeek-V3 fragments quoted on the
other pages, and the OCP OFP8 specification for E4M3).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

OK = 0
ERR_INVALID = 1
ERR_CAPACITY = 3

GCC_FLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, u32 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint32
        lib.oracle_route.argtypes = [P, i32, i32, i32, i32, P, P]
        lib.oracle_route.restype = i32
        lib.oracle_route_ex.argtypes = [P, i32, i32, i32, i32, i32, ctypes.c_float, P, P, i32, i32, P, P]
        lib.oracle_route_ex.restype = i32
        lib.oracle_layout.argtypes = [P, i32, i32, i32, i32, i32, i64, P, P, P, P, P, P]
        lib.oracle_layout.restype = i32
        lib.oracle_private_layout.argtypes = [P, i32, i32, i32, i32, i32, P, P, P]
        lib.oracle_private_layout.restype = i32
        lib.oracle_dispatch_bf16.argtypes = [P, i32, i32, i32, P, P, i64]
        lib.oracle_dispatch_bf16.restype = i32
        lib.oracle_dispatch_fp8.argtypes = [P, i32, i32, i32, P, P, P, i64]
        lib.oracle_dispatch_fp8.restype = i32
        lib.oracle_quantize_tokens.argtypes = [P, i32, i32, P, i32, P, P]
        lib.oracle_quantize_tokens.restype = i32
        lib.oracle_combine.argtypes = [P, P, P, i32, i32, i32, i64, P, i32, P, P]
        lib.oracle_combine.restype = i32
        lib.oracle_combine_fp8.argtypes = [P, P, P, P, i32, i32, i32, i64, P, i32, P, P]
        lib.oracle_combine_fp8.restype = i32
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_float
        lib.oracle_e4m3_encode_array.argtypes = [P, i64, P]
        lib.oracle_e4m3_encode_array.restype = None
        lib.oracle_e4m3_count_mismatch.argtypes = [u32, i64, P, ctypes.POINTER(ctypes.c_int64)]
        lib.oracle_e4m3_count_mismatch.restype = i64
        lib.oracle_float_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_float_to_bf16.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# route
# --------------------------------------------------------------------------

def route(logits: np.ndarray, k: int, renormalize: bool = False):
    """Top-k experts by (logit desc, index asc) and their softmax weights.

    Returns (topk_idx int32 [T][k], topk_w float32 [T][k])."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    st = _load().oracle_route(_ptr(logits), T, E, k, int(renormalize), _ptr(idx), _ptr(w))
    if st != OK:
        raise ValueError(f"oracle_route status {st}")
    return idx, w


def route_ex(logits: np.ndarray, k: int, n_shared: int = 0, shared_weight: float = 1.0,
             replica_offsets=None, replica_ids=None, E_phys: int | None = None,
             T_r: int = 1, renormalize: bool = False):
    """Top-k over the routed logits, then n_shared always-selected shared
    experts, every logical expert mapped to a physical replica chosen by the
    token's source rank.  Returns (topk_idx [T][k+n_shared] physical ids,
    topk_w [T][k+n_shared], status)."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    kk = k + n_shared
    if E_phys is None:
        E_phys = E + n_shared
    ro = None if replica_offsets is None else _c(replica_offsets, np.int32)
    ri = None if replica_ids is None else _c(replica_ids, np.int32)
    idx = np.empty((T, kk), np.int32)
    w = np.empty((T, kk), np.float32)
    st = _load().oracle_route_ex(_ptr(logits), T, E, k, int(renormalize), n_shared,
                                 float(shared_weight), _ptr(ro), _ptr(ri), E_phys, T_r,
                                 _ptr(idx), _ptr(w))
    return idx, w, st


# --------------------------------------------------------------------------
# layout
# --------------------------------------------------------------------------

def packed_rows(T: int, k: int) -> int:
    return T * k


def layout(topk_idx: np.ndarray, E: int, R: int, capacity: int = 0, rows: int | None = None):
    """Counts, offsets and index maps; see ``oracle_layout`` in moe_oracle.c.

    Returns a dict of numpy arrays plus the integer ``status``."""
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    if rows is None:
        rows = T * k if capacity == 0 else E * capacity
    out = dict(
        expert_counts=np.empty(E, np.int32),
        expert_src_counts=np.empty((E, R), np.int32),
        rank_counts=np.empty(R, np.int32),
        expert_offsets=np.empty(E + 1, np.int32),
        dispatch_pos=np.empty((T, k), np.int32),
        recv_src=np.empty(rows, np.int32),
    )
    st = _load().oracle_layout(
        _ptr(topk_idx), T, k, E, R, capacity, rows,
        _ptr(out["expert_counts"]), _ptr(out["expert_src_counts"]), _ptr(out["rank_counts"]),
        _ptr(out["expert_offsets"]), _ptr(out["dispatch_pos"]), _ptr(out["recv_src"]))
    if st == ERR_INVALID and rows < 0:
        raise ValueError("bad rows")
    out["status"] = st
    return out


def private_layout(topk_idx: np.ndarray, E: int, R: int, max_m: int):
    """Two-phase layout: private row of each slot in the (expert, source rank)
    regions of max_m rows, the packed row base of each region, and the slot
    held by each private row.  Returns (private_pos [T][k], region_base
    [E][R], recv_src_private [E*R*max_m], status)."""
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    pos = np.empty((T, k), np.int32)
    base = np.empty((E, R), np.int32)
    src = np.empty(E * R * max_m, np.int32)
    st = _load().oracle_private_layout(_ptr(topk_idx), T, k, E, R, max_m, _ptr(pos), _ptr(base),
                                       _ptr(src))
    return pos, base, src, st


# --------------------------------------------------------------------------
# dispatch
# --------------------------------------------------------------------------

def dispatch_bf16(x_bits: np.ndarray, dispatch_pos: np.ndarray, rows: int,
                  recv_x: np.ndarray | None = None):
    """recv_x[dispatch_pos[g, j]] = x[g].  ``x_bits`` is the bf16 bit pattern
    (uint16 [T][H]).  Rows no slot fills keep the contents of ``recv_x``
    (zeros when it is not given)."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    pos = _c(dispatch_pos, np.int32)
    k = pos.shape[1]
    if recv_x is None:
        recv_x = np.zeros((rows, H), np.uint16)
    st = _load().oracle_dispatch_bf16(_ptr(x_bits), T, H, k, _ptr(pos), _ptr(recv_x), rows)
    if st != OK:
        raise ValueError(f"oracle_dispatch_bf16 status {st}")
    return recv_x


def dispatch_fp8(x_bits: np.ndarray, dispatch_pos: np.ndarray, rows: int):
    """FP8 e4m3 dispatch with 1x128 binary32 block scales.

    Returns (recv_q uint8 [rows][H], recv_scale float32 [rows][H/128]); rows no
    slot fills are zero."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    pos = _c(dispatch_pos, np.int32)
    k = pos.shape[1]
    q = np.zeros((rows, H), np.uint8)
    s = np.zeros((rows, H // 128), np.float32)
    st = _load().oracle_dispatch_fp8(_ptr(x_bits), T, H, k, _ptr(pos), _ptr(q), _ptr(s), rows)
    if st != OK:
        raise ValueError(f"oracle_dispatch_fp8 status {st}")
    return q, s


def quantize_tokens(x_bits: np.ndarray, tokens):
    """Codes and scales of the listed tokens: (q [n][H], s [n][H/128])."""
    x_bits = _c(x_bits, np.uint16)
    T, H = x_bits.shape
    tok = _c(tokens, np.int32)
    n = tok.shape[0]
    q = np.empty((n, H), np.uint8)
    s = np.empty((n, H // 128), np.float32)
    st = _load().oracle_quantize_tokens(_ptr(x_bits), T, H, _ptr(tok), n, _ptr(q), _ptr(s))
    if st != OK:
        raise ValueError(f"oracle_quantize_tokens status {st}")
    return q, s


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------

def combine(y_bits: np.ndarray, dispatch_pos: np.ndarray, topk_w: np.ndarray,
            tokens=None):
    """Router-weighted sum of the k expert rows of each token, accumulated in
    binary32 in ascending j.  Returns (acc float32 [n][H], out_bits uint16
    [n][H]) for the listed tokens (all tokens when ``tokens`` is None)."""
    y_bits = _c(y_bits, np.uint16)
    rows, H = y_bits.shape
    pos = _c(dispatch_pos, np.int32)
    T, k = pos.shape
    w = _c(topk_w, np.float32)
    assert w.shape == (T, k)
    if tokens is None:
        tok, n = None, T
    else:
        tok = _c(tokens, np.int32)
        n = tok.shape[0]
    acc = np.empty((n, H), np.float32)
    out = np.empty((n, H), np.uint16)
    st = _load().oracle_combine(_ptr(y_bits), _ptr(pos), _ptr(w), T, H, k, rows,
                                _ptr(tok), n, _ptr(acc), _ptr(out))
    if st != OK:
        raise ValueError(f"oracle_combine status {st}")
    return acc, out


def combine_fp8(yq: np.ndarray, ys: np.ndarray, dispatch_pos: np.ndarray, topk_w: np.ndarray,
                tokens=None):
    """Combine with E4M3 expert rows: each element restored as decode(q) * s
    (one binary32 product), then the router-weighted binary32 sum over j
    ascending.  yq uint8 [rows][H], ys float32 [rows][H/128].  Returns (acc
    float32 [n][H], out_bits uint16 [n][H])."""
    yq = _c(yq, np.uint8)
    rows, H = yq.shape
    ys = _c(ys, np.float32)
    assert ys.shape == (rows, H // 128)
    pos = _c(dispatch_pos, np.int32)
    T, k = pos.shape
    w = _c(topk_w, np.float32)
    assert w.shape == (T, k)
    if tokens is None:
        tok, n = None, T
    else:
        tok = _c(tokens, np.int32)
        n = tok.shape[0]
    acc = np.empty((n, H), np.float32)
    out = np.empty((n, H), np.uint16)
    st = _load().oracle_combine_fp8(_ptr(yq), _ptr(ys), _ptr(pos), _ptr(w), T, H, k, rows,
                                    _ptr(tok), n, _ptr(acc), _ptr(out))
    if st != OK:
        raise ValueError(f"oracle_combine_fp8 status {st}")
    return acc, out


# --------------------------------------------------------------------------
# scalar formats
# --------------------------------------------------------------------------

def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    q = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(q))
    return q


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(codes, np.uint8).ravel()
    table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], np.float32)
    return table[flat].reshape(np.shape(codes))


def e4m3_count_mismatch(first_bits: int, codes: np.ndarray):
    """Encode the binary32 bit patterns first_bits .. first_bits+n-1 and count
    the codes that differ from ``codes``; returns (count, first bad index)."""
    codes = _c(codes, np.uint8)
    first_bad = ctypes.c_int64(-1)
    n = _load().oracle_e4m3_count_mismatch(first_bits, codes.size, _ptr(codes),
                                           ctypes.byref(first_bad))
    return int(n), int(first_bad.value)


def float_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(v, np.float32).ravel()
    return np.array([lib.oracle_float_to_bf16(float(x)) for x in flat],
                    np.uint16).reshape(np.shape(v))
