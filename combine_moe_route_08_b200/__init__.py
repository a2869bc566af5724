"""combine_moe_route_08_b200 -- Mixture-of-Experts route, dispatch and combine
on one B200 (sm_100a).

A thin ctypes binding over ``libmoe_route.so`` (C ABI in
``include/moe_route.h``): the functions here carry the C names, marshal
torch CUDA tensors to device pointers and the current stream, allocate the
outputs the caller did not pass (torch is used for device memory and
streams only), and raise :class:`MoeError` on a non-OK status.  Every step of
the path runs in the library's CUDA kernels; there is no CPU or torch
fallback: importing this package fails if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MoeError", "lib", "moe_status_string", "moe_route_topk", "moe_route_topk_ex",
    "moe_layout_workspace_bytes", "moe_dispatch_layout_launches", "kernels_per_step",
    "moe_combine_bf16_long_form",
    "moe_dispatch_layout", "moe_dispatch_bf16", "moe_dispatch_fp8", "moe_combine_bf16",
    "moe_quantize_e4m3", "moe_dispatch_layout_noalloc", "moe_dispatch_fp8_ex", "Workspace",
    "LIB_PATH", "MOE_SCALE_ROW_MAJOR", "MOE_SCALE_COL_MAJOR", "moe_dispatch_layout_private",
    "moe_compact_fp8", "moe_compact_bf16", "moe_route_dispatch_workspace_bytes",
    "moe_route_dispatch_fp8", "moe_route_dispatch_bf16", "moe_route_dispatch_ex_fp8",
    "moe_route_dispatch_ex_bf16", "moe_combine_fp8", "MOE_HOST_FUSED",
    "moe_route_dispatch_fp8_host", "moe_route_dispatch_bf16_host", "moe_combine_bf16_host",
    "moe_combine_fp8_host",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_route.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python combine_moe_route_08_b200/build.py` "
        "(nvcc, sm_100a). This package has no fallback path.")

lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_i32, _i64, _sz = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t

lib.moe_status_string.argtypes = [_i32]
lib.moe_status_string.restype = ctypes.c_char_p
lib.moe_route_topk.argtypes = [_P, _i32, _i32, _i32, _i32, _P, _P, _P]
lib.moe_route_topk.restype = _i32
lib.moe_route_topk_ex.argtypes = [_P, _i32, _i32, _i32, _i32, _i32, ctypes.c_float, _P, _P, _i32,
                                  _i32, _i32, _P, _P, _P, _P]
lib.moe_route_topk_ex.restype = _i32
lib.moe_layout_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32]
lib.moe_layout_workspace_bytes.restype = _sz
lib.moe_dispatch_layout_launches.argtypes = [_i32, _i32, _i32, _i32]
lib.moe_dispatch_layout_launches.restype = _i32
lib.moe_combine_bf16_long_form.argtypes = [_i32, _i32, _i32]
lib.moe_combine_bf16_long_form.restype = _i32
lib.moe_dispatch_layout.argtypes = [_P, _i32, _i32, _i32, _i32, _i32, _i64, _P, _P, _P, _P, _P, _P,
                                    _P, _sz, _P, _P]
lib.moe_dispatch_layout.restype = _i32
lib.moe_dispatch_layout_noalloc.argtypes = [_P, _i32, _i32, _i32, _i32, _i32, _i64, _P, _P, _P,
                                            _P, _P, _P, _P, _P]
lib.moe_dispatch_layout_noalloc.restype = _i32
lib.moe_dispatch_layout_private.argtypes = [_P, _i32, _i32, _i32, _i32, _i32, _i64, _P, _P, _P, _P,
                                            _P, _P, _P, _P, _sz, _P, _P]
lib.moe_dispatch_layout_private.restype = _i32
lib.moe_compact_fp8.argtypes = [_P, _P, _i64, _P, _P, _i32, _i32, _i32, _P, _P, _i64, _P, _P]
lib.moe_compact_fp8.restype = _i32
lib.moe_compact_bf16.argtypes = [_P, _i64, _P, _P, _i32, _i32, _i32, _P, _i64, _P, _P]
lib.moe_compact_bf16.restype = _i32
lib.moe_dispatch_bf16.argtypes = [_P, _i32, _i32, _i32, _P, _P, _i64, _P, _P]
lib.moe_dispatch_bf16.restype = _i32
lib.moe_dispatch_fp8.argtypes = [_P, _i32, _i32, _i32, _P, _P, _P, _i64, _P, _P]
lib.moe_dispatch_fp8.restype = _i32
lib.moe_dispatch_fp8_ex.argtypes = [_P, _i32, _i32, _i32, _P, _P, _P, _i64, _i32, _i64, _P, _P]
lib.moe_dispatch_fp8_ex.restype = _i32
lib.moe_combine_bf16.argtypes = [_P, _P, _P, _i32, _i32, _i32, _i64, _P, _P, _P]
lib.moe_combine_bf16.restype = _i32
lib.moe_route_dispatch_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32]
lib.moe_route_dispatch_workspace_bytes.restype = _sz
lib.moe_route_dispatch_fp8.argtypes = [_P, _i32, _i32, _i32, _i32, _i32, _i32, _P, _i32, _P, _P,
                                       _P, _P, _P, _P, _P, _P, _P, _P, _i64, _P, _sz, _P, _P]
lib.moe_route_dispatch_fp8.restype = _i32
lib.moe_route_dispatch_bf16.argtypes = [_P, _i32, _i32, _i32, _i32, _i32, _i32, _P, _i32, _P, _P,
                                        _P, _P, _P, _P, _P, _P, _P, _i64, _P, _sz, _P, _P]
lib.moe_route_dispatch_bf16.restype = _i32
_EX = [_i32, ctypes.c_float, _P, _P, _i32, _i32]  # n_shared .. E_phys
lib.moe_route_dispatch_ex_fp8.argtypes = ([_P, _i32, _i32, _i32, _i32] + _EX +
                                          [_i32, _i32, _P, _i32] + [_P] * 10 +
                                          [_i64, _P, _sz, _P, _P])
lib.moe_route_dispatch_ex_fp8.restype = _i32
lib.moe_route_dispatch_ex_bf16.argtypes = ([_P, _i32, _i32, _i32, _i32] + _EX +
                                           [_i32, _i32, _P, _i32] + [_P] * 9 +
                                           [_i64, _P, _sz, _P, _P])
lib.moe_route_dispatch_ex_bf16.restype = _i32
lib.moe_combine_fp8.argtypes = [_P, _P, _P, _P, _i32, _i32, _i32, _i64, _P, _P, _P]
lib.moe_combine_fp8.restype = _i32
lib.moe_quantize_e4m3.argtypes = [_P, _i64, _P, _P]
lib.moe_quantize_e4m3.restype = _i32
_HOST_HEAD = [_P, _P] + [_i32] * 8 + [_P] * 10       # host inputs .. recv_src
lib.moe_route_dispatch_fp8_host.argtypes = _HOST_HEAD + [_P, _P, _i64, _P, _sz, _P, _P]
lib.moe_route_dispatch_fp8_host.restype = _i32
lib.moe_route_dispatch_bf16_host.argtypes = _HOST_HEAD + [_P, _i64, _P, _sz, _P, _P]
lib.moe_route_dispatch_bf16_host.restype = _i32
lib.moe_combine_bf16_host.argtypes = [_P, _P, _P, _i32, _i32, _i32, _i64, _P, _P, _P, _P]
lib.moe_combine_bf16_host.restype = _i32
lib.moe_combine_fp8_host.argtypes = [_P, _P, _P, _P, _i32, _i32, _i32, _i64, _P, _P, _P, _P]
lib.moe_combine_fp8_host.restype = _i32

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CAPACITY = 3
MOE_ERR_WORKSPACE = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_CUDA = 6
MOE_SCALE_ROW_MAJOR = 0
MOE_SCALE_COL_MAJOR = 1
MOE_LAYOUT_NOALLOC_SCRATCH_BYTES = 1 << 20   # the fixed scratch of moe_dispatch_layout_noalloc
MOE_HOST_FUSED = 1                           # host-buffer route+dispatch: the single launch


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)}")


def moe_status_string(status: int) -> str:
    return lib.moe_status_string(status).decode()


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr() or None


def _host_ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("expected a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr() or None


def _stream(stream) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _bits16(t: torch.Tensor) -> torch.Tensor:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise ValueError(f"expected bf16 data, got {t.dtype}")
    return t


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def moe_route_topk(logits: torch.Tensor, k: int, renormalize: bool = False,
                   topk_idx: torch.Tensor | None = None, topk_w: torch.Tensor | None = None,
                   stream=None):
    """Router softmax + top-k.  logits fp32 [T][E] -> (topk_idx int32 [T][k],
    topk_w fp32 [T][k])."""
    assert logits.dtype == torch.float32 and logits.dim() == 2
    T, E = logits.shape
    dev = logits.device
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
    _check(lib.moe_route_topk(_ptr(logits), T, E, k, int(renormalize), _ptr(topk_idx),
                              _ptr(topk_w), _stream(stream)), "moe_route_topk")
    return topk_idx, topk_w


def moe_route_topk_ex(logits: torch.Tensor, k: int, n_shared: int = 0, shared_weight: float = 1.0,
                      replica_offsets: torch.Tensor | None = None,
                      replica_ids: torch.Tensor | None = None, E_phys: int | None = None,
                      tokens_per_rank: int = 1, renormalize: bool = False,
                      topk_idx: torch.Tensor | None = None, topk_w: torch.Tensor | None = None,
                      dev_status: torch.Tensor | None = None, stream=None):
    """Top-k over the routed logits plus n_shared always-selected shared
    experts, each logical expert mapped to a physical replica by the token's
    source rank.  Returns (topk_idx int32 [T][k+n_shared] physical ids,
    topk_w fp32 [T][k+n_shared])."""
    assert logits.dtype == torch.float32 and logits.dim() == 2
    T, E = logits.shape
    kk = k + n_shared
    dev = logits.device
    if E_phys is None:
        E_phys = E + n_shared
    if topk_idx is None:
        topk_idx = torch.empty(T, kk, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, kk, dtype=torch.float32, device=dev)
    n_ids = 0 if replica_ids is None else replica_ids.numel()
    _check(lib.moe_route_topk_ex(_ptr(logits), T, E, k, int(renormalize), n_shared,
                                 float(shared_weight), _ptr(replica_offsets), _ptr(replica_ids),
                                 n_ids, E_phys, tokens_per_rank, _ptr(topk_idx), _ptr(topk_w),
                                 _ptr(dev_status), _stream(stream)), "moe_route_topk_ex")
    return topk_idx, topk_w


def moe_layout_workspace_bytes(T: int, k: int, E: int, R: int) -> int:
    return int(lib.moe_layout_workspace_bytes(T, k, E, R))


def moe_dispatch_layout_launches(T: int, k: int, E: int, R: int) -> int:
    return int(lib.moe_dispatch_layout_launches(T, k, E, R))


def moe_combine_bf16_long_form(T: int, H: int, k: int) -> int:
    """1 when moe_combine_bf16 runs its long (32-byte load) form for these
    sizes and 32-byte aligned buffers, else 0."""
    return int(lib.moe_combine_bf16_long_form(T, H, k))


def kernels_per_step(T: int, k: int, E: int, R: int, two_phase: bool = False) -> int:
    """Library kernels of one route -> layout -> dispatch -> combine pass
    (with two_phase, the receiver's compaction too)."""
    return 1 + moe_dispatch_layout_launches(T, k, E, R) + 1 + (1 if two_phase else 0) + 1


class Workspace:
    """A zero-filled device workspace for moe_dispatch_layout, grown on demand."""

    def __init__(self, device="cuda"):
        self.device = torch.device(device)
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws: dict[torch.device, Workspace] = {}


def moe_dispatch_layout(topk_idx: torch.Tensor, E: int, R: int, capacity: int = 0,
                        rows: int | None = None, out: dict | None = None,
                        workspace: Workspace | None = None, dev_status: torch.Tensor | None = None,
                        stream=None) -> dict:
    """Counts, offsets and index maps.  Returns a dict with expert_counts [E],
    expert_src_counts [E][R], rank_counts [R], expert_offsets [E+1],
    dispatch_pos [T][k], recv_src [rows] (int32 CUDA tensors) and ``rows``."""
    assert topk_idx.dtype == torch.int32 and topk_idx.dim() == 2
    T, k = topk_idx.shape
    dev = topk_idx.device
    if rows is None:
        rows = T * k if capacity == 0 else E * capacity
    if out is None:
        out = dict(
            expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
            expert_src_counts=torch.empty(E, R, dtype=torch.int32, device=dev),
            rank_counts=torch.empty(R, dtype=torch.int32, device=dev),
            expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            dispatch_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
            recv_src=torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
        )
    if workspace is None:
        workspace = _default_ws.setdefault(dev, Workspace(dev))
    nbytes = moe_layout_workspace_bytes(T, k, E, R)
    if nbytes == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_layout_workspace_bytes")
    ws = workspace.get(nbytes)
    _check(lib.moe_dispatch_layout(
        _ptr(topk_idx), T, k, E, R, capacity, rows,
        _ptr(out["expert_counts"]), _ptr(out["expert_src_counts"]), _ptr(out["rank_counts"]),
        _ptr(out["expert_offsets"]), _ptr(out["dispatch_pos"]), _ptr(out["recv_src"]),
        _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)), "moe_dispatch_layout")
    out["rows"] = rows
    return out


def moe_dispatch_layout_noalloc(topk_idx: torch.Tensor, E: int, R: int, capacity: int = 0,
                                rows: int | None = None, out: dict | None = None,
                                dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """moe_dispatch_layout without a workspace, for callers that cannot
    allocate device memory: the library's fixed 1 MiB device scratch is used
    instead (see include/moe_route.h).  Calls that overlap on the GPU race on
    that scratch."""
    assert topk_idx.dtype == torch.int32 and topk_idx.dim() == 2
    T, k = topk_idx.shape
    dev = topk_idx.device
    if rows is None:
        rows = T * k if capacity == 0 else E * capacity
    if out is None:
        out = dict(
            expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
            expert_src_counts=torch.empty(E, R, dtype=torch.int32, device=dev),
            rank_counts=torch.empty(R, dtype=torch.int32, device=dev),
            expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            dispatch_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
            recv_src=torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
        )
    _check(lib.moe_dispatch_layout_noalloc(
        _ptr(topk_idx), T, k, E, R, capacity, rows,
        _ptr(out["expert_counts"]), _ptr(out["expert_src_counts"]), _ptr(out["rank_counts"]),
        _ptr(out["expert_offsets"]), _ptr(out["dispatch_pos"]), _ptr(out["recv_src"]),
        _ptr(dev_status), _stream(stream)), "moe_dispatch_layout_noalloc")
    out["rows"] = rows
    return out


def moe_dispatch_layout_private(topk_idx: torch.Tensor, E: int, R: int, max_m: int,
                                rows: int | None = None, out: dict | None = None,
                                workspace: Workspace | None = None,
                                dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """Two-phase layout: everything moe_dispatch_layout (packed) returns plus
    private_pos [T][k], the row of each slot in its (expert, source rank)
    private region of max_m rows (E*R*max_m private rows in all)."""
    assert topk_idx.dtype == torch.int32 and topk_idx.dim() == 2
    T, k = topk_idx.shape
    dev = topk_idx.device
    if rows is None:
        rows = T * k
    if out is None:
        out = dict(
            expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
            expert_src_counts=torch.empty(E, R, dtype=torch.int32, device=dev),
            rank_counts=torch.empty(R, dtype=torch.int32, device=dev),
            expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
            dispatch_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
            recv_src=torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
            private_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
        )
    if workspace is None:
        workspace = _default_ws.setdefault(dev, Workspace(dev))
    nbytes = moe_layout_workspace_bytes(T, k, E, R)
    if nbytes == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_layout_workspace_bytes")
    ws = workspace.get(nbytes)
    _check(lib.moe_dispatch_layout_private(
        _ptr(topk_idx), T, k, E, R, max_m, rows,
        _ptr(out["expert_counts"]), _ptr(out["expert_src_counts"]), _ptr(out["rank_counts"]),
        _ptr(out["expert_offsets"]), _ptr(out["dispatch_pos"]), _ptr(out["recv_src"]),
        _ptr(out["private_pos"]), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)),
        "moe_dispatch_layout_private")
    out["rows"] = rows
    out["private_rows"] = E * R * max_m
    return out


def moe_compact_fp8(priv_q: torch.Tensor, priv_scale: torch.Tensor, private_pos: torch.Tensor,
                    dispatch_pos: torch.Tensor, rows: int, recv_q: torch.Tensor | None = None,
                    recv_scale: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                    stream=None):
    """Receive phase: copy each slot's private fp8 row and scales to its packed row."""
    prows, H = priv_q.shape
    T, k = dispatch_pos.shape
    if recv_q is None:
        recv_q = torch.empty(rows, H, dtype=torch.uint8, device=priv_q.device)
    if recv_scale is None:
        recv_scale = torch.empty(rows, max(H // 128, 1), dtype=torch.float32, device=priv_q.device)
    _check(lib.moe_compact_fp8(_ptr(priv_q), _ptr(priv_scale), prows, _ptr(private_pos),
                               _ptr(dispatch_pos), T, H, k, _ptr(recv_q), _ptr(recv_scale), rows,
                               _ptr(dev_status), _stream(stream)), "moe_compact_fp8")
    return recv_q, recv_scale


def moe_compact_bf16(priv_x: torch.Tensor, private_pos: torch.Tensor, dispatch_pos: torch.Tensor,
                     rows: int, recv_x: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Receive phase: copy each slot's private bf16 row to its packed row."""
    priv_x = _bits16(priv_x)
    prows, H = priv_x.shape
    T, k = dispatch_pos.shape
    if recv_x is None:
        recv_x = torch.empty(rows, H, dtype=priv_x.dtype, device=priv_x.device)
    _check(lib.moe_compact_bf16(_ptr(priv_x), prows, _ptr(private_pos), _ptr(dispatch_pos), T, H, k,
                                _ptr(recv_x), rows, _ptr(dev_status), _stream(stream)),
           "moe_compact_bf16")
    return recv_x


def moe_dispatch_bf16(x: torch.Tensor, dispatch_pos: torch.Tensor, rows: int,
                      recv_x: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """recv_x[dispatch_pos[g, j]] = x[g]; x bf16 [T][H] -> recv_x bf16 [rows][H]."""
    x = _bits16(x)
    T, H = x.shape
    k = dispatch_pos.shape[1]
    if recv_x is None:
        recv_x = torch.empty(rows, H, dtype=x.dtype, device=x.device)
    _check(lib.moe_dispatch_bf16(_ptr(x), T, H, k, _ptr(dispatch_pos), _ptr(recv_x), rows,
                                 _ptr(dev_status), _stream(stream)), "moe_dispatch_bf16")
    return recv_x


def moe_dispatch_fp8(x: torch.Tensor, dispatch_pos: torch.Tensor, rows: int,
                     recv_q: torch.Tensor | None = None, recv_scale: torch.Tensor | None = None,
                     dev_status: torch.Tensor | None = None, stream=None):
    """FP8 e4m3 dispatch with 1x128 fp32 scales: x bf16 [T][H] ->
    (recv_q uint8 [rows][H], recv_scale fp32 [rows][H/128])."""
    x = _bits16(x)
    T, H = x.shape
    k = dispatch_pos.shape[1]
    if recv_q is None:
        recv_q = torch.empty(rows, H, dtype=torch.uint8, device=x.device)
    if recv_scale is None:
        recv_scale = torch.empty(rows, max(H // 128, 1), dtype=torch.float32, device=x.device)
    _check(lib.moe_dispatch_fp8(_ptr(x), T, H, k, _ptr(dispatch_pos), _ptr(recv_q),
                                _ptr(recv_scale), rows, _ptr(dev_status), _stream(stream)),
           "moe_dispatch_fp8")
    return recv_q, recv_scale


def moe_dispatch_fp8_ex(x: torch.Tensor, dispatch_pos: torch.Tensor, rows: int,
                        scale_layout: int = MOE_SCALE_COL_MAJOR, scale_ld: int | None = None,
                        recv_q: torch.Tensor | None = None, recv_scale: torch.Tensor | None = None,
                        dev_status: torch.Tensor | None = None, stream=None):
    """moe_dispatch_fp8 with the scales column-major [H/128][scale_ld]
    (scale_ld = rows rounded up to a multiple of 4 by default) or row-major.
    Returns (recv_q uint8 [rows][H], recv_scale)."""
    x = _bits16(x)
    T, H = x.shape
    k = dispatch_pos.shape[1]
    S = max(H // 128, 1)
    if scale_ld is None:
        scale_ld = (rows + 3) // 4 * 4 if scale_layout == MOE_SCALE_COL_MAJOR else 0
    if recv_q is None:
        recv_q = torch.empty(rows, H, dtype=torch.uint8, device=x.device)
    if recv_scale is None:
        shape = (S, scale_ld) if scale_layout == MOE_SCALE_COL_MAJOR else (rows, S)
        recv_scale = torch.empty(shape, dtype=torch.float32, device=x.device)
    _check(lib.moe_dispatch_fp8_ex(_ptr(x), T, H, k, _ptr(dispatch_pos), _ptr(recv_q),
                                   _ptr(recv_scale), rows, scale_layout, scale_ld,
                                   _ptr(dev_status), _stream(stream)), "moe_dispatch_fp8_ex")
    return recv_q, recv_scale


def moe_combine_bf16(y: torch.Tensor, dispatch_pos: torch.Tensor, topk_w: torch.Tensor,
                     out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """out[g] = bf16(sum_j w[g, j] * y[dispatch_pos[g, j]]) in fp32, ascending j."""
    y = _bits16(y)
    rows, H = y.shape
    T, k = dispatch_pos.shape
    assert topk_w.dtype == torch.float32 and tuple(topk_w.shape) == (T, k)
    if out is None:
        out = torch.empty(T, H, dtype=y.dtype, device=y.device)
    _check(lib.moe_combine_bf16(_ptr(y), _ptr(dispatch_pos), _ptr(topk_w), T, H, k, rows,
                                _ptr(out), _ptr(dev_status), _stream(stream)), "moe_combine_bf16")
    return out


def moe_combine_fp8(y_q: torch.Tensor, y_scale: torch.Tensor, dispatch_pos: torch.Tensor,
                    topk_w: torch.Tensor, out: torch.Tensor | None = None,
                    dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[g] = bf16(sum_j w[g, j] * (decode(y_q[row]) * y_scale[row])) in fp32,
    ascending j.  y_q uint8 [rows][H] (E4M3), y_scale fp32 [rows][H/128]."""
    assert y_q.dtype == torch.uint8 and y_scale.dtype == torch.float32
    rows, H = y_q.shape
    T, k = dispatch_pos.shape
    assert topk_w.dtype == torch.float32 and tuple(topk_w.shape) == (T, k)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y_q.device)
    _check(lib.moe_combine_fp8(_ptr(y_q), _ptr(y_scale), _ptr(dispatch_pos), _ptr(topk_w), T, H,
                               k, rows, _ptr(out), _ptr(dev_status), _stream(stream)),
           "moe_combine_fp8")
    return out


def moe_route_dispatch_workspace_bytes(T: int, k: int, E: int, R: int) -> int:
    return int(lib.moe_route_dispatch_workspace_bytes(T, k, E, R))


# The fused entry keeps its grid barrier in the first 256 bytes of its
# workspace (zero before first use, left ready by every completed call), so it
# gets workspaces of its own, never shared with the layout's.
_default_fused_ws: dict[torch.device, Workspace] = {}


def _path_outputs(fp8: bool, T: int, k: int, E: int, R: int, H: int, rows: int, x_dtype,
                  dev) -> dict:
    """Device outputs of route + layout + dispatch (the layout over E experts
    and k slots per token)."""
    out = dict(
        topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
        topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
        expert_counts=torch.empty(E, dtype=torch.int32, device=dev),
        expert_src_counts=torch.empty(E, R, dtype=torch.int32, device=dev),
        rank_counts=torch.empty(R, dtype=torch.int32, device=dev),
        expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
        dispatch_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
        recv_src=torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
    )
    if fp8:
        out["recv_q"] = torch.empty(max(rows, 1), H, dtype=torch.uint8, device=dev)
        out["recv_scale"] = torch.empty(max(rows, 1), H // 128, dtype=torch.float32, device=dev)
    else:
        out["recv_x"] = torch.empty(max(rows, 1), H, dtype=x_dtype, device=dev)
    return out


def _route_dispatch(fp8: bool, logits, x, k, R, capacity, rows, renormalize, out, workspace,
                    dev_status, stream, ex: dict | None = None) -> dict:
    assert logits.dtype == torch.float32 and logits.dim() == 2
    x = _bits16(x)
    T, E_route = logits.shape
    k_route = k
    if ex is not None:  # the layout's view: k + n_shared slots over E_phys experts
        k = k_route + ex["n_shared"]
        E = ex["E_phys"]
    else:
        E = E_route
    H = x.shape[1]
    assert x.shape[0] == T
    dev = logits.device
    if rows is None:
        rows = T * k if capacity == 0 else E * capacity
    if out is None:
        out = _path_outputs(fp8, T, k, E, R, H, rows, x.dtype, dev)
    if workspace is None:
        workspace = _default_fused_ws.setdefault(dev, Workspace(dev))
    nbytes = moe_route_dispatch_workspace_bytes(T, k, E, R)
    if nbytes == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_route_dispatch_workspace_bytes")
    ws = workspace.get(nbytes)
    tail = (_ptr(out["topk_idx"]), _ptr(out["topk_w"]), _ptr(out["expert_counts"]),
            _ptr(out["expert_src_counts"]), _ptr(out["rank_counts"]),
            _ptr(out["expert_offsets"]), _ptr(out["dispatch_pos"]), _ptr(out["recv_src"]))
    if ex is not None:
        ids = ex.get("replica_ids")
        head = (_ptr(logits), T, E_route, k_route, int(renormalize), ex["n_shared"],
                float(ex.get("shared_weight", 1.0)), _ptr(ex.get("replica_offsets")), _ptr(ids),
                0 if ids is None else ids.numel(), E, R, capacity, _ptr(x), H) + tail
        if fp8:
            _check(lib.moe_route_dispatch_ex_fp8(*head, _ptr(out["recv_q"]),
                                                 _ptr(out["recv_scale"]), rows, _ptr(ws),
                                                 ws.numel(), _ptr(dev_status), _stream(stream)),
                   "moe_route_dispatch_ex_fp8")
        else:
            _check(lib.moe_route_dispatch_ex_bf16(*head, _ptr(out["recv_x"]), rows, _ptr(ws),
                                                  ws.numel(), _ptr(dev_status), _stream(stream)),
                   "moe_route_dispatch_ex_bf16")
        out["rows"] = rows
        return out
    common = (_ptr(logits), T, E, k, int(renormalize), R, capacity, _ptr(x), H) + tail
    if fp8:
        _check(lib.moe_route_dispatch_fp8(*common, _ptr(out["recv_q"]), _ptr(out["recv_scale"]),
                                          rows, _ptr(ws), ws.numel(), _ptr(dev_status),
                                          _stream(stream)), "moe_route_dispatch_fp8")
    else:
        _check(lib.moe_route_dispatch_bf16(*common, _ptr(out["recv_x"]), rows, _ptr(ws),
                                           ws.numel(), _ptr(dev_status), _stream(stream)),
               "moe_route_dispatch_bf16")
    out["rows"] = rows
    return out


def moe_route_dispatch_fp8(logits: torch.Tensor, x: torch.Tensor, k: int, R: int,
                           capacity: int = 0, rows: int | None = None, renormalize: bool = False,
                           out: dict | None = None, workspace: Workspace | None = None,
                           dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """Route + layout + FP8 dispatch in one cooperative launch.  Returns a dict
    with topk_idx, topk_w, the layout arrays of moe_dispatch_layout, recv_q
    [rows][H] uint8 and recv_scale [rows][H/128] fp32, and ``rows``.  A given
    ``workspace`` must be used by this entry (and _bf16) only."""
    return _route_dispatch(True, logits, x, k, R, capacity, rows, renormalize, out, workspace,
                           dev_status, stream)


def moe_route_dispatch_bf16(logits: torch.Tensor, x: torch.Tensor, k: int, R: int,
                            capacity: int = 0, rows: int | None = None, renormalize: bool = False,
                            out: dict | None = None, workspace: Workspace | None = None,
                            dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """Route + layout + bf16 dispatch in one cooperative launch (see
    moe_route_dispatch_fp8); the rows are returned as recv_x [rows][H]."""
    return _route_dispatch(False, logits, x, k, R, capacity, rows, renormalize, out, workspace,
                           dev_status, stream)


def _ex_spec(E, n_shared, shared_weight, replica_offsets, replica_ids, E_phys) -> dict:
    return dict(n_shared=n_shared, shared_weight=shared_weight, replica_offsets=replica_offsets,
                replica_ids=replica_ids, E_phys=E + n_shared if E_phys is None else E_phys)


def moe_route_dispatch_ex_fp8(logits: torch.Tensor, x: torch.Tensor, k: int, R: int,
                              n_shared: int = 0, shared_weight: float = 1.0,
                              replica_offsets: torch.Tensor | None = None,
                              replica_ids: torch.Tensor | None = None, E_phys: int | None = None,
                              capacity: int = 0, rows: int | None = None,
                              renormalize: bool = False, out: dict | None = None,
                              workspace: Workspace | None = None,
                              dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """moe_route_dispatch_fp8 with the routing of moe_route_topk_ex (shared
    experts, replicas chosen by source rank = token // (T // R)); the layout
    arrays are over E_phys experts and k + n_shared slots per token."""
    ex = _ex_spec(logits.shape[1], n_shared, shared_weight, replica_offsets, replica_ids, E_phys)
    return _route_dispatch(True, logits, x, k, R, capacity, rows, renormalize, out, workspace,
                           dev_status, stream, ex)


def moe_route_dispatch_ex_bf16(logits: torch.Tensor, x: torch.Tensor, k: int, R: int,
                               n_shared: int = 0, shared_weight: float = 1.0,
                               replica_offsets: torch.Tensor | None = None,
                               replica_ids: torch.Tensor | None = None, E_phys: int | None = None,
                               capacity: int = 0, rows: int | None = None,
                               renormalize: bool = False, out: dict | None = None,
                               workspace: Workspace | None = None,
                               dev_status: torch.Tensor | None = None, stream=None) -> dict:
    """moe_route_dispatch_bf16 with the routing of moe_route_topk_ex (see
    moe_route_dispatch_ex_fp8)."""
    ex = _ex_spec(logits.shape[1], n_shared, shared_weight, replica_offsets, replica_ids, E_phys)
    return _route_dispatch(False, logits, x, k, R, capacity, rows, renormalize, out, workspace,
                           dev_status, stream, ex)


# ---------------------------------------------------------------------------
# host-buffer entry points: inputs from, and the result to, host memory
# ---------------------------------------------------------------------------

def _route_dispatch_host(fp8: bool, logits_host, x_host, k, R, capacity, rows, renormalize, fused,
                         out, workspace, dev_status, stream, device) -> dict:
    assert logits_host.dtype == torch.float32 and logits_host.dim() == 2
    x_host = _bits16(x_host)
    T, E = logits_host.shape
    H = x_host.shape[1]
    assert x_host.shape[0] == T
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if rows is None:
        rows = T * k if capacity == 0 else E * capacity
    if out is None:
        out = _path_outputs(fp8, T, k, E, R, H, rows, x_host.dtype, dev)
        out["logits"] = torch.empty(T, E, dtype=torch.float32, device=dev)
        out["x"] = torch.empty(T, H, dtype=x_host.dtype, device=dev)
    if workspace is None:
        workspace = (_default_fused_ws if fused else _default_ws).setdefault(dev, Workspace(dev))
    nbytes = (moe_route_dispatch_workspace_bytes(T, k, E, R) if fused
              else moe_layout_workspace_bytes(T, k, E, R))
    if nbytes == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "workspace size")
    ws = workspace.get(nbytes)
    args = (_host_ptr(logits_host), _host_ptr(x_host), T, E, k, int(renormalize), R, capacity, H,
            MOE_HOST_FUSED if fused else 0, _ptr(out["logits"]), _ptr(out["x"]),
            _ptr(out["topk_idx"]), _ptr(out["topk_w"]), _ptr(out["expert_counts"]),
            _ptr(out["expert_src_counts"]), _ptr(out["rank_counts"]),
            _ptr(out["expert_offsets"]), _ptr(out["dispatch_pos"]), _ptr(out["recv_src"]))
    tail = (rows, _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    if fp8:
        _check(lib.moe_route_dispatch_fp8_host(*args, _ptr(out["recv_q"]), _ptr(out["recv_scale"]),
                                               *tail), "moe_route_dispatch_fp8_host")
    else:
        _check(lib.moe_route_dispatch_bf16_host(*args, _ptr(out["recv_x"]), *tail),
               "moe_route_dispatch_bf16_host")
    out["rows"] = rows
    return out


def moe_route_dispatch_fp8_host(logits_host: torch.Tensor, x_host: torch.Tensor, k: int, R: int,
                                capacity: int = 0, rows: int | None = None,
                                renormalize: bool = False, fused: bool = False,
                                out: dict | None = None, workspace: Workspace | None = None,
                                dev_status: torch.Tensor | None = None, stream=None,
                                device=None) -> dict:
    """Route + layout + FP8 dispatch of host logits fp32 [T][E] and host x
    bf16 [T][H]: both are copied (asynchronously when pinned) into device
    buffers ``out["logits"]``, ``out["x"]``, then the separate kernels run
    (``fused``: the single launch).  Returns the dict of
    moe_route_dispatch_fp8 plus those two buffers.  Keep the host tensors
    unchanged until the stream has passed the copies."""
    return _route_dispatch_host(True, logits_host, x_host, k, R, capacity, rows, renormalize,
                                fused, out, workspace, dev_status, stream, device)


def moe_route_dispatch_bf16_host(logits_host: torch.Tensor, x_host: torch.Tensor, k: int, R: int,
                                 capacity: int = 0, rows: int | None = None,
                                 renormalize: bool = False, fused: bool = False,
                                 out: dict | None = None, workspace: Workspace | None = None,
                                 dev_status: torch.Tensor | None = None, stream=None,
                                 device=None) -> dict:
    """moe_route_dispatch_fp8_host with the bf16 dispatch (rows in recv_x)."""
    return _route_dispatch_host(False, logits_host, x_host, k, R, capacity, rows, renormalize,
                                fused, out, workspace, dev_status, stream, device)


def moe_combine_bf16_host(y: torch.Tensor, dispatch_pos: torch.Tensor, topk_w: torch.Tensor,
                          out_host: torch.Tensor | None = None, out: torch.Tensor | None = None,
                          dev_status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """moe_combine_bf16 into the device buffer ``out``, then copied into the
    host tensor ``out_host`` (pinned when allocated here), which is returned:
    read it after the stream has been synchronised."""
    y = _bits16(y)
    rows, H = y.shape
    T, k = dispatch_pos.shape
    assert topk_w.dtype == torch.float32 and tuple(topk_w.shape) == (T, k)
    if out is None:
        out = torch.empty(T, H, dtype=y.dtype, device=y.device)
    if out_host is None:
        out_host = torch.empty(T, H, dtype=y.dtype, pin_memory=True)
    _check(lib.moe_combine_bf16_host(_ptr(y), _ptr(dispatch_pos), _ptr(topk_w), T, H, k, rows,
                                     _ptr(out), _host_ptr(out_host), _ptr(dev_status),
                                     _stream(stream)), "moe_combine_bf16_host")
    return out_host


def moe_combine_fp8_host(y_q: torch.Tensor, y_scale: torch.Tensor, dispatch_pos: torch.Tensor,
                         topk_w: torch.Tensor, out_host: torch.Tensor | None = None,
                         out: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """moe_combine_fp8 into ``out``, then copied into the host tensor
    ``out_host`` (see moe_combine_bf16_host)."""
    assert y_q.dtype == torch.uint8 and y_scale.dtype == torch.float32
    rows, H = y_q.shape
    T, k = dispatch_pos.shape
    assert topk_w.dtype == torch.float32 and tuple(topk_w.shape) == (T, k)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y_q.device)
    if out_host is None:
        out_host = torch.empty(T, H, dtype=torch.bfloat16, pin_memory=True)
    _check(lib.moe_combine_fp8_host(_ptr(y_q), _ptr(y_scale), _ptr(dispatch_pos), _ptr(topk_w), T,
                                    H, k, rows, _ptr(out), _host_ptr(out_host), _ptr(dev_status),
                                    _stream(stream)), "moe_combine_fp8_host")
    return out_host


def moe_quantize_e4m3(v: torch.Tensor, q: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """q = e4m3(v) elementwise with the dispatch kernel's converter."""
    assert v.dtype == torch.float32
    if q is None:
        q = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(lib.moe_quantize_e4m3(_ptr(v), v.numel(), _ptr(q), _stream(stream)), "moe_quantize_e4m3")
    return q
