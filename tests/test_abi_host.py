"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/moe_route.h declares, and rejects bad arguments
synchronously, before anything touches the CUDA runtime."""
import ctypes
import os
import re
import shutil
import subprocess

import pytest
import torch

from conftest import ROOT, build_cuda_lib

HEADER = os.path.join(ROOT, "include", "moe_route.h")

# fake device addresses: never dereferenced, because every call below must
# fail validation (or be a no-op) before a kernel could be launched
A16 = 0x10000
A4 = 0x10004


@pytest.fixture(scope="module")
def moe():
    build_cuda_lib()
    import combine_moe_route_08_b200 as m
    return m


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_path():
    names = declared_functions()
    for want in ["moe_route_topk", "moe_layout_workspace_bytes", "moe_dispatch_layout",
                 "moe_dispatch_bf16", "moe_dispatch_fp8", "moe_combine_bf16",
                 "moe_status_string", "moe_quantize_e4m3"]:
        assert want in names


def test_library_exports_every_declared_symbol(moe):
    for name in declared_functions():
        assert hasattr(moe.lib, name), name
        assert callable(getattr(moe.lib, name))


def test_python_binding_has_the_c_names(moe):
    for name in declared_functions():
        assert callable(getattr(moe, name)), name


def test_status_strings(moe):
    assert moe.moe_status_string(0) == "MOE_OK"
    assert moe.moe_status_string(3) == "MOE_ERR_CAPACITY"
    assert moe.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_bytes(moe):
    # one int32 histogram row of E per chunk; a chunk holds at most 2048 slots
    # of one logical rank.  dsv3-like decode: 32 ranks of 128 tokens -> 32 chunks
    assert moe.moe_layout_workspace_bytes(4096, 8, 256, 32) == 32 * 256 * 4
    # prefill-like: 4096 tokens per rank cut into chunks of 256 tokens
    assert moe.moe_layout_workspace_bytes(32768, 8, 256, 8) == 128 * 256 * 4
    assert moe.moe_layout_workspace_bytes(0, 2, 8, 2) == 256  # rounded up to 256 B
    for bad in [(-1, 2, 8, 2), (64, 0, 8, 2), (64, 33, 64, 2), (64, 2, 8, 3), (63, 2, 8, 2),
                (64, 9, 8, 2), (64, 2, 2048, 2)]:
        assert moe.moe_layout_workspace_bytes(*bad) == 0, bad


def test_route_rejects_bad_arguments(moe):
    f = moe.lib.moe_route_topk
    assert f(A4, 4, 8, 0, 0, A4, A4, None) == moe.MOE_ERR_INVALID_ARG      # k = 0
    assert f(A4, 4, 8, 9, 0, A4, A4, None) == moe.MOE_ERR_INVALID_ARG      # k > E
    assert f(A4, 4, 2048, 8, 0, A4, A4, None) == moe.MOE_ERR_INVALID_ARG   # E > 1024
    assert f(None, 4, 8, 2, 0, A4, A4, None) == moe.MOE_ERR_INVALID_ARG    # NULL
    assert f(A4 + 1, 4, 8, 2, 0, A4, A4, None) == moe.MOE_ERR_INVALID_ARG  # misaligned
    assert f(None, 0, 8, 2, 0, None, None, None) == moe.MOE_OK             # T = 0: no-op


def test_layout_rejects_bad_arguments(moe):
    f = moe.lib.moe_dispatch_layout
    ws = moe.moe_layout_workspace_bytes(8, 2, 4, 2)
    ok = dict(idx=A4, T=8, k=2, E=4, R=2, cap=0, rows=16, ws=A16 * 16, wsb=ws)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["idx"], a["T"], a["k"], a["E"], a["R"], a["cap"], a["rows"], A4, A4, A4, A4,
                 A4, A4, a["ws"], a["wsb"], None, None)

    assert call(R=3) == moe.MOE_ERR_INVALID_ARG            # E % R != 0
    assert call(T=7) == moe.MOE_ERR_INVALID_ARG            # T % R != 0
    assert call(rows=15) == moe.MOE_ERR_INVALID_ARG        # fewer rows than T*k
    assert call(cap=5, rows=19) == moe.MOE_ERR_INVALID_ARG  # fewer rows than E*cap
    assert call(cap=-1) == moe.MOE_ERR_INVALID_ARG
    assert call(idx=None) == moe.MOE_ERR_INVALID_ARG
    assert call(wsb=ws - 4) == moe.MOE_ERR_WORKSPACE
    assert call(ws=A16 + 16) == moe.MOE_ERR_WORKSPACE      # not 256-byte aligned
    assert call(ws=None) == moe.MOE_ERR_WORKSPACE


def test_dispatch_and_combine_reject_bad_arguments(moe):
    d16, d8, c16 = moe.lib.moe_dispatch_bf16, moe.lib.moe_dispatch_fp8, moe.lib.moe_combine_bf16
    assert d16(A16, 4, 100, 2, A4, A16, 8, None, None) == moe.MOE_ERR_INVALID_ARG   # H % 8
    assert d16(A16 + 8, 4, 256, 2, A4, A16, 8, None, None) == moe.MOE_ERR_INVALID_ARG  # x align
    assert d16(A16, 4, 256, 0, A4, A16, 8, None, None) == moe.MOE_ERR_INVALID_ARG   # k = 0
    assert d16(A16, 4, 256, 2, None, A16, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert d16(None, 0, 256, 2, None, None, 0, None, None) == moe.MOE_OK            # T = 0
    assert d8(A16, 4, 200, 2, A4, A16, A4, 8, None, None) == moe.MOE_ERR_UNSUPPORTED  # H % 128
    assert d8(A16, 4, 256, 2, A4, A16 + 4, A4, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert d8(A16, 4, 256, 2, A4, A16, A4 + 1, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(A16, A4, A4, 4, 256, 2, 8, A16 + 2, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(A16, A4, None, 4, 256, 2, 8, A16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(A16, A4, A4, 4, 256, 2, -1, A16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(None, None, None, 0, 256, 2, 0, None, None, None) == moe.MOE_OK
    assert moe.lib.moe_quantize_e4m3(A4, -1, A16, None) == moe.MOE_ERR_INVALID_ARG
    assert moe.lib.moe_quantize_e4m3(None, 0, None, None) == moe.MOE_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_cuda_error(moe):
    # arguments pass validation; the launch fails (no device) and is reported
    st = moe.lib.moe_route_topk(A4, 4, 8, 2, 0, A4, A4, None)
    assert st == moe.MOE_ERR_CUDA


def test_dispatch_fp8_ex_rejects_bad_scale_layouts(moe):
    f = moe.lib.moe_dispatch_fp8_ex
    C = moe.MOE_SCALE_COL_MAJOR
    assert f(A16, 4, 256, 2, A4, A16, A16, 8, 7, 8, None, None) == moe.MOE_ERR_INVALID_ARG  # layout
    assert f(A16, 4, 256, 2, A4, A16, A16, 8, C, 6, None, None) == moe.MOE_ERR_INVALID_ARG  # ld < rows
    assert f(A16, 4, 256, 2, A4, A16, A16, 8, C, 10, None, None) == moe.MOE_ERR_INVALID_ARG  # ld % 4
    assert f(A16, 4, 256, 2, A4, A16, A4, 8, C, 8, None, None) == moe.MOE_ERR_INVALID_ARG  # align 16
    assert f(A16, 4, 200, 2, A4, A16, A16, 8, C, 8, None, None) == moe.MOE_ERR_UNSUPPORTED
    assert f(None, 0, 256, 2, None, None, None, 0, C, 0, None, None) == moe.MOE_OK


def test_two_phase_entries_reject_bad_arguments(moe):
    f = moe.lib.moe_dispatch_layout_private
    ws = moe.moe_layout_workspace_bytes(8, 2, 4, 2)
    args = lambda max_m=2, rows=16, wsb=ws: (A4, 8, 2, 4, 2, max_m, rows, A4, A4, A4, A4, A4, A4, A4,
                                             A16 * 16, wsb, None, None)
    assert f(*args(max_m=0)) == moe.MOE_ERR_INVALID_ARG
    assert f(*args(rows=15)) == moe.MOE_ERR_INVALID_ARG
    assert f(*args(max_m=1 << 28)) == moe.MOE_ERR_INVALID_ARG     # E*R*max_m >= 2^31
    assert f(*args(wsb=ws - 4)) == moe.MOE_ERR_WORKSPACE
    c8, c16 = moe.lib.moe_compact_fp8, moe.lib.moe_compact_bf16
    assert c8(A16, A4, 8, A4, A4, 4, 200, 2, A16, A4, 8, None, None) == moe.MOE_ERR_UNSUPPORTED
    assert c8(A16, A4, -1, A4, A4, 4, 256, 2, A16, A4, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c8(A16 + 4, A4, 8, A4, A4, 4, 256, 2, A16, A4, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(A16, 8, None, A4, 4, 256, 2, A16, 8, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(None, 0, None, None, 0, 256, 2, None, 0, None, None) == moe.MOE_OK


def test_fused_route_dispatch_rejects_bad_arguments(moe):
    for bad in [(-1, 2, 8, 2), (64, 0, 8, 2), (64, 2, 8, 3), (63, 2, 8, 2)]:
        assert moe.moe_route_dispatch_workspace_bytes(*bad) == 0, bad
    f8, f16 = moe.lib.moe_route_dispatch_fp8, moe.lib.moe_route_dispatch_bf16
    ws = 0x100000  # 256-byte aligned fake address

    def call8(T=64, E=8, k=2, R=2, cap=0, x=A16, H=256, rows=128, wsp=ws, recv_q=A16,
              scale=A4, logits=A4):
        return f8(logits, T, E, k, 0, R, cap, x, H, A4, A4, A4, A4, A4, A4, A4, A4, recv_q,
                  scale, rows, wsp, 1 << 20, None, None)

    assert call8(k=0) == moe.MOE_ERR_INVALID_ARG
    assert call8(k=9) == moe.MOE_ERR_INVALID_ARG            # k > E
    assert call8(R=3) == moe.MOE_ERR_INVALID_ARG            # E % R != 0
    assert call8(T=63) == moe.MOE_ERR_INVALID_ARG           # T % R != 0
    assert call8(H=204) == moe.MOE_ERR_INVALID_ARG          # H % 8 != 0
    assert call8(H=264) == moe.MOE_ERR_UNSUPPORTED          # fp8 needs H % 128 == 0
    assert call8(H=1 << 21) == moe.MOE_ERR_INVALID_ARG      # H > 2^20
    assert call8(rows=127) == moe.MOE_ERR_INVALID_ARG       # packed rows < T*k
    assert call8(cap=4, rows=31) == moe.MOE_ERR_INVALID_ARG  # padded rows < E*cap
    assert call8(x=A16 + 8) == moe.MOE_ERR_INVALID_ARG      # x not 16-byte aligned
    assert call8(recv_q=A16 + 4) == moe.MOE_ERR_INVALID_ARG
    assert call8(scale=None) == moe.MOE_ERR_INVALID_ARG
    assert call8(logits=None) == moe.MOE_ERR_INVALID_ARG
    assert call8(wsp=None) == moe.MOE_ERR_WORKSPACE
    assert call8(wsp=ws + 128) == moe.MOE_ERR_WORKSPACE     # not 256-byte aligned
    assert f16(A4, 64, 8, 2, 0, 2, 0, A16, 204, A4, A4, A4, A4, A4, A4, A4, A4, A16, 128, ws,
               1 << 20, None, None) == moe.MOE_ERR_INVALID_ARG
    assert f16(A4, 64, 8, 2, 0, 2, 0, A16, 56, A4, A4, A4, A4, A4, A4, A4, A4, A16, 128, ws,
               1 << 20, None, None) == moe.MOE_ERR_UNSUPPORTED   # bf16 needs H >= 64


def test_fused_route_dispatch_ex_rejects_bad_arguments(moe):
    f8, f16 = moe.lib.moe_route_dispatch_ex_fp8, moe.lib.moe_route_dispatch_ex_bf16
    ws = 0x100000

    def call8(T=64, E=8, k=2, ns=1, offs=None, ids=None, nids=0, Ep=10, R=2, cap=0, H=256,
              rows=192, wsp=ws):
        return f8(A4, T, E, k, 0, ns, 1.0, offs, ids, nids, Ep, R, cap, A16, H, A4, A4, A4, A4,
                  A4, A4, A4, A4, A16, A4, rows, wsp, 1 << 20, None, None)

    assert call8(ns=-1) == moe.MOE_ERR_INVALID_ARG
    assert call8(k=0) == moe.MOE_ERR_INVALID_ARG
    assert call8(k=9) == moe.MOE_ERR_INVALID_ARG              # k > E
    assert call8(k=30, E=64, ns=3, Ep=68) == moe.MOE_ERR_INVALID_ARG  # k + n_shared > 32
    assert call8(Ep=8) == moe.MOE_ERR_INVALID_ARG             # no table: E_phys < E + n_shared
    assert call8(Ep=1025) == moe.MOE_ERR_INVALID_ARG          # E_phys > 1024
    assert call8(Ep=9) == moe.MOE_ERR_INVALID_ARG             # R = 2 does not divide E_phys
    assert call8(offs=A4, ids=None, nids=4) == moe.MOE_ERR_INVALID_ARG  # table without ids
    assert call8(offs=A4, ids=A4, nids=0) == moe.MOE_ERR_INVALID_ARG
    assert call8(offs=A4 + 2, ids=A4, nids=4) == moe.MOE_ERR_INVALID_ARG  # misaligned table
    assert call8(rows=191) == moe.MOE_ERR_INVALID_ARG         # packed rows < T * (k + n_shared)
    assert call8(cap=4, rows=39) == moe.MOE_ERR_INVALID_ARG   # padded rows < E_phys * cap
    assert call8(H=264) == moe.MOE_ERR_UNSUPPORTED
    assert call8(wsp=None) == moe.MOE_ERR_WORKSPACE
    assert f16(A4, 64, 8, 2, 0, 1, 1.0, None, None, 0, 10, 2, 0, A16, 56, A4, A4, A4, A4, A4, A4,
               A4, A4, A16, 192, ws, 1 << 20, None, None) == moe.MOE_ERR_UNSUPPORTED


def test_combine_fp8_rejects_bad_arguments(moe):
    f = moe.lib.moe_combine_fp8
    assert f(A16, A4, A4, A4, 4, 200, 2, 8, A16, None, None) == moe.MOE_ERR_UNSUPPORTED  # H % 128
    assert f(A16, A4, A4, A4, 4, 128, 0, 8, A16, None, None) == moe.MOE_ERR_INVALID_ARG  # k = 0
    assert f(A16 + 4, A4, A4, A4, 4, 128, 2, 8, A16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert f(A16, None, A4, A4, 4, 128, 2, 8, A16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert f(None, None, None, None, 0, 128, 2, 0, None, None, None) == moe.MOE_OK  # T = 0


def test_layout_launch_count_on_the_host(moe):
    """The launch count is a host query: 0 for invalid sizes, 2 (histogram +
    placement) for layouts beyond the single-launch limit, 1 or 2 for small
    ones (1 only where a device can schedule the cluster)."""
    assert moe.moe_dispatch_layout_launches(64, 2, 8, 3) == 0          # R does not divide E
    assert moe.moe_dispatch_layout_launches(-1, 2, 8, 2) == 0
    assert moe.moe_dispatch_layout_launches(4096, 8, 256, 32) == 2     # 32768 slots
    assert moe.moe_dispatch_layout_launches(32768, 8, 256, 8) == 2     # 16 chunks per rank
    assert moe.moe_dispatch_layout_launches(64, 2, 8, 2) in (1, 2)
    assert moe.kernels_per_step(4096, 8, 256, 32) == 5


def test_host_buffer_entries_reject_bad_arguments(moe):
    """Every step's arguments are checked before a copy is enqueued: a bad
    flag, a NULL host buffer, a bad route, layout, dispatch or workspace
    argument, and the combine's missing host output."""
    f8, f16 = moe.lib.moe_route_dispatch_fp8_host, moe.lib.moe_route_dispatch_bf16_host
    ws = 0x100000
    wsb = moe.moe_layout_workspace_bytes(64, 2, 8, 2)

    def call8(lh=A16, xh=A16, T=64, E=8, k=2, R=2, cap=0, H=256, flags=0, x=A16, rows=128,
              wsp=ws, nbytes=wsb, recv_q=A16):
        return f8(lh, xh, T, E, k, 0, R, cap, H, flags, A4, x, A4, A4, A4, A4, A4, A4, A4, A4,
                  recv_q, A4, rows, wsp, nbytes, None, None)

    assert call8(flags=2) == moe.MOE_ERR_INVALID_ARG          # unknown flag bit
    assert call8(lh=None) == moe.MOE_ERR_INVALID_ARG          # no host logits with T > 0
    assert call8(xh=None) == moe.MOE_ERR_INVALID_ARG
    assert call8(k=0) == moe.MOE_ERR_INVALID_ARG              # route
    assert call8(R=3) == moe.MOE_ERR_INVALID_ARG              # layout: E % R != 0
    assert call8(rows=127) == moe.MOE_ERR_INVALID_ARG         # layout: rows < T*k
    assert call8(nbytes=wsb - 4) == moe.MOE_ERR_WORKSPACE     # layout workspace short
    assert call8(wsp=None) == moe.MOE_ERR_WORKSPACE
    assert call8(H=264) == moe.MOE_ERR_UNSUPPORTED            # fp8 dispatch: H % 128
    assert call8(x=A16 + 8) == moe.MOE_ERR_INVALID_ARG        # staging x not 16-byte aligned
    assert call8(recv_q=A16 + 4) == moe.MOE_ERR_INVALID_ARG
    assert call8(flags=moe.MOE_HOST_FUSED, H=264) == moe.MOE_ERR_UNSUPPORTED
    assert call8(flags=moe.MOE_HOST_FUSED, wsp=None) == moe.MOE_ERR_WORKSPACE
    assert f16(A16, A16, 64, 8, 2, 0, 2, 0, 100, 0, A4, A16, A4, A4, A4, A4, A4, A4, A4, A4, A16,
               128, ws, wsb, None, None) == moe.MOE_ERR_INVALID_ARG   # H % 8
    c16, c8 = moe.lib.moe_combine_bf16_host, moe.lib.moe_combine_fp8_host
    assert c16(A16, A4, A4, 4, 256, 2, 8, A16, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(A16, A4, A4, 4, 256, 2, 8, A16 + 2, A16, None, None) == moe.MOE_ERR_INVALID_ARG
    assert c16(None, None, None, 0, 256, 2, 0, None, None, None, None) == moe.MOE_OK  # T = 0
    assert c8(A16, A4, A4, A4, 4, 200, 2, 8, A16, A16, None, None) == moe.MOE_ERR_UNSUPPORTED
    assert c8(A16, A4, A4, A4, 4, 256, 2, 8, A16, None, None, None) == moe.MOE_ERR_INVALID_ARG


def test_combine_long_form_query(moe):
    """The bf16 combine's long form is chosen from the sizes alone: k <= 8,
    H % 16 == 0 and at least 2 GiB of rows read."""
    assert moe.moe_combine_bf16_long_form(32768, 7168, 8) == 1     # 3.76 GB of rows
    assert moe.moe_combine_bf16_long_form(16384, 8192, 8) == 1     # exactly 2 GiB
    assert moe.moe_combine_bf16_long_form(16383, 8192, 8) == 0
    assert moe.moe_combine_bf16_long_form(4096, 7168, 8) == 0      # decode sizes
    assert moe.moe_combine_bf16_long_form(32768, 7168, 9) == 0     # k > 8
    assert moe.moe_combine_bf16_long_form(65536, 7160, 8) == 0     # H % 16 != 0
    assert moe.moe_combine_bf16_long_form(-1, 7168, 8) == 0


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_header_is_plain_c():
    """include/moe_route.h compiles as C99 on its own (no C++ or CUDA types in
    the boundary) and as C++17."""
    for lang, std in (("c", "-std=c99"), ("c++", "-std=c++17")):
        p = subprocess.run(["gcc", std, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", lang,
                            HEADER], capture_output=True, text=True, timeout=60)
        assert p.returncode == 0, p.stderr
