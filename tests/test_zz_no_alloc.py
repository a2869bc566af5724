"""moe_dispatch_layout_noalloc: the layout for callers that cannot allocate
device memory (a plugin handed only its buffers, a loop where cudaMalloc
would synchronise the device, a fixed memory budget).  It uses the library's
fixed 1 MiB device scratch instead of a caller workspace.

Called through the C ABI (ctypes, raw device pointers) twice in a row on
different routings, each time compared with moe_dispatch_layout given its
own workspace and with the oracle's layout: the outputs are integer maps, so
they must be identical.  The size limit is checked at its exact boundary.
The file is collected last so that a failure here leaves every other test
run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from harness import inputs

pytestmark = pytest.mark.gpu

KEYS = ["expert_counts", "expert_src_counts", "rank_counts", "expert_offsets", "dispatch_pos",
        "recv_src"]


def _alloc(T, k, E, R, rows, dev):
    return dict(
        expert_counts=torch.full((E,), -5, dtype=torch.int32, device=dev),
        expert_src_counts=torch.full((E, R), -5, dtype=torch.int32, device=dev),
        rank_counts=torch.full((R,), -5, dtype=torch.int32, device=dev),
        expert_offsets=torch.full((E + 1,), -5, dtype=torch.int32, device=dev),
        dispatch_pos=torch.full((T, k), -5, dtype=torch.int32, device=dev),
        recv_src=torch.full((rows,), -5, dtype=torch.int32, device=dev),
    )


def _ptrs(out):
    return [out[key].data_ptr() for key in KEYS]


def _routing(name):
    cfg = inputs.CONFIGS[name]
    idx, _ = oracle.route(inputs.make_logits(cfg).numpy(), cfg.k)
    cap = 0
    if cfg.layout == "padded":
        cap = int(oracle.layout(idx, cfg.E, cfg.R)["expert_counts"].max())
    return cfg, torch.from_numpy(idx).cuda(), cap


def test_noalloc_layout_matches_workspace_layout_twice_in_a_row():
    import combine_moe_route_08_b200 as moe
    lib = moe.lib
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream().cuda_stream or None
    for name in ["kimi", "prefill"]:          # two calls in a row, different shapes
        cfg, idx, cap = _routing(name)
        T, k, E, R = cfg.T, cfg.k, cfg.E, cfg.R
        rows = T * k if cap == 0 else E * cap
        st_a = torch.zeros(1, dtype=torch.int32, device=dev)
        st_b = torch.zeros(1, dtype=torch.int32, device=dev)

        # the existing entry point with a caller workspace
        want = _alloc(T, k, E, R, rows, dev)
        nbytes = lib.moe_layout_workspace_bytes(T, k, E, R)
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        rc = lib.moe_dispatch_layout(idx.data_ptr(), T, k, E, R, cap, rows, *_ptrs(want),
                                     ws.data_ptr(), nbytes, st_a.data_ptr(), stream)
        assert rc == moe.MOE_OK

        # the allocation-free entry point
        got = _alloc(T, k, E, R, rows, dev)
        rc = lib.moe_dispatch_layout_noalloc(idx.data_ptr(), T, k, E, R, cap, rows, *_ptrs(got),
                                             st_b.data_ptr(), stream)
        assert rc == moe.MOE_OK
        torch.cuda.synchronize()
        ref = oracle.layout(idx.cpu().numpy(), E, R, cap, rows)
        for key in KEYS:
            assert torch.equal(got[key], want[key]), f"{name}: {key}"
            assert np.array_equal(got[key].cpu().numpy(), ref[key].reshape(got[key].shape)), \
                f"{name}: {key} vs the oracle"
        assert st_a.item() == st_b.item() == 0


def _noalloc_bytes(T, k, E, R):
    """The documented size of the scratch a (T, k, E, R) needs: one E-wide
    int32 histogram row per chunk of at most floor(2048 / k) tokens of one
    logical rank, rounded up to 256 bytes (at least 256)."""
    per_chunk = max(1, 2048 // k)
    chunks = R * max(1, -(-(T // R) // per_chunk))
    return max(256, -(-chunks * E * 4 // 256) * 256)


def test_noalloc_limit_at_its_exact_boundary():
    """E = 1024, k = 8, R = 256: 256 tokens per rank fill one chunk per rank,
    256 rows of 4 KiB = exactly the 1 MiB scratch, and run (compared with
    the oracle); 257 tokens per rank need a second, almost empty chunk per
    rank and are rejected although T * k is far below 2^21."""
    import combine_moe_route_08_b200 as moe
    lib = moe.lib
    limit = moe.MOE_LAYOUT_NOALLOC_SCRATCH_BYTES
    E, k, R = 1024, 8, 256
    T_fit, T_over = 256 * R, 257 * R
    assert lib.moe_layout_workspace_bytes(T_fit, k, E, R) == _noalloc_bytes(T_fit, k, E, R) == limit
    assert lib.moe_layout_workspace_bytes(T_over, k, E, R) == _noalloc_bytes(T_over, k, E, R) > limit
    fake = ctypes.c_void_p(0x10000)
    rc = lib.moe_dispatch_layout_noalloc(fake, T_over, k, E, R, 0, T_over * k, fake, fake, fake,
                                         fake, fake, fake, None, None)
    assert rc == moe.MOE_ERR_WORKSPACE
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(5)
    idx_np = np.argsort(rng.random((T_fit, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    idx = torch.from_numpy(idx_np).cuda()
    rows = T_fit * k
    got = _alloc(T_fit, k, E, R, rows, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = lib.moe_dispatch_layout_noalloc(idx.data_ptr(), T_fit, k, E, R, 0, rows, *_ptrs(got),
                                         st.data_ptr(), torch.cuda.current_stream().cuda_stream or None)
    assert rc == moe.MOE_OK
    torch.cuda.synchronize()
    ref = oracle.layout(idx_np, E, R)
    for key in KEYS:
        assert np.array_equal(got[key].cpu().numpy(), ref[key].reshape(got[key].shape)), key
    assert st.item() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import combine_moe_route_08_b200 as moe
    lib = moe.lib
    # E = 1024 experts and 512 logical ranks: 512 chunks x 1024 int32 = 2 MiB
    T, k, E, R = 512, 8, 1024, 512
    assert lib.moe_layout_workspace_bytes(T, k, E, R) > (1 << 20)
    fake = ctypes.c_void_p(0x10000)
    rc = lib.moe_dispatch_layout_noalloc(fake, T, k, E, R, 0, T * k, fake, fake, fake, fake,
                                         fake, fake, None, None)
    assert rc == moe.MOE_ERR_WORKSPACE
