"""The allocation-free entry point on B200: against the oracle and against the
workspace entry point.

fp8_paged_decode_attention_noalloc serves callers that cannot call cudaMalloc
(code inside a custom allocator, a plug-in whose host owns all device memory, a
path that must not create allocations): it keeps the split partials in the
library's own static device array instead of a caller workspace.  These tests
call it through the C ABI twice in a row and check each result against the
fp64 oracle and against the workspace entry point within the parity
tolerances; check that the calls change neither the device's free memory nor
torch's allocations; run a shape whose partials reach the far end of the
array; and check that a shape needing more scratch than the array holds is
refused before any launch.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_paged_decode_b200 as fpd
import oracle
from fp8_paged_decode_b200 import workloads as W
from tests.gpu_util import assert_parity, to_device

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _noalloc(lib, wl, dev, out, lse):
    vp = ctypes.c_void_p
    stream = vp(torch.cuda.current_stream().cuda_stream)
    return lib.fp8_paged_decode_attention_noalloc(
        vp(dev["q"].data_ptr()), vp(dev["k_cache"].data_ptr()), vp(dev["v_cache"].data_ptr()),
        vp(dev["block_table"].data_ptr()), vp(dev["seq_lens"].data_ptr()),
        wl.B, wl.Hq, wl.Hkv, wl.D, wl.num_blocks, wl.block_tokens, wl.max_blocks,
        ctypes.c_float(wl.k_scale), ctypes.c_float(wl.v_scale), ctypes.c_float(wl.sm_scale),
        wl.window_left, vp(dev["sinks"].data_ptr()) if dev["sinks"] is not None else None,
        vp(out.data_ptr()), vp(lse.data_ptr()), stream)


def _host(out, lse):
    return (out.float().cpu().numpy().astype(np.float64),
            lse.cpu().numpy().astype(np.float64))


def _outputs(wl, n):
    """n pairs of (out, lse) device buffers, filled with NaN."""
    return [(torch.full((wl.B, wl.Hq, wl.D), float("nan"), dtype=torch.bfloat16, device="cuda"),
             torch.full((wl.B, wl.Hq), float("nan"), dtype=torch.float32, device="cuda"))
            for _ in range(n)]


def test_noalloc_twice_matches_oracle_and_workspace_entry_point_without_allocating():
    lib = fpd.load_library()
    # window and sinks on; lengths long enough that several splits write
    # partials into the scratch
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16,
                       seq_lens=[3000, 17, 555, 4000], sinks=True, window_left=2500,
                       seed=91)
    plan = fpd.fp8_paged_decode_plan(wl.B, wl.Hq, wl.Hkv, wl.D, wl.block_tokens,
                                     wl.max_blocks, wl.window_left)
    assert plan["max_splits"] > 1
    assert plan["workspace_bytes"] <= fpd.FPD_NOALLOC_SCRATCH_BYTES
    ref_out, ref_lse = oracle.decode_workload(wl)
    dev = to_device(wl)
    ws_out, ws_lse = fpd.fp8_paged_decode_attention(
        dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
        wl.k_scale, wl.v_scale, wl.sm_scale, window_left=wl.window_left, sinks=dev["sinks"])
    torch.cuda.synchronize()
    ws_out, ws_lse = _host(ws_out, ws_lse)
    bufs = _outputs(wl, 3)
    # first call on this device: looks up the scratch address and loads the kernels
    assert _noalloc(lib, wl, dev, *bufs[0]) == fpd.FPD_OK
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for out, lse in bufs[1:]:   # two calls in a row on one stream
        st = _noalloc(lib, wl, dev, out, lse)
        assert st == fpd.FPD_OK, fpd.fp8_paged_decode_status_string(st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "device memory was allocated"
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    for i, (out, lse) in enumerate(bufs[1:]):
        o, l = _host(out, lse)
        assert_parity(o, l, ref_out, ref_lse, what=f"no-alloc call {i} vs oracle")
        assert_parity(o, l, ws_out, ws_lse, what=f"no-alloc call {i} vs workspace entry point")


def test_noalloc_partials_at_the_far_end_of_the_scratch():
    """D = 64, 16 query heads per KV head, a window and sinks, the batch sized
    so that the plan's partials fill the scratch to within 1/16 of its end.
    Every odd sequence's window starts inside a page, so it touches the plan's
    largest number of splits, and the last row's last split writes the array's
    last partial; the even sequences are short (one split), so the lengths are
    unequal and the kernel keeps the plan's split size."""
    lib = fpd.load_library()
    Hq, Hkv, D, bt, W_left, L = 64, 4, 64, 16, 511, 520
    max_blocks = (L + bt - 1) // bt
    limit = fpd.FPD_NOALLOC_SCRATCH_BYTES
    best = None
    for B in range(1, 1025):
        plan = fpd.fp8_paged_decode_plan(B, Hq, Hkv, D, bt, max_blocks, W_left)
        if plan["max_splits"] > 1 and plan["workspace_bytes"] <= limit:
            if best is None or plan["workspace_bytes"] > best[1]["workspace_bytes"]:
                best = (B, plan)
    assert best is not None
    B, plan = best
    assert plan["workspace_bytes"] > limit - limit // 16, plan
    first, end = (L - 1 - W_left) // bt, max_blocks   # the window's pages
    assert -(-(end - first) // plan["chunk_pages"]) == plan["max_splits"], plan
    assert B % 2 == 0   # the last sequence is a long one
    lens = [100 if b % 2 == 0 else L for b in range(B)]
    wl = W.make_custom(B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                       sinks=True, window_left=W_left, seed=93, sm_scale=0.125)
    assert wl.max_blocks == max_blocks
    ref_out, ref_lse = oracle.decode_workload(wl)
    dev = to_device(wl)
    for i, (out, lse) in enumerate(_outputs(wl, 2)):
        st = _noalloc(lib, wl, dev, out, lse)
        assert st == fpd.FPD_OK, fpd.fp8_paged_decode_status_string(st)
        torch.cuda.synchronize()
        o, l = _host(out, lse)
        assert_parity(o, l, ref_out, ref_lse, what=f"far end of the scratch, call {i}")


def test_noalloc_rejects_shapes_beyond_the_scratch():
    lib = fpd.load_library()
    B, Hq, Hkv, D, bt, max_blocks = 256, 64, 8, 128, 16, 2048
    plan = fpd.fp8_paged_decode_plan(B, Hq, Hkv, D, bt, max_blocks, -1)
    assert plan["workspace_bytes"] > fpd.FPD_NOALLOC_SCRATCH_BYTES
    vp = ctypes.c_void_p
    fake = vp(1 << 20)   # never dereferenced: the size check comes first
    st = lib.fp8_paged_decode_attention_noalloc(
        fake, fake, fake, fake, fake, B, Hq, Hkv, D, 10, bt, max_blocks, ctypes.c_float(1.0),
        ctypes.c_float(1.0), ctypes.c_float(0.1), -1, None, fake, fake,
        vp(torch.cuda.current_stream().cuda_stream))
    assert st == fpd.FPD_ERR_WORKSPACE_TOO_SMALL
