"""The allocation-free entry point against the workspace entry point (B200).

fp8_paged_decode_attention_noalloc serves callers that cannot call cudaMalloc
(code inside a custom allocator, a plug-in whose host owns all device memory, a
path that must not create allocations): it keeps the split partials in the
library's own static device array instead of a caller workspace.  This test
calls it through the C ABI twice in a row and checks each result against the
workspace entry point within the parity tolerances, and checks that a shape
needing more scratch than the static array holds is refused before any launch.
The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_paged_decode_b200 as fpd
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


def test_noalloc_matches_workspace_entry_point_twice():
    lib = fpd.load_library()
    # lengths long enough that several splits write partials into the scratch
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16,
                       seq_lens=[3000, 17, 555, 4000], sinks=True, window_left=2500,
                       seed=91)
    plan = fpd.fp8_paged_decode_plan(wl.B, wl.Hq, wl.Hkv, wl.D, wl.block_tokens,
                                     wl.max_blocks, wl.window_left)
    assert plan["max_splits"] > 1
    assert plan["workspace_bytes"] <= fpd.FPD_NOALLOC_SCRATCH_BYTES
    dev = to_device(wl)
    ref_out, ref_lse = fpd.fp8_paged_decode_attention(
        dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
        wl.k_scale, wl.v_scale, wl.sm_scale, window_left=wl.window_left, sinks=dev["sinks"])
    torch.cuda.synchronize()
    ref_out = ref_out.float().cpu().numpy().astype(np.float64)
    ref_lse = ref_lse.cpu().numpy().astype(np.float64)
    for _ in range(2):
        out = torch.full((wl.B, wl.Hq, wl.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((wl.B, wl.Hq), float("nan"), dtype=torch.float32, device="cuda")
        st = _noalloc(lib, wl, dev, out, lse)
        assert st == fpd.FPD_OK, fpd.fp8_paged_decode_status_string(st)
        torch.cuda.synchronize()
        assert_parity(out.float().cpu().numpy().astype(np.float64),
                      lse.cpu().numpy().astype(np.float64), ref_out, ref_lse,
                      what="no-alloc entry point vs workspace entry point")


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
