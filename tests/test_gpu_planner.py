"""The split kernel's own choice between the plan's split size and the larger
one it offers for calls of a few rounds of items (equal-length sequences),
checked against the fp64 oracle, together with the split size the call
reports in the workspace header (word 3).  Tolerances as everywhere:
|out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3."""
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


CASES = {  # Hq, Hkv, D, bt, lens, max_blocks, q_len, larger split taken
    "equal-64-token-pages": (32, 8, 128, 64, [16384] * 4, None, 1, True),
    "equal-one-head-stages": (8, 2, 128, 16, [16384] * 8, None, 1, True),
    "equal-several-queries": (64, 8, 64, 64, [16384] * 2, None, 3, True),
    "unequal-lengths": (32, 8, 128, 64, [16384, 3000, 9000, 16000], None, 1, False),
    "short-in-wide-table": (32, 8, 128, 64, [4096] * 4, 256, 1, False),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_split_size_choice(name):
    Hq, Hkv, D, bt, lens, mb, Q, taken = CASES[name]
    wl = W.make_custom(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                       max_blocks=mb, q_len=Q, sinks=True, seed=700 + len(name))
    plan = fpd.fp8_paged_decode_plan_qlen(wl.B, Q, Hq, Hkv, D, bt, wl.max_blocks, -1)
    assert plan["adapt_chunk_pages"] > plan["chunk_pages"]
    dev = to_device(wl)
    ws = torch.zeros(plan["workspace_bytes"], dtype=torch.uint8, device="cuda")
    out, lse = fpd.fp8_paged_decode_attention(dev["q"], dev["k_cache"], dev["v_cache"],
                                              dev["block_table"], dev["seq_lens"], wl.k_scale,
                                              wl.v_scale, wl.sm_scale, sinks=dev["sinks"],
                                              workspace=ws)
    torch.cuda.synchronize()
    used = int(ws[12:16].view(torch.int32).item())
    assert used == (plan["adapt_chunk_pages"] if taken else plan["chunk_pages"])
    assert fpd.fp8_paged_decode_check_status(ws) == 0
    ro, rl = oracle.decode_workload(wl)
    n = wl.B * Q
    assert_parity(out.float().cpu().numpy().reshape(n, Hq, D).astype(np.float64),
                  lse.cpu().numpy().reshape(n, Hq).astype(np.float64),
                  ro.reshape(n, Hq, D), rl.reshape(n, Hq), what=name)


def test_forced_split_size_is_kept():
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=64, seq_lens=[16384] * 4, seed=9)
    dev = to_device(wl)
    need = fpd.fp8_paged_decode_workspace_bytes_ex(4, 32, 8, 128, 64, wl.max_blocks, -1, 4)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out, lse = fpd.fp8_paged_decode_attention(dev["q"], dev["k_cache"], dev["v_cache"],
                                              dev["block_table"], dev["seq_lens"], wl.k_scale,
                                              wl.v_scale, wl.sm_scale, workspace=ws,
                                              chunk_pages_override=4)
    torch.cuda.synchronize()
    assert int(ws[12:16].view(torch.int32).item()) == 4
    ro, rl = oracle.decode_workload(wl)
    assert_parity(out.float().cpu().numpy().astype(np.float64),
                  lse.cpu().numpy().astype(np.float64), ro, rl, what="forced split size")
