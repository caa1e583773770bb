"""CUDA path vs the fp64 CPU oracle on the same seeded inputs (B200).

Tolerances (bf16 output): |out - ref| <= 1e-2 + 1e-2 |ref| element-wise and
|lse - ref| <= 1e-3.  Unattended cache slots hold the E4M3 NaN code, so any read
outside the attended range shows up as NaN.
"""
import itertools

import numpy as np
import pytest
import torch

import fp8_paged_decode_b200 as fpd
import oracle
from fp8_paged_decode_b200 import workloads as W
from tests.gpu_util import assert_parity, run_cuda, to_device

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def check(wl, chunk_pages=0, rows=None, what=None):
    ref_out, ref_lse = oracle.decode_workload(wl, rows=rows)
    out, lse = run_cuda(wl, chunk_pages=chunk_pages)
    return assert_parity(out, lse, ref_out, ref_lse, rows=rows, what=what or wl.name)


def test_tiny_config():
    check(W.make_workload("tiny"))


GRID = list(itertools.product([64, 128], [1, 2, 4, 8, 16], [16, 32, 64], [2, 4]))


@pytest.mark.parametrize("D,g,bt,Hkv", GRID,
                         ids=[f"D{d}-g{g}-bt{b}-kv{h}" for d, g, b, h in GRID])
def test_shape_grid(D, g, bt, Hkv):
    """Hkv = 2: one KV head per stage.  Hkv = 4: four heads per stage."""
    lens = [1, bt - 1, bt, bt + 1, 3 * bt + 5, 700]
    wl = W.make_custom(B=len(lens), Hq=g * Hkv, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                       seed=100 + D + g + bt + Hkv, sm_scale=1.0 / np.sqrt(D))
    check(wl)
    check(wl, chunk_pages=64 // bt)          # 64 tokens per split: many splits + combine
    if Hkv == 4:
        check(wl, chunk_pages=10 ** 4)       # one split per sequence: output written directly


def test_stage_shape_choice():
    """The shapes above really exercise both stage layouts."""
    kw = dict(B=6, D=128, block_tokens=16, max_blocks=44, window_left=-1)
    assert fpd.fp8_paged_decode_plan(Hq=8, Hkv=2, **kw)["heads_per_stage"] == 1
    assert fpd.fp8_paged_decode_plan(Hq=16, Hkv=4, chunk_pages_override=4,
                                     **kw)["heads_per_stage"] == 4


@pytest.mark.parametrize("window,sinks", [(0, True), (5, False), (40, True), (129, True),
                                          (10 ** 6, True)])
def test_window_and_sinks(window, sinks):
    for Hkv in (2, 4):
        wl = W.make_custom(B=6, Hq=8 * Hkv, Hkv=Hkv, D=128, block_tokens=16,
                           seq_lens=[1, 2, 17, 130, 300, 1000], window_left=window, sinks=sinks,
                           seed=7 + window + Hkv, sm_scale=0.1, sigma=2.0)
        check(wl)
        check(wl, chunk_pages=4)
        check(wl, chunk_pages=10 ** 4)


@pytest.mark.parametrize("Hkv,chunk", [(2, 0), (4, 1), (4, 10 ** 4)])
def test_empty_sequence(Hkv, chunk):
    for sinks in (True, False):
        w = W.make_custom(B=3, Hq=4 * Hkv, Hkv=Hkv, D=64, block_tokens=16, seq_lens=[0, 5, 0],
                          sinks=sinks, seed=31)
        out, lse = run_cuda(w, chunk_pages=chunk)
        ref_out, ref_lse = oracle.decode_workload(w)
        assert_parity(out, lse, ref_out, ref_lse, what="empty")
        assert (out[0] == 0).all() and (out[2] == 0).all()


@pytest.mark.parametrize("chunk", [0, 1, 2, 3, 8, 40, 10 ** 4])
def test_forced_splits_agree(chunk):
    wl = W.make_custom(B=3, Hq=32, Hkv=4, D=128, block_tokens=64,
                       seq_lens=[64 * 37 + 11, 999, 64], sinks=True, seed=41)
    check(wl, chunk_pages=chunk)


def test_workspace_reused_across_calls_and_counters_reset():
    """The work counters live in the workspace and are reset by the kernel
    itself: back-to-back calls on one workspace stay correct and leave those
    words at zero."""
    wl = W.make_custom(B=5, Hq=16, Hkv=4, D=128, block_tokens=32,
                       seq_lens=[4000, 1, 2100, 640, 3333], sinks=True, seed=81)
    dev = to_device(wl)
    need = fpd.fp8_paged_decode_workspace_bytes_ex(5, 16, 4, 128, 32, wl.max_blocks, -1, 4)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ref_out, ref_lse = oracle.decode_workload(wl)
    for _ in range(3):
        out, lse = run_cuda(wl, dev, chunk_pages=4, workspace=ws)
        assert_parity(out, lse, ref_out, ref_lse, what="workspace reuse")
    words = ws[:256].view(torch.int32).cpu().numpy()
    assert (words[1:3] == 0).all(), "work counters not reset"
    assert fpd.fp8_paged_decode_check_status(ws) == 0


def test_page_permutation_bitwise():
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[3000, 17, 555, 1024],
                       sinks=True, seed=51)
    out1, lse1 = run_cuda(wl)
    perm = np.random.default_rng(3).permutation(wl.num_blocks)
    inv = np.argsort(perm)
    wl.k_cache, wl.v_cache = wl.k_cache[inv].copy(), wl.v_cache[inv].copy()
    wl.block_table = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)],
                              -1).astype(np.int32)
    out2, lse2 = run_cuda(wl)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


# Each CTA's producer warp builds the call's work list with ceil(B / 32)
# sequences per lane and one warp scan: batches that are not a multiple of 32,
# lanes holding more sequences than the loads it issues back to back (8),
# empty sequences among them, and several queries per sequence.
MANY = [(33, 1, -1), (100, 1, 64), (1000, 1, -1), (300, 3, -1)]


@pytest.mark.parametrize("B,Q,window", MANY, ids=[f"B{b}-q{q}-w{w}" for b, q, w in MANY])
def test_many_sequences_per_producer_lane(B, Q, window):
    rng = np.random.default_rng(900 + B + Q)
    lens = rng.integers(1, 400, size=B)
    if Q == 1:
        lens[::7] = 0
    wl = W.make_custom(B=B, Hq=16, Hkv=8, D=128, block_tokens=16, seq_lens=lens.tolist(),
                       window_left=window, sinks=True, seed=910 + B, q_len=Q)
    ref_out, ref_lse = oracle.decode_workload(wl)
    n = B * Q
    for chunk in (0, 3):
        out, lse = run_cuda(wl, chunk_pages=chunk)
        assert_parity(out.reshape(n, wl.Hq, wl.D), lse.reshape(n, wl.Hq),
                      ref_out.reshape(n, wl.Hq, wl.D), ref_lse.reshape(n, wl.Hq),
                      what=f"B={B} q_len={Q} window={window} chunk={chunk}")


def test_deterministic_repeat():
    wl = W.make_workload("tiny")
    dev = to_device(wl)
    a = run_cuda(wl, dev)
    b = run_cuda(wl, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_invalid_table_entries_flagged_and_contained():
    wl = W.make_custom(B=3, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[100, 200, 50],
                       seed=61)
    ref_out, ref_lse = oracle.decode_workload(wl)
    dev = to_device(wl)
    bt_bad = dev["block_table"].clone()
    bt_bad[1, 3] = wl.num_blocks + 7        # out of range
    bt_bad[1, 5] = -5                      # negative
    dev["block_table"] = bt_bad
    ws = torch.zeros(fpd.fp8_paged_decode_workspace_bytes(3, 8, 2, 128, 16, wl.max_blocks) + 256,
                     dtype=torch.uint8, device="cuda")
    out, lse = run_cuda(wl, dev, workspace=ws)
    bits = fpd.fp8_paged_decode_check_status(ws, clear=True)
    assert bits & fpd.FPD_DEVERR_BLOCK_TABLE
    assert fpd.fp8_paged_decode_check_status(ws) == 0
    # sequences with valid tables are untouched
    for b in (0, 2):
        assert_parity(out[b:b + 1], lse[b:b + 1], ref_out[b:b + 1], ref_lse[b:b + 1],
                      what="valid rows next to a bad table")
    assert np.isfinite(out[1]).all()


def test_seq_len_out_of_range_flagged():
    wl = W.make_custom(B=2, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[30, 40], seed=62)
    dev = to_device(wl)
    dev["seq_lens"] = torch.tensor([30, wl.max_blocks * 16 + 100], dtype=torch.int32,
                                   device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    run_cuda(wl, dev, workspace=ws)
    assert fpd.fp8_paged_decode_check_status(ws) & fpd.FPD_DEVERR_SEQ_LEN
    dev["seq_lens"] = torch.tensor([-3, 40], dtype=torch.int32, device="cuda")
    fpd.fp8_paged_decode_check_status(ws, clear=True)
    out, lse = run_cuda(wl, dev, workspace=ws)
    assert fpd.fp8_paged_decode_check_status(ws) & fpd.FPD_DEVERR_SEQ_LEN
    assert (out[0] == 0).all()


def test_workspace_too_small_rejected():
    wl = W.make_custom(B=2, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[3000, 40], seed=63)
    dev = to_device(wl)
    need = fpd.fp8_paged_decode_workspace_bytes_ex(2, 8, 2, 128, 16, wl.max_blocks, -1, 4)
    assert need > 256
    ws = torch.zeros(need - 4, dtype=torch.uint8, device="cuda")
    with pytest.raises(fpd.FpdError) as e:
        run_cuda(wl, dev, chunk_pages=4, workspace=ws)
    assert e.value.status == fpd.FPD_ERR_WORKSPACE_TOO_SMALL


def test_graph_capture_no_allocation():
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[2000, 10, 700, 4000],
                       sinks=True, seed=71)
    dev = to_device(wl)
    need = fpd.fp8_paged_decode_workspace_bytes(4, 32, 8, 128, 16, wl.max_blocks)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty((4, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((4, 32), dtype=torch.float32, device="cuda")
    args = (dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
            wl.k_scale, wl.v_scale, wl.sm_scale)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fpd.fp8_paged_decode_attention(*args, sinks=dev["sinks"], out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        # measured inside the capture: torch's own capture set-up may allocate
        before = torch.cuda.memory_allocated()
        fpd.fp8_paged_decode_attention(*args, sinks=dev["sinks"], out=out, lse=lse, workspace=ws)
        after = torch.cuda.memory_allocated()
    assert after == before
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.decode_workload(wl)
    assert_parity(out.float().cpu().numpy().astype(np.float64),
                  lse.cpu().numpy().astype(np.float64), ref_out, ref_lse, what="graph replay")


@pytest.mark.parametrize("name", ["tiny", "llama3_8b", "swa_sinks", "long_context",
                                  "large_mixed"])
def test_full_config_every_row(name):
    """Every (sequence, head) row of each full-size workload against the
    oracle, element by element, in the bench's launch configuration: the
    default plan, the descriptor entry point, one workspace reused by back-to-
    back calls (the second call runs on the counters the first one reset), and
    cache slots outside the attended ranges holding the E4M3 NaN code."""
    wl = W.make_workload(name)
    ref_out, ref_lse = oracle.decode_workload(wl)
    dev = to_device(wl)
    need = fpd.fp8_paged_decode_workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.D, wl.block_tokens,
                                                wl.max_blocks, wl.window_left)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    for call in range(2):
        out, lse = run_cuda(wl, dev, workspace=ws)
        assert_parity(out, lse, ref_out, ref_lse, what=f"{name}, call {call}, every row")
    assert fpd.fp8_paged_decode_check_status(ws) == 0
