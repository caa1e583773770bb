"""Several query tokens per sequence (causal within the new tokens) vs the fp64
oracle: |out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3, element-wise."""
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


def check(wl, chunk_pages=0, what=None):
    ref_out, ref_lse = oracle.decode_workload(wl)
    out, lse = run_cuda(wl, chunk_pages=chunk_pages)
    B, Q = wl.B, wl.q_len
    assert out.shape == (B, Q, wl.Hq, wl.D) and lse.shape == (B, Q, wl.Hq)
    return assert_parity(out.reshape(B * Q, wl.Hq, wl.D), lse.reshape(B * Q, wl.Hq),
                         ref_out.reshape(B * Q, wl.Hq, wl.D), ref_lse.reshape(B * Q, wl.Hq),
                         what=what or f"{wl.name} q_len={Q} chunk={chunk_pages}")


# (g, q_len) with q_len * g <= 16: one and two MMA n-tiles
GQ = [(1, 2), (1, 5), (1, 16), (2, 3), (2, 8), (4, 2), (4, 4), (8, 2)]
GRID = list(itertools.product(GQ, [2, 4], [64, 128], [16, 64]))


@pytest.mark.parametrize("gq,Hkv,D,bt", GRID,
                         ids=[f"g{g}-q{q}-kv{h}-D{d}-bt{b}" for (g, q), h, d, b in GRID])
def test_grid(gq, Hkv, D, bt):
    g, Q = gq
    lens = [1, Q, Q + 1, bt - 1, 3 * bt + 5, 700]
    wl = W.make_custom(B=len(lens), Hq=g * Hkv, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                       seed=300 + g + Q + Hkv + D + bt, sm_scale=1.0 / np.sqrt(D), sinks=True,
                       q_len=Q)
    check(wl)
    check(wl, chunk_pages=64 // bt)   # many splits: early queries see no key in the last ones
    if Hkv == 4:
        check(wl, chunk_pages=1)      # four-head stages, one page per split


# more than 16 columns: a sequence's queries are cut into several work items
GQC = [(1, 17), (2, 9), (4, 5), (4, 8), (8, 3), (8, 8), (16, 2), (16, 3)]
GRIDC = list(itertools.product(GQC, [2, 4], [64, 128]))


@pytest.mark.parametrize("gq,Hkv,D", GRIDC,
                         ids=[f"g{g}-q{q}-kv{h}-D{d}" for (g, q), h, d in GRIDC])
def test_query_chunks(gq, Hkv, D):
    g, Q = gq
    lens = [1, Q - 1, Q, 2 * Q + 1, 37, 300, 700]
    wl = W.make_custom(B=len(lens), Hq=g * Hkv, Hkv=Hkv, D=D, block_tokens=16, seq_lens=lens,
                       seed=500 + g + Q + Hkv + D, sm_scale=1.0 / np.sqrt(D), sinks=True,
                       q_len=Q)
    check(wl)
    check(wl, chunk_pages=2)
    wl.window_left = 20
    check(wl, what=f"{wl.name} q_len={Q} window 20")


@pytest.mark.parametrize("window", [0, 3, 40, 129, 10 ** 6])
def test_windows(window):
    for Hkv, Q in ((2, 4), (4, 3)):
        wl = W.make_custom(B=5, Hq=4 * Hkv, Hkv=Hkv, D=128, block_tokens=16,
                           seq_lens=[2, 5, 130, 300, 1000], window_left=window, sinks=True,
                           seed=400 + window + Q, sm_scale=0.1, sigma=2.0, q_len=Q)
        check(wl)
        check(wl, chunk_pages=2)


def test_one_query_matches_the_single_query_entry_bitwise():
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[3000, 17, 555, 1024],
                       sinks=True, seed=61)
    dev = to_device(wl)
    a_out, a_lse = run_cuda(wl, dev)
    q4 = dev["q"].unsqueeze(1)                        # [B, 1, Hq, D]
    b_out, b_lse = fpd.fp8_paged_decode_attention(q4, dev["k_cache"], dev["v_cache"],
                                                  dev["block_table"], dev["seq_lens"],
                                                  wl.k_scale, wl.v_scale, wl.sm_scale,
                                                  sinks=dev["sinks"])
    torch.cuda.synchronize()
    assert np.array_equal(a_out, b_out[:, 0].float().cpu().numpy())
    assert np.array_equal(a_lse, b_lse[:, 0].cpu().numpy())


def test_unsupported_q_len():
    Q = fpd.FPD_MAX_Q_LEN + 1
    wl = W.make_custom(B=2, Hq=4, Hkv=2, D=64, block_tokens=16, seq_lens=[70, 80], seed=62,
                       q_len=Q)
    dev = to_device(wl)
    with pytest.raises(fpd.FpdError) as e:
        fpd.fp8_paged_decode_attention(dev["q"], dev["k_cache"], dev["v_cache"],
                                       dev["block_table"], dev["seq_lens"], wl.k_scale,
                                       wl.v_scale, wl.sm_scale)
    assert e.value.status == fpd.FPD_ERR_UNSUPPORTED


@pytest.mark.parametrize("name,Q", [("llama3_8b", 4), ("large_mixed", 2)])
def test_full_workload_speculative_every_row(name, Q):
    """The full-size workloads with Q draft tokens per sequence (the bench's
    `--q-len Q` calls): every (sequence, query, head) row against the oracle in
    the default launch configuration."""
    wl = W.make_workload(name, q_len=Q)
    ref_out, ref_lse = oracle.decode_workload(wl)
    out, lse = run_cuda(wl)
    assert out.shape == ref_out.shape == (wl.B, Q, wl.Hq, wl.D)
    assert_parity(out, lse, ref_out, ref_lse, what=f"{name} q_len={Q}, every row")


@pytest.mark.parametrize("g,Hkv", [(1, 4), (16, 1)])
def test_max_q_len(g, Hkv):
    """q_len at its limit: 64 queries per sequence (4 items of 16 positions for
    g = 1, 64 one-position items for g = 16)."""
    Q = fpd.FPD_MAX_Q_LEN
    lens = [Q - 10, Q, 200, 1000]
    wl = W.make_custom(B=len(lens), Hq=g * Hkv, Hkv=Hkv, D=64, block_tokens=16, seq_lens=lens,
                       seed=700 + g, sm_scale=0.125, sinks=True, q_len=Q)
    check(wl)
    check(wl, chunk_pages=3)
    wl.window_left = 30
    check(wl, what=f"q_len {Q} window 30")
