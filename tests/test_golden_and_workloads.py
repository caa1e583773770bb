"""Stored oracle values and the input generator's recipe (no GPU)."""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from fp8_paged_decode_b200 import workloads as W

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_golden_unchanged():
    wl = W.make_workload("tiny")
    out, lse = oracle.decode_workload(wl, threads=2)
    rows = [l.split() for l in open(os.path.join(HERE, "golden", "tiny_oracle.txt"))
            if not l.startswith("#")]
    assert len(rows) == wl.B * wl.Hq
    for r in rows:
        b, h = int(r[0]), int(r[1])
        vals = [float(x) for x in r[2:]]
        o = out[b, h]
        got = [lse[b, h], o[0], o[1], o[63], o[127], o.sum()]
        np.testing.assert_allclose(got, vals, rtol=1e-13, atol=1e-15)


def test_generator_recipe():
    wl = W.make_custom(B=3, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[5, 40, 100],
                       window_left=20, sinks=True, seed=9, keep_dense=True)
    # table: every used page distinct and inside the pool, unused slots -1
    used = []
    for b in range(wl.B):
        n = -(-int(wl.seq_lens[b]) // 16)
        assert (wl.block_table[b, :n] >= 0).all() and (wl.block_table[b, n:] == -1).all()
        used += wl.block_table[b, :n].tolist()
    assert len(set(used)) == len(used) and max(used) < wl.num_blocks
    # scale = amax/448 over attended values: the largest attended code is +-448
    att = np.concatenate([wl.k_dense[b][max(0, int(L) - 21):int(L)] for b, L in enumerate(wl.seq_lens)])
    vals = torch.from_numpy(att).view(torch.float8_e4m3fn).float().abs()
    assert vals.max().item() == 448.0
    # non-attended slots hold the NaN code
    assert (wl.k_dense[2][:100 - 21] == W.E4M3_NAN_CODE).all()
    # q is bf16 of N(0,1) samples, sinks float32 [Hq]
    assert wl.q.dtype == np.uint16 and wl.sinks.shape == (8,)


def test_configs_shapes():
    wl = W.make_workload("tiny")
    assert wl.seq_lens.tolist() == [37, 300] and wl.max_blocks == 19
    assert wl.kv_bytes() == (37 + 300) * 2 * 128 * 2
    for name in W.CONFIG_ORDER:
        c = W.CONFIGS[name]
        assert c["Hq"] % c["Hkv"] == 0


def test_generator_deterministic():
    a = W.make_custom(B=2, Hq=4, Hkv=2, D=64, block_tokens=16, seq_lens=[33, 7], seed=5)
    b = W.make_custom(B=2, Hq=4, Hkv=2, D=64, block_tokens=16, seq_lens=[33, 7], seed=5)
    assert np.array_equal(a.k_cache, b.k_cache) and np.array_equal(a.q, b.q)
    assert np.array_equal(a.block_table, b.block_table)


def test_lognormal_lengths():
    wl_lens = W._draw_lens(np.random.default_rng(0), 4096, ("lognormal", 2048.0, 1.0, 1, 32768))
    assert wl_lens.min() >= 1 and wl_lens.max() <= 32768
    assert abs(math.log(np.median(wl_lens)) - math.log(2048)) < 0.1


def test_kernel_hash_ignores_comments_only():
    """The traffic record is keyed by the kernels' code without comments: a
    comment edit keeps the key, a code edit changes it."""
    import bench
    src = 'int a = 1;  // one\n// a comment line\n\nasm("x // y");\nint b = 2;\n'
    assert bench._code_lines(src) == 'int a = 1;\nasm("x // y");\nint b = 2;'
    assert bench._code_lines(src.replace("// one", "// uno")) == bench._code_lines(src)
    assert bench._code_lines(src.replace("b = 2", "b = 3")) != bench._code_lines(src)


def test_bench_per_config_selection():
    """The default E4M3 single-query run measures every other workload after the
    headline; an explicit list or "none" overrides that; other runs measure the
    headline alone."""
    import argparse
    import bench
    base = dict(config=bench.DEFAULT_CONFIG, q_len=1, kv_format="e4m3", per_config="")
    ns = lambda **kw: argparse.Namespace(**{**base, **kw})   # noqa: E731
    others = bench.per_config_names(ns())
    assert bench.DEFAULT_CONFIG == "large_mixed" and bench.DEFAULT_CONFIG not in others
    assert sorted(others + [bench.DEFAULT_CONFIG]) == sorted(
        ["tiny", "llama3_8b", "swa_sinks", "long_context", "large_mixed"])
    assert bench.per_config_names(ns(per_config="none")) == []
    assert bench.per_config_names(ns(per_config="tiny,large_mixed")) == ["tiny"]
    assert bench.per_config_names(ns(q_len=4)) == []
    assert bench.per_config_names(ns(kv_format="nvfp4")) == []
    assert bench.per_config_names(ns(config="llama3_8b")) == []


def test_bench_per_config_entry_keeps_both_timing_forms():
    import bench
    line = {"config": {"workload": "w", "kv_bytes_per_call": 10, "plan": {"ctas": 1}},
            "us_per_call": 2.0, "value": 5.0, "pct_of_peak": 1.0, "split_kernel_us": 1.5,
            "combine_kernel_us": 0.5, "roofline": {"frac": 0.5, "traffic": None},
            "graph_replay_cold_l2": {"median_us": 3.0}, "e2e": {"value": 4.0},
            "parity_guard": {"ok": True}, "clocks": {"sm_mhz": 1}, "steps": 20, "warmup": 5}
    e = bench.per_config_entry(line)
    assert e["us_per_call"] == 2.0 and e["graph_replay_cold_l2"]["median_us"] == 3.0
    assert e["roofline_frac"] == 0.5 and e["e2e"]["value"] == 4.0 and e["steps"] == 20
