"""Context-parallel decode on the CPU: the key partition (cp_shard), the
partial-buffer layout, the oracle's merge pinned against the oracle's own
decode over all keys, and the exchange as two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from fp8_paged_decode_b200 import cp
from fp8_paged_decode_b200 import workloads as W


def test_shard_covers_every_page_once_in_order():
    rng = np.random.default_rng(3)
    for world in (1, 2, 3, 8):
        for bt in (1, 16, 64):
            lens = rng.integers(0, 40 * bt, size=7)
            lens[0] = 0
            lens[1] = 1
            pages = -(-lens // bt)
            width = int(max(1, pages.max()))
            table = rng.permutation(10_000)[: 7 * width].reshape(7, width).astype(np.int32)
            shards = [cp.cp_shard(table, lens, world, r, bt) for r in range(world)]
            for b in range(7):
                got_pages, got_tokens = [], 0
                counts = []
                for r, (t_r, l_r) in enumerate(shards):
                    n = -(-int(l_r[b]) // bt)
                    counts.append(n)
                    got_pages += list(t_r[b, :n])
                    got_tokens += int(l_r[b])
                    # whole pages, except at the end of the sequence
                    if l_r[b] % bt and sum(counts) != pages[b]:
                        pytest.fail("a partly filled page before the sequence's end")
                assert got_pages == list(table[b, : pages[b]])
                assert got_tokens == lens[b]
                assert max(counts) - min(counts) <= 1


def test_shard_rejects_bad_ranks():
    with pytest.raises(ValueError):
        cp.cp_shard(np.zeros((1, 1), np.int32), [3], 2, 2, 16)
    with pytest.raises(ValueError):
        cp.cp_shard(np.zeros((1, 1), np.int32), [3], 0, 0, 16)


def test_partial_buffer_layout():
    for rows, D in ((1, 64), (6, 128), (8, 64), (33, 128)):
        n = cp.partial_block_floats(rows, D)
        assert n % 4 == 0 and rows * (D + 1) <= n < rows * (D + 1) + 4
    buf = torch.arange(cp.partial_block_floats(2 * 3, 64), dtype=torch.float32)
    o, lse = cp.partial_views(buf, (2,), 3, 64)
    assert o.shape == (2, 3, 64) and lse.shape == (2, 3)
    assert o[1, 2, 63].item() == 6 * 64 - 1 and lse[0, 0].item() == 6 * 64
    assert lse.data_ptr() - buf.data_ptr() == 6 * 64 * 4   # 16-byte aligned lse
    with pytest.raises(ValueError):
        cp.partial_views(buf[:-4], (2,), 3, 64)


def _shard_partials(wl, world):
    """Oracle decode of every rank's keys, without sinks: [R, B, Hq, D], [R, B, Hq]."""
    o_parts, l_parts = [], []
    for r in range(world):
        t_r, l_r = cp.cp_shard(wl.block_table, wl.seq_lens, world, r, wl.block_tokens)
        o, l = oracle.decode(wl.q, wl.k_cache, wl.v_cache, t_r, l_r, k_scale=wl.k_scale,
                             v_scale=wl.v_scale, sm_scale=wl.sm_scale, sinks=None, threads=1)
        o_parts.append(o)
        l_parts.append(l)
    return np.stack(o_parts), np.stack(l_parts)


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("sinks", [False, True])
def test_oracle_merge_of_shards_is_the_decode(world, sinks):
    # lengths from empty to several pages per rank; 5 ranks leave some ranks
    # without a page of the short sequences
    wl = W.make_custom(B=5, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[0, 1, 17, 40, 300],
                       sinks=sinks, seed=11)
    o_parts, l_parts = _shard_partials(wl, world)
    out, lse = oracle.merge(o_parts, l_parts, 8, wl.sinks)
    ref_out, ref_lse = oracle.decode_workload(wl, threads=1)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_oracle_merge_special_cases():
    rng = np.random.default_rng(5)
    o = rng.normal(size=(1, 3, 4, 64))
    lse = rng.normal(size=(1, 3, 4))
    out, l = oracle.merge(o, lse, 4)
    np.testing.assert_array_equal(out, o[0])          # one part, no sink: itself
    np.testing.assert_array_equal(l, lse[0])
    # no key anywhere: 0 and -inf; with a sink: 0 and the sink
    o2 = np.zeros((2, 1, 4, 64))
    l2 = np.full((2, 1, 4), -np.inf)
    out, l = oracle.merge(o2, l2, 4)
    assert (out == 0).all() and np.isneginf(l).all()
    s = np.array([0.5, -1.0, 2.0, 0.0], np.float32)
    out, l = oracle.merge(o2, l2, 4, s)
    assert (out == 0).all()
    np.testing.assert_array_equal(l[0], s.astype(np.float64))
    # two equal parts: the same output, lse up by ln 2
    o3 = np.stack([o[0], o[0]])
    l3 = np.stack([lse[0], lse[0]])
    out, l = oracle.merge(o3, l3, 4)
    np.testing.assert_allclose(out, o[0], rtol=1e-14)
    np.testing.assert_allclose(l, lse[0] + np.log(2.0), rtol=1e-14)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _cp_worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wl = W.make_custom(B=3, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[5, 70, 257],
                           sinks=True, seed=23)
        t_r, l_r = cp.cp_shard(wl.block_table, wl.seq_lens, world, rank, wl.block_tokens)
        o, l = oracle.decode(wl.q, wl.k_cache, wl.v_cache, t_r, l_r, k_scale=wl.k_scale,
                             v_scale=wl.v_scale, sm_scale=wl.sm_scale, sinks=None, threads=1)
        buf = torch.zeros(cp.partial_block_floats(3 * 8, 128), dtype=torch.float32)
        o_view, l_view = cp.partial_views(buf, (3,), 8, 128)
        o_view.copy_(torch.from_numpy(o))
        l_view.copy_(torch.from_numpy(l))
        gathered = cp.cp_exchange(buf)
        assert gathered.shape == (world, buf.numel())
        views = [cp.partial_views(gathered[r], (3,), 8, 128) for r in range(world)]
        o_all = np.stack([v[0].double().numpy() for v in views])
        l_all = np.stack([v[1].double().numpy() for v in views])
        out, lse = oracle.merge(o_all, l_all, 8, wl.sinks)
        ref_out, ref_lse = oracle.decode_workload(wl, threads=1)
        # the partials crossed the exchange as f32
        err_o = float(np.abs(out - ref_out).max())
        err_l = float(np.abs(lse - ref_lse).max())
        dist.barrier()
        q.put((rank, err_o, err_l))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_exchange_and_merge():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, err_o, err_l in res:
        assert err_o < 1e-5 and err_l < 1e-5, (rank, err_o, err_l)


def test_exchange_epochs_alternate_parity_and_skip_zero():
    """The fused exchange alternates its two buffers by the epoch's parity: the
    epoch sequence must never hit 0 (the flags' initial value) and must keep
    alternating across the wrap."""
    ex = cp.CpExchange.__new__(cp.CpExchange)   # host logic only, no buffers
    ex.epoch = 0
    seen = [ex.next_epoch() for _ in range(4)]
    assert seen == [1, 2, 3, 4]
    ex.epoch = 0xFFFFFFFD
    seq = [ex.next_epoch() for _ in range(4)]
    assert seq == [0xFFFFFFFE, 1, 2, 3]
    assert all((a ^ b) & 1 for a, b in zip([0xFFFFFFFD] + seq, seq))


def test_rank_calls_reject_bad_input_before_any_device_work():
    q4 = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        cp.fp8_paged_decode_attention_cp(q4, None, None, None, None, 1.0, 1.0, 0.1)
    ex = cp.CpExchange.__new__(cp.CpExchange)
    ex.epoch, ex.rank = 0, 0
    with pytest.raises(ValueError):
        cp.fp8_paged_decode_attention_cp_fused(q4, None, None, None, None, 1.0, 1.0, 0.1,
                                               exchange=ex)
    q3 = torch.zeros((1, 8, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):   # no epoch started
        cp.fp8_paged_decode_attention_cp_fused(q3, None, None, None, None, 1.0, 1.0, 0.1,
                                               exchange=ex)
