"""Context-parallel decode on the GPU vs the fp64 oracle.

* The f32 output mode (each rank's partial): every row finished by the
  combine, with one split or several, E4M3 and NVFP4 pages, several queries.
* The merge kernel on random partials (ranks without a key, rows no rank and
  no sink covers, more than 32 ranks) vs the oracle's merge.
* R ranks emulated on one GPU: R independent partial decodes over
  ``cp_shard``'s parts (separate launches that never wait on one another),
  then the merge, vs the oracle over all keys.
* The whole rank-side call through a one-rank NCCL process group.
Tolerances as everywhere: |out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3."""
import datetime
import socket

import numpy as np
import pytest
import torch

import fp8_paged_decode_b200 as fpd
import oracle
from fp8_paged_decode_b200 import cp
from fp8_paged_decode_b200 import workloads as W
from tests.gpu_util import assert_parity, to_device

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _flat(o, l, Hq, D):
    return (np.asarray(o, np.float64).reshape(-1, Hq, D), np.asarray(l, np.float64).reshape(-1, Hq))


def _decode_f32(wl, dev, table=None, lens=None, sinks="keep", chunk_pages=0, out=None, lse=None):
    t = dev["block_table"] if table is None else table
    s = dev["seq_lens"] if lens is None else lens
    return fpd.fp8_paged_decode_attention(
        dev["q"], dev["k_cache"], dev["v_cache"], t, s, wl.k_scale, wl.v_scale, wl.sm_scale,
        window_left=wl.window_left, sinks=dev["sinks"] if sinks == "keep" else sinks,
        chunk_pages_override=chunk_pages, out=out, lse=lse, out_dtype="f32")


F32_CASES = [  # (Hq, Hkv, D, bt, lens, window, sinks, q_len, chunk_pages)
    (8, 2, 128, 16, [37, 300], -1, False, 1, 0),           # one split each (tiny-shaped)
    (32, 8, 128, 16, [0, 1, 17, 2000, 5000], -1, True, 1, 0),   # split sequences, an empty one
    (64, 8, 64, 16, [100, 3000], 128, True, 1, 0),         # window, sinks, D = 64
    (16, 2, 128, 64, [129, 64, 5], -1, False, 1, 1),       # one head per stage, forced splits
    (32, 8, 128, 16, [40, 700], -1, True, 3, 0),           # several queries per sequence
    (16, 2, 64, 32, [9, 1000], 20, False, 4, 2),
]


@pytest.mark.parametrize("case", range(len(F32_CASES)))
def test_f32_output_parity(case):
    Hq, Hkv, D, bt, lens, window, sinks, Q, cpg = F32_CASES[case]
    wl = W.make_custom(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                       window_left=window, sinks=sinks, seed=100 + case, q_len=Q)
    dev = to_device(wl)
    out, lse = _decode_f32(wl, dev, chunk_pages=cpg)
    torch.cuda.synchronize()
    assert out.dtype == torch.float32
    ro, rl = oracle.decode_workload(wl)
    o, l = _flat(out.cpu().numpy(), lse.cpu().numpy(), Hq, D)
    assert_parity(o, l, *_flat(ro, rl, Hq, D), what=f"f32 case {case}")
    # the bf16 call on the same inputs agrees to bf16 rounding
    ob, lb = fpd.fp8_paged_decode_attention(
        dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
        wl.k_scale, wl.v_scale, wl.sm_scale, window_left=window, sinks=dev["sinks"],
        chunk_pages_override=cpg)
    torch.cuda.synchronize()
    np.testing.assert_allclose(ob.float().cpu().numpy(), out.cpu().numpy(), rtol=2 ** -7,
                               atol=1e-6)
    np.testing.assert_allclose(lb.cpu().numpy(), lse.cpu().numpy(), rtol=0, atol=1e-5)


def test_f32_output_nvfp4():
    wl = W.make_custom_nvfp4(B=3, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[1, 300, 4000],
                             sinks=True, seed=7)
    q = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).cuda()
    pages = torch.from_numpy(wl.kv_cache).cuda()
    out, lse = fpd.fp8_paged_decode_attention_nvfp4(
        q, pages, torch.from_numpy(wl.block_table).cuda(), torch.from_numpy(wl.seq_lens).cuda(),
        wl.k_scale, wl.v_scale, wl.sm_scale, Hkv=8, block_tokens=16,
        sinks=torch.from_numpy(wl.sinks).cuda(), out_dtype="f32")
    torch.cuda.synchronize()
    ro, rl = oracle.decode_nvfp4_workload(wl)
    assert_parity(*_flat(out.cpu().numpy(), lse.cpu().numpy(), 32, 128), *_flat(ro, rl, 32, 128),
                  what="nvfp4 f32")


def test_f32_workspace_holds_a_partial_per_row():
    wl = W.make_custom(B=2, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[37, 300], seed=1)
    dev = to_device(wl)
    a = fpd.fpd_decode_args()
    a.B, a.q_len, a.Hq, a.Hkv, a.D = 2, 1, 8, 2, 128
    a.num_blocks, a.block_tokens, a.max_blocks = wl.num_blocks, 16, wl.max_blocks
    a.window_left = -1
    bf16_need = fpd.fp8_paged_decode_workspace_bytes_args(a)
    a.out_dtype = fpd.FPD_OUT_F32
    f32_need = fpd.fp8_paged_decode_workspace_bytes_args(a)
    assert bf16_need == 256                                   # one split: no partials
    assert f32_need >= 256 + 2 * 8 * (128 + 1) * 4
    a.out_dtype = 7
    assert fpd.fp8_paged_decode_workspace_bytes_args(a) == 0  # unknown output type
    ws = torch.zeros(bf16_need, dtype=torch.uint8, device="cuda")
    with pytest.raises(fpd.FpdError) as e:
        fpd.fp8_paged_decode_attention(
            dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
            wl.k_scale, wl.v_scale, wl.sm_scale, out_dtype="f32", workspace=ws)
    assert e.value.status == fpd.FPD_ERR_WORKSPACE_TOO_SMALL


def _random_partials(R, rows, D, seed, dead=0.2):
    rng = np.random.default_rng(seed)
    o = rng.normal(size=(R, rows, D)) * 2.0
    l = rng.normal(size=(R, rows)) * 3.0
    l[rng.random((R, rows)) < dead] = -np.inf
    o[np.isneginf(l)] = 0.0
    return o.astype(np.float32), l.astype(np.float32)


@pytest.mark.parametrize("R,D,B,Hq,sinks", [(1, 128, 3, 8, False), (3, 64, 5, 16, True),
                                            (8, 128, 4, 32, True), (40, 128, 2, 4, False),
                                            (33, 64, 3, 2, True)])
def test_merge_kernel_vs_oracle(R, D, B, Hq, sinks):
    rows = B * Hq
    o, l = _random_partials(R, rows, D, seed=R * 7 + D)
    l[:, 0] = -np.inf                     # a row no rank covers
    o[:, 0] = 0.0
    block = cp.partial_block_floats(rows, D)
    buf = np.zeros((R, block), np.float32)
    buf[:, : rows * D] = o.reshape(R, -1)
    buf[:, rows * D: rows * D + rows] = l
    s = np.random.default_rng(1).normal(size=Hq).astype(np.float32) if sinks else None
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    fpd.fp8_paged_decode_cp_merge(torch.from_numpy(buf).cuda(), out, lse,
                                  None if s is None else torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    ro, rl = oracle.merge(o.reshape(R, B, Hq, D).astype(np.float64),
                          l.reshape(R, B, Hq).astype(np.float64), Hq, s)
    assert_parity(*_flat(out.float().cpu().numpy(), lse.cpu().numpy(), Hq, D),
                  *_flat(ro, rl, Hq, D), what=f"merge R={R}")
    if not sinks:   # row 0: no key and no sink
        assert (out[0, 0] == 0).all() and torch.isneginf(lse[0, 0])


def test_merge_rejects_bad_arguments():
    buf = torch.zeros((2, cp.partial_block_floats(8, 128)), dtype=torch.float32, device="cuda")
    out = torch.empty((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fpd.FpdError) as e:
        fpd.fp8_paged_decode_cp_merge(buf[:, :-1].contiguous(), out)   # block not a multiple of 4
    assert e.value.status == fpd.FPD_ERR_INVALID_ARG
    with pytest.raises(fpd.FpdError) as e:
        fpd.fp8_paged_decode_cp_merge(buf[:, : 8 * 128].contiguous(), out)   # no room for lse
    assert e.value.status == fpd.FPD_ERR_INVALID_ARG
    out96 = torch.empty((1, 8, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fpd.FpdError) as e:
        fpd.fp8_paged_decode_cp_merge(buf, out96)
    assert e.value.status == fpd.FPD_ERR_UNSUPPORTED


CP_CASES = [  # (Hq, Hkv, D, bt, lens, sinks, ranks)
    (8, 2, 128, 16, [37, 300], False, 2),
    (8, 2, 128, 16, [37, 300], True, 3),
    (32, 8, 128, 16, [1, 20, 1500, 6000], True, 4),
    (32, 8, 128, 64, [9000, 130, 64], False, 8),          # long and short: empty ranks
    (64, 8, 64, 16, [5000, 33], True, 8),
    (16, 2, 128, 32, [2, 700, 3001], True, 5),
]


@pytest.mark.parametrize("case", range(len(CP_CASES)))
def test_emulated_ranks_vs_oracle(case):
    Hq, Hkv, D, bt, lens, sinks, R = CP_CASES[case]
    B = len(lens)
    wl = W.make_custom(B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens, sinks=sinks,
                       seed=300 + case)
    dev = to_device(wl)
    rows = B * Hq
    gathered = torch.full((R, cp.partial_block_floats(rows, D)), float("nan"),
                          dtype=torch.float32, device="cuda")
    for r in range(R):
        t_r, l_r = cp.cp_shard(wl.block_table, wl.seq_lens, R, r, bt)
        o_v, l_v = cp.partial_views(gathered[r], (B,), Hq, D)
        _decode_f32(wl, dev, table=torch.from_numpy(t_r).cuda(), lens=torch.from_numpy(l_r).cuda(),
                    sinks=None, out=o_v, lse=l_v)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    fpd.fp8_paged_decode_cp_merge(gathered, out, lse, dev["sinks"])
    torch.cuda.synchronize()
    ro, rl = oracle.decode_workload(wl)
    assert_parity(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                  ro, rl, what=f"cp case {case}, {R} ranks")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_rank_call_through_nccl():
    import torch.distributed as dist
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[3, 800, 2500, 4096],
                       sinks=True, seed=41)
    dev = to_device(wl)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        out, lse = cp.fp8_paged_decode_attention_cp(
            dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
            wl.k_scale, wl.v_scale, wl.sm_scale, sinks=dev["sinks"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ro, rl = oracle.decode_workload(wl)
    assert_parity(out.float().cpu().numpy().astype(np.float64),
                  lse.cpu().numpy().astype(np.float64), ro, rl, what="one-rank NCCL call")


def test_rank_call_rejects_several_queries():
    q = torch.zeros((1, 2, 8, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        cp.fp8_paged_decode_attention_cp(q, None, None, None, None, 1.0, 1.0, 0.1)


# ---------------------------------------------------------- fused exchange --

def _fused_step(wl, dev, ex, R, ranks_publishing=None):
    """One step of R ranks on one GPU: every rank's publishing decode (one after
    another), then every rank's waiting merge.  Returns the R (out, lse)."""
    ex.next_epoch()
    for r in (range(R) if ranks_publishing is None else ranks_publishing):
        t_r, l_r = cp.cp_shard(wl.block_table, wl.seq_lens, R, r, wl.block_tokens)
        cp.fp8_paged_decode_attention_cp_fused(
            dev["q"], dev["k_cache"], dev["v_cache"], torch.from_numpy(t_r).cuda(),
            torch.from_numpy(l_r).cuda(), wl.k_scale, wl.v_scale, wl.sm_scale, exchange=ex,
            rank=r, merge=False)
    return [cp.fp8_paged_decode_attention_cp_fused(
                dev["q"], None, None, None, None, wl.k_scale, wl.v_scale, wl.sm_scale,
                exchange=ex, rank=r, sinks=dev["sinks"], publish=False)
            for r in range(R)]


@pytest.mark.parametrize("case", [0, 2, 3, 5])
def test_fused_exchange_vs_oracle(case):
    """Each rank's combine kernel stores its rows into every rank's gather
    buffer and raises its flag there; each rank's merge waits for the flags.
    All ranks agree bitwise, with each other and with the unfused path."""
    Hq, Hkv, D, bt, lens, sinks, R = CP_CASES[case]
    B = len(lens)
    wl = W.make_custom(B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens, sinks=sinks,
                       seed=300 + case)
    dev = to_device(wl)
    ex = cp.CpExchange.local(R, B, Hq, D)
    try:
        res = _fused_step(wl, dev, ex, R)
        torch.cuda.synchronize()
        flags = ex.flags(0).cpu()
        assert (flags == ex.epoch).all()
        # the unfused path: f32 partials, then the merge of the gathered rows
        gathered = torch.zeros((R, cp.partial_block_floats(B * Hq, D)), dtype=torch.float32,
                               device="cuda")
        for r in range(R):
            t_r, l_r = cp.cp_shard(wl.block_table, wl.seq_lens, R, r, bt)
            o_v, l_v = cp.partial_views(gathered[r], (B,), Hq, D)
            _decode_f32(wl, dev, table=torch.from_numpy(t_r).cuda(),
                        lens=torch.from_numpy(l_r).cuda(), sinks=None, out=o_v, lse=l_v)
        ref = fpd.fp8_paged_decode_cp_merge(gathered, torch.empty_like(res[0][0]),
                                            torch.empty_like(res[0][1]), dev["sinks"])
        torch.cuda.synchronize()
        for o, l in res:
            assert torch.equal(o, ref[0]) and torch.equal(l, ref[1])
        ro, rl = oracle.decode_workload(wl)
        assert_parity(res[0][0].float().cpu().numpy().astype(np.float64),
                      res[0][1].cpu().numpy().astype(np.float64), ro, rl,
                      what=f"fused exchange, case {case}, {R} ranks")
    finally:
        ex.close()


def test_fused_exchange_consecutive_steps():
    """The flags keep the last epoch and the finished-CTA counter resets itself:
    a second step with another query is right too."""
    wl = W.make_custom(B=3, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[40, 3000, 7000],
                       sinks=True, seed=51)
    dev = to_device(wl)
    ex = cp.CpExchange.local(4, 3, 32, 128)
    try:
        ws = None
        for step in range(3):
            wl.q = W.make_custom(B=3, Hq=32, Hkv=8, D=128, block_tokens=16,
                                 seq_lens=[40, 3000, 7000], seed=60 + step).q
            dev["q"] = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).cuda()
            out, lse = _fused_step(wl, dev, ex, 4)[2]
            torch.cuda.synchronize()
            ro, rl = oracle.decode_workload(wl)
            assert_parity(out.float().cpu().numpy().astype(np.float64),
                          lse.cpu().numpy().astype(np.float64), ro, rl, what=f"step {step}")
        assert ex.epoch == 3
    finally:
        ex.close()


def test_fused_exchange_missing_rank_times_out():
    """A rank whose flag never arrives: the merge's bounded wait gives up,
    records FPD_DEVERR_TIMEOUT and writes nothing; the GPU stays usable."""
    wl = W.make_custom(B=2, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[100, 300], seed=71)
    dev = to_device(wl)
    ex = cp.CpExchange.local(2, 2, 8, 128)
    try:
        ex.next_epoch()
        t_r, l_r = cp.cp_shard(wl.block_table, wl.seq_lens, 2, 0, 16)
        cp.fp8_paged_decode_attention_cp_fused(
            dev["q"], dev["k_cache"], dev["v_cache"], torch.from_numpy(t_r).cuda(),
            torch.from_numpy(l_r).cuda(), wl.k_scale, wl.v_scale, wl.sm_scale, exchange=ex,
            rank=0, merge=False)   # rank 1 never publishes
        out = torch.full((2, 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        cp.fp8_paged_decode_attention_cp_fused(
            dev["q"], None, None, None, None, wl.k_scale, wl.v_scale, wl.sm_scale, exchange=ex,
            rank=0, publish=False, out=out, timeout_ns=2_000_000, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) & fpd.FPD_DEVERR_TIMEOUT
        assert (out == 7.0).all()
        # the context is fine: an ordinary call still works
        o, l = fpd.fp8_paged_decode_attention(dev["q"], dev["k_cache"], dev["v_cache"],
                                              dev["block_table"], dev["seq_lens"], wl.k_scale,
                                              wl.v_scale, wl.sm_scale)
        torch.cuda.synchronize()
        ro, rl = oracle.decode_workload(wl)
        assert_parity(o.float().cpu().numpy().astype(np.float64),
                      l.cpu().numpy().astype(np.float64), ro, rl, what="after the timeout")
    finally:
        ex.close()


def test_fused_exchange_rejects_bad_descriptors():
    wl = W.make_custom(B=2, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[100, 300], seed=72)
    dev = to_device(wl)
    ex = cp.CpExchange.local(2, 2, 8, 128)
    try:
        ex.next_epoch()
        g, f, R, _, e, blk = ex.publish_fields(0)
        for fields in ((g, f, R, 2, e, blk),          # rank out of range
                       (g, f, R, 0, 0, blk),          # epoch 0
                       (g, f, R, 0, e, blk - 4),      # slot too small
                       (0, f, R, 0, e, blk)):         # no gather pointers
            with pytest.raises(fpd.FpdError) as err:
                fpd.fp8_paged_decode_attention(dev["q"], dev["k_cache"], dev["v_cache"],
                                               dev["block_table"], dev["seq_lens"], wl.k_scale,
                                               wl.v_scale, wl.sm_scale, cp_publish=fields)
            assert err.value.status == fpd.FPD_ERR_INVALID_ARG
    finally:
        ex.close()


def test_fused_exchange_through_a_process_group():
    """The distributed constructor (IPC handles gathered over the group) with
    one rank, and the fused call through it."""
    import torch.distributed as dist
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[3, 800, 2500, 4096],
                       sinks=True, seed=43)
    dev = to_device(wl)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("gloo", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ex = cp.CpExchange(4, 32, 128)
        try:
            ex.next_epoch()
            out, lse = cp.fp8_paged_decode_attention_cp_fused(
                dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
                wl.k_scale, wl.v_scale, wl.sm_scale, exchange=ex, sinks=dev["sinks"])
            torch.cuda.synchronize()
        finally:
            ex.close()
    finally:
        dist.destroy_process_group()
    ro, rl = oracle.decode_workload(wl)
    assert_parity(out.float().cpu().numpy().astype(np.float64),
                  lse.cpu().numpy().astype(np.float64), ro, rl, what="one-rank exchange")
