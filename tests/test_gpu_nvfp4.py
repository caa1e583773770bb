"""NVFP4 KV pages on the GPU vs the fp64 oracle: decode parity
(|out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3, element-wise) over both
stage shapes, head dims, several queries, windows and sinks; the NVFP4 cache
write bit-exact against the oracle's writer; write-then-decode."""
import ctypes
import itertools

import numpy as np
import pytest
import torch

import fp8_paged_decode_b200 as fpd
import oracle
from fp8_paged_decode_b200 import workloads as W
from tests.gpu_util import assert_parity

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def dev_inputs(wl):
    return dict(q=torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).cuda(),
                kv=torch.from_numpy(wl.kv_cache).cuda(),
                table=torch.from_numpy(wl.block_table).cuda(),
                lens=torch.from_numpy(wl.seq_lens).cuda(),
                sinks=None if wl.sinks is None else torch.from_numpy(wl.sinks).cuda())


def run_nvfp4(wl, d=None, chunk=0, **kw):
    d = d or dev_inputs(wl)
    out, lse = fpd.fp8_paged_decode_attention_nvfp4(
        d["q"], d["kv"], d["table"], d["lens"], wl.k_scale, wl.v_scale, wl.sm_scale,
        Hkv=wl.Hkv, block_tokens=wl.block_tokens, window_left=wl.window_left, sinks=d["sinks"],
        chunk_pages_override=chunk, **kw)
    torch.cuda.synchronize()
    return out, lse


def check(wl, chunk=0, rows=None, what=""):
    n = wl.B * wl.q_len
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")
    out, lse = run_nvfp4(wl, chunk=chunk, workspace=ws)
    bits = fpd.fp8_paged_decode_check_status(ws)
    assert bits == 0, f"device status {bits:#x} ({what or wl.name}, chunk {chunk})"
    ro, rl = oracle.decode_nvfp4_workload(wl, rows=rows)
    o = out.float().cpu().numpy().astype(np.float64).reshape(n, wl.Hq, wl.D)
    l = lse.cpu().numpy().astype(np.float64).reshape(n, wl.Hq)
    ro = ro.reshape(n, wl.Hq, wl.D)
    rl = rl.reshape(n, wl.Hq)
    if rows is not None:
        rows = np.asarray(rows)
        tok, h = np.divmod(rows, wl.Hq)
        return assert_parity(o[tok, h][None], l[tok, h][None], ro[tok, h][None],
                             rl[tok, h][None], what=what)
    return assert_parity(o, l, ro, rl, what=what or f"{wl.name} chunk {chunk}")


SHAPES = [  # (Hq, Hkv, D, bt): four-head stages (Hkv % 4 == 0) and one-head stages
    (32, 8, 128, 16), (64, 8, 64, 32), (16, 4, 128, 64), (16, 2, 128, 64), (32, 2, 64, 16),
    (8, 1, 128, 32),
]
GRID = list(itertools.product(SHAPES, [1, 3], [-1, 40]))


@pytest.mark.parametrize("shape,Q,window", GRID,
                         ids=[f"h{a}-kv{b}-D{c}-bt{d}-q{q}-w{w}" for (a, b, c, d), q, w in GRID])
def test_decode_parity(shape, Q, window):
    Hq, Hkv, D, bt = shape
    lens = [1, 2, bt - 1, bt, bt + 1, 3 * bt + 5, 700]
    wl = W.make_custom_nvfp4(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                             window_left=window, sinks=True, seed=600 + Hq + D + bt + Q + window,
                             sm_scale=1.0 / np.sqrt(D), q_len=Q)
    check(wl)
    check(wl, chunk=1)        # one page per split: many partials, both stage shapes
    if Hkv % 4 == 0:
        check(wl, chunk=3)


def test_no_sinks_and_empty_sequence():
    wl = W.make_custom_nvfp4(B=4, Hq=16, Hkv=4, D=128, block_tokens=16, seq_lens=[0, 1, 33, 257],
                             sinks=False, seed=611)
    check(wl)
    check(wl, chunk=1)


@pytest.mark.parametrize("name", ["llama3_8b", "long_context", "large_mixed"])
def test_full_workload_every_row(name):
    """Every (sequence, head) row of the full-size workloads over NVFP4 pages
    against the oracle, in the bench's launch configuration (the default plan),
    with the block scales of every slot the decode must not read set to the
    NaN code."""
    check(W.make_workload_nvfp4(name), what=f"{name} NVFP4, every row")


def test_invalid_page_flagged():
    wl = W.make_custom_nvfp4(B=2, Hq=8, Hkv=4, D=128, block_tokens=16, seq_lens=[40, 64], seed=613)
    d = dev_inputs(wl)
    d["table"][1, 2] = wl.num_blocks + 3
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    out, lse = run_nvfp4(wl, d, workspace=ws)
    assert fpd.fp8_paged_decode_check_status(ws) & fpd.FPD_DEVERR_BLOCK_TABLE
    assert torch.isfinite(out.float()).all()
    ro, rl = oracle.decode_nvfp4_workload(wl, rows=list(range(wl.Hq)))
    assert_parity(out[:1].float().cpu().numpy().astype(np.float64),
                  lse[:1].cpu().numpy().astype(np.float64), ro[:1], rl[:1], what="row 0")


def test_descriptor_errors():
    """NVFP4 needs head-major pages and scale pointers; checked before launch."""
    wl = W.make_custom_nvfp4(B=2, Hq=8, Hkv=4, D=128, block_tokens=16, seq_lens=[40, 64], seed=614)
    d = dev_inputs(wl)
    lay = fpd.nvfp4_page_layout(4, 16, 128)
    out = torch.empty((2, 8, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    a = fpd.fpd_decode_args()
    base = d["kv"].data_ptr()
    a.q, a.out = d["q"].data_ptr(), out.data_ptr()
    a.k_cache, a.v_cache = base + lay["k_data"], base + lay["v_data"]
    a.k_scales, a.v_scales = base + lay["k_sf"], base + lay["v_sf"]
    a.kv_page_stride = a.sf_page_stride = lay["page_bytes"]
    a.kv_format = fpd.FPD_KV_NVFP4
    a.kv_layout = fpd.FPD_KV_HND
    a.block_table, a.seq_lens = d["table"].data_ptr(), d["lens"].data_ptr()
    a.B, a.q_len, a.Hq, a.Hkv, a.D = 2, 1, 8, 4, 128
    a.num_blocks, a.block_tokens, a.max_blocks = wl.num_blocks, 16, wl.max_blocks
    a.k_scale, a.v_scale, a.sm_scale, a.window_left = wl.k_scale, wl.v_scale, 0.1, -1
    f = fpd.load_library().fp8_paged_decode_attention_args
    vp = ctypes.c_void_p
    assert f(ctypes.byref(a), vp(ws.data_ptr()), ws.numel(), None) == fpd.FPD_OK
    torch.cuda.synchronize()
    a.kv_layout = fpd.FPD_KV_NHD
    assert f(ctypes.byref(a), vp(ws.data_ptr()), ws.numel(), None) == fpd.FPD_ERR_UNSUPPORTED
    a.kv_layout = fpd.FPD_KV_HND
    a.k_scales = None
    assert f(ctypes.byref(a), vp(ws.data_ptr()), ws.numel(), None) == fpd.FPD_ERR_INVALID_ARG
    a.k_scales = base + lay["k_sf"]
    a.kv_page_stride = lay["page_bytes"] + 8      # not a multiple of 16
    assert f(ctypes.byref(a), vp(ws.data_ptr()), ws.numel(), None) == fpd.FPD_ERR_INVALID_ARG


def test_fp16_query_device_scales():
    wl = W.make_custom_nvfp4(B=3, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[5, 300, 1000],
                             sinks=True, seed=615, q_len=2)
    rng = np.random.default_rng(616)
    q16 = (rng.standard_normal(wl.q.shape) * 2).astype(np.float16)
    d = dev_inputs(wl)
    d["q"] = torch.from_numpy(q16.view(np.int16)).view(torch.float16).cuda()
    ks = torch.tensor([wl.k_scale], dtype=torch.float32, device="cuda")
    vs = torch.tensor([wl.v_scale], dtype=torch.float32, device="cuda")
    out, lse = fpd.fp8_paged_decode_attention_nvfp4(d["q"], d["kv"], d["table"], d["lens"], ks, vs,
                                                    wl.sm_scale, Hkv=8, block_tokens=16,
                                                    sinks=d["sinks"])
    torch.cuda.synchronize()
    ro, rl = oracle.decode_nvfp4(q16.view(np.uint16), wl.kv_cache, wl.block_table, wl.seq_lens,
                                 Hkv=8, block_tokens=16, k_scale=wl.k_scale, v_scale=wl.v_scale,
                                 sm_scale=wl.sm_scale, sinks=wl.sinks, q_dtype="f16")
    n = wl.B * 2
    assert_parity(out.float().cpu().numpy().astype(np.float64).reshape(n, 32, 128),
                  lse.cpu().numpy().astype(np.float64).reshape(n, 32), ro.reshape(n, 32, 128),
                  rl.reshape(n, 32), what="NVFP4 fp16 q, device scales")


def bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("Hkv,D,bt,T", [(2, 64, 16, 37), (8, 128, 16, 300), (4, 128, 64, 129),
                                        (1, 64, 32, 70)])
def test_cache_write_bit_exact(Hkv, D, bt, T):
    rng = np.random.default_rng(620 + Hkv + D + bt + T)
    x = rng.standard_normal((2, T, Hkv, D)).astype(np.float32) * 2
    x[:, ::5, :, :16] *= 1e-4          # small blocks
    x[:, 1::7, :, 16:32] *= 300        # large blocks (scales near the E4M3 top)
    x[:, 2, :, :16] = 0.0              # all-zero block
    kb, vb = bf16_bits(x[0]), bf16_bits(x[1])
    nb = T // bt + 3
    lay = fpd.nvfp4_page_layout(Hkv, bt, D)
    pages0 = rng.integers(0, 256, (nb, lay["page_bytes"]), dtype=np.uint8)
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    slots[::6] = -1
    for ks, vs in ((0.05, 0.02), (1.0, 1.0), (0.003, 0.7)):
        pg = torch.from_numpy(pages0.copy()).cuda()
        fpd.fp8_paged_decode_cache_write_nvfp4(
            torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda(),
            torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).cuda(),
            torch.from_numpy(slots).cuda(), pg, ks, vs, block_tokens=bt)
        torch.cuda.synchronize()
        want = pages0.copy()
        assert oracle.cache_write_nvfp4(kb, vb, slots, want, block_tokens=bt, k_scale=ks,
                                        v_scale=vs) == 0
        got = pg.cpu().numpy()
        diff = np.flatnonzero(got != want)
        assert diff.size == 0, (f"scales {ks},{vs}: {diff.size} bytes differ, first at "
                                f"{np.unravel_index(diff[0], got.shape)}: {got.reshape(-1)[diff[0]]:#x} "
                                f"vs {want.reshape(-1)[diff[0]]:#x}")


def test_cache_write_out_of_range_slot():
    Hkv, D, bt, T, nb = 2, 64, 16, 10, 2
    lay = fpd.nvfp4_page_layout(Hkv, bt, D)
    pg = torch.zeros((nb, lay["page_bytes"]), dtype=torch.uint8, device="cuda")
    key = torch.randn(T, Hkv, D, device="cuda").to(torch.bfloat16)
    slots = torch.arange(T, dtype=torch.int64, device="cuda")
    slots[3] = nb * bt
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    fpd.fp8_paged_decode_cache_write_nvfp4(key, key, slots, pg, 0.1, 0.1, block_tokens=bt,
                                           status=status)
    torch.cuda.synchronize()
    assert int(status[0].item()) & fpd.FPD_DEVERR_SLOT


def test_write_then_decode():
    """The GPU writer fills NVFP4 pages from bf16 K/V; decoding them on the GPU
    matches the oracle on the pages the oracle's writer fills (identical bytes)."""
    rng = np.random.default_rng(630)
    B, Hq, Hkv, D, bt = 3, 32, 8, 128, 16
    lens = [300, 17, 1000]
    wl = W.make_custom_nvfp4(B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens,
                             sinks=True, seed=631, sm_scale=0.08)
    slots = np.concatenate([wl.block_table[b, np.arange(L) // bt].astype(np.int64) * bt
                            + np.arange(L) % bt for b, L in enumerate(lens)])
    T = slots.size
    kb = bf16_bits(rng.standard_normal((T, Hkv, D)) * 2)
    vb = bf16_bits(rng.standard_normal((T, Hkv, D)))
    ks, vs = 2.0 / 448 / 6 * 2, 1.0 / 448 / 6 * 3
    pg = torch.from_numpy(wl.kv_cache.copy()).cuda()
    fpd.fp8_paged_decode_cache_write_nvfp4(
        torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).cuda(),
        torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).cuda(),
        torch.from_numpy(slots).cuda(), pg, ks, vs, block_tokens=bt)
    torch.cuda.synchronize()
    want = wl.kv_cache.copy()
    oracle.cache_write_nvfp4(kb, vb, slots, want, block_tokens=bt, k_scale=ks, v_scale=vs)
    assert np.array_equal(pg.cpu().numpy(), want)
    wl.kv_cache, wl.k_scale, wl.v_scale = want, float(np.float32(ks)), float(np.float32(vs))
    check(wl, what="write then decode")


def test_graph_capture_device_scales_no_allocation():
    """NVFP4 decode captured in a CUDA graph with device scales: nothing is
    allocated during capture, and replays after new scale values use them."""
    wl = W.make_custom_nvfp4(B=4, Hq=32, Hkv=8, D=128, block_tokens=16,
                             seq_lens=[2000, 10, 700, 4000], sinks=True, seed=640)
    d = dev_inputs(wl)
    ks = torch.tensor([wl.k_scale], dtype=torch.float32, device="cuda")
    vs = torch.tensor([wl.v_scale], dtype=torch.float32, device="cuda")
    out = torch.empty((4, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((4, 32), dtype=torch.float32, device="cuda")
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")

    def call():
        fpd.fp8_paged_decode_attention_nvfp4(d["q"], d["kv"], d["table"], d["lens"], ks, vs,
                                             wl.sm_scale, Hkv=8, block_tokens=16,
                                             sinks=d["sinks"], out=out, lse=lse, workspace=ws)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        before = torch.cuda.memory_allocated()
        call()
        after = torch.cuda.memory_allocated()
    assert after == before
    for kx, vx in ((wl.k_scale, wl.v_scale), (wl.k_scale * 1.5, wl.v_scale * 0.5)):
        ks.fill_(kx)
        vs.fill_(vx)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        ro, rl = oracle.decode_nvfp4(wl.q, wl.kv_cache, wl.block_table, wl.seq_lens, Hkv=8,
                                     block_tokens=16, k_scale=np.float32(kx),
                                     v_scale=np.float32(vx), sm_scale=wl.sm_scale,
                                     sinks=wl.sinks)
        assert_parity(out.float().cpu().numpy().astype(np.float64),
                      lse.cpu().numpy().astype(np.float64), ro, rl, what=f"replay {kx}, {vx}")


def test_page_permutation_bitwise_and_repeat():
    """Moving pages to other physical slots (and the table with them) changes no
    bit of the result; two identical calls give identical bits."""
    wl = W.make_custom_nvfp4(B=5, Hq=16, Hkv=4, D=128, block_tokens=32,
                             seq_lens=[33, 500, 1, 1024, 77], sinks=True, seed=641)
    out1, lse1 = run_nvfp4(wl, chunk=2)
    out1b, lse1b = run_nvfp4(wl, chunk=2)
    assert torch.equal(out1, out1b) and torch.equal(lse1, lse1b)
    perm = np.random.default_rng(642).permutation(wl.num_blocks)
    inv = np.argsort(perm)
    wl2 = W.make_custom_nvfp4(B=5, Hq=16, Hkv=4, D=128, block_tokens=32,
                              seq_lens=[33, 500, 1, 1024, 77], sinks=True, seed=641)
    wl2.kv_cache = np.ascontiguousarray(wl.kv_cache[inv])       # page p moves to slot perm[p]
    table = wl.block_table.copy()
    table[table >= 0] = perm[table[table >= 0]]
    wl2.block_table = table
    out2, lse2 = run_nvfp4(wl2, chunk=2)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_cache_write_strided_key_value():
    """key and value as slices of a fused [T, (Hq + 2 Hkv) * D] projection."""
    rng = np.random.default_rng(643)
    T, Hq, Hkv, D, bt = 50, 16, 4, 128, 16
    fused = torch.from_numpy(rng.standard_normal((T, (Hq + 2 * Hkv) * D)).astype(np.float32)) \
        .to(torch.bfloat16).cuda()
    key = fused[:, Hq * D:(Hq + Hkv) * D].view(T, Hkv, D)
    value = fused[:, (Hq + Hkv) * D:].view(T, Hkv, D)
    nb = T // bt + 2
    lay = fpd.nvfp4_page_layout(Hkv, bt, D)
    pg = torch.zeros((nb, lay["page_bytes"]), dtype=torch.uint8, device="cuda")
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    fpd.fp8_paged_decode_cache_write_nvfp4(key, value, torch.from_numpy(slots).cuda(), pg, 0.05,
                                           0.02, block_tokens=bt)
    torch.cuda.synchronize()
    kb = fused.cpu().view(torch.int16).numpy().view(np.uint16)
    want = np.zeros((nb, lay["page_bytes"]), dtype=np.uint8)
    oracle.cache_write_nvfp4(np.ascontiguousarray(kb[:, Hq * D:(Hq + Hkv) * D]).reshape(T, Hkv, D),
                             np.ascontiguousarray(kb[:, (Hq + Hkv) * D:]).reshape(T, Hkv, D),
                             slots, want, block_tokens=bt, k_scale=0.05, v_scale=0.02)
    assert np.array_equal(pg.cpu().numpy(), want)
