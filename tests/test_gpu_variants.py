"""Interface variants on the GPU vs the fp64 oracle: fp16 queries, head-major
(HND) pages, strided q/out (slices of wider buffers), scales in device memory
(and a CUDA graph replayed with new scales), and all of them together.
Tolerances as everywhere: |out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3."""
import itertools

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


def to_hnd(cache: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(cache.transpose(0, 2, 1, 3))


def f16_query(wl, seed):
    """fp16 bit patterns of wl.q's shape: normal values with some tiny ones."""
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal(wl.q.shape) * 2.0).astype(np.float16)
    q.reshape(-1)[::5] *= np.float16(1e-3)
    return q.view(np.uint16)


def flat(o, lse, wl):
    n = wl.B * wl.q_len
    return (o.reshape(n, wl.Hq, wl.D).astype(np.float64), lse.reshape(n, wl.Hq).astype(np.float64))


def compare(wl, out, lse, ref_out, ref_lse, what):
    o, l = flat(out.float().cpu().numpy(), lse.cpu().numpy(), wl)
    ro, rl = flat(ref_out, ref_lse, wl)
    return assert_parity(o, l, ro, rl, what=what)


def ref(wl, q=None, q_dtype="bf16", k_scale=None, v_scale=None):
    return oracle.decode(wl.q if q is None else q, wl.k_cache, wl.v_cache, wl.block_table,
                         wl.seq_lens, k_scale=wl.k_scale if k_scale is None else k_scale,
                         v_scale=wl.v_scale if v_scale is None else v_scale,
                         sm_scale=wl.sm_scale, window_left=wl.window_left, sinks=wl.sinks,
                         q_dtype=q_dtype)


SHAPES = [  # (Hq, Hkv, D, bt, q_len): four-head and one-head stages, one and two n-tiles
    (32, 8, 128, 16, 1), (64, 8, 64, 32, 1), (16, 2, 128, 64, 1), (32, 2, 64, 16, 1),
    (32, 8, 128, 16, 3), (16, 2, 64, 32, 4),
]
LENS = [1, 15, 16, 17, 300, 1000]


def shape_wl(Hq, Hkv, D, bt, Q, seed, window=-1):
    return W.make_custom(B=len(LENS), Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=LENS,
                         sinks=True, window_left=window, seed=seed, sm_scale=1.0 / np.sqrt(D),
                         q_len=Q)


@pytest.mark.parametrize("shape", SHAPES, ids=[f"h{a}-kv{b}-D{c}-bt{d}-q{e}" for a, b, c, d, e in SHAPES])
def test_fp16_query(shape):
    Hq, Hkv, D, bt, Q = shape
    wl = shape_wl(Hq, Hkv, D, bt, Q, seed=800 + Hq + D + bt + Q)
    q16 = f16_query(wl, 1)
    dev = to_device(wl)
    qd = torch.from_numpy(q16.view(np.int16)).view(torch.float16).cuda()
    for chunk in (0, 2):
        out, lse = fpd.fp8_paged_decode_attention(qd, dev["k_cache"], dev["v_cache"],
                                                  dev["block_table"], dev["seq_lens"], wl.k_scale,
                                                  wl.v_scale, wl.sm_scale, sinks=dev["sinks"],
                                                  chunk_pages_override=chunk)
        torch.cuda.synchronize()
        ro, rl = ref(wl, q=q16, q_dtype="f16")
        compare(wl, out, lse, ro, rl, f"fp16 q {shape} chunk {chunk}")


@pytest.mark.parametrize("shape,window", list(itertools.product(SHAPES, [-1, 20])),
                         ids=[f"h{a}-kv{b}-D{c}-bt{d}-q{e}-w{w}"
                              for (a, b, c, d, e), w in itertools.product(SHAPES, [-1, 20])])
def test_hnd_pages(shape, window):
    Hq, Hkv, D, bt, Q = shape
    wl = shape_wl(Hq, Hkv, D, bt, Q, seed=900 + Hq + D + bt + Q, window=window)
    dev = to_device(wl)
    kh = torch.from_numpy(to_hnd(wl.k_cache)).cuda()
    vh = torch.from_numpy(to_hnd(wl.v_cache)).cuda()
    ro, rl = ref(wl)
    oracle_hnd = oracle.decode(wl.q, to_hnd(wl.k_cache), to_hnd(wl.v_cache), wl.block_table,
                               wl.seq_lens, k_scale=wl.k_scale, v_scale=wl.v_scale,
                               sm_scale=wl.sm_scale, window_left=wl.window_left, sinks=wl.sinks,
                               kv_layout="HND")
    assert np.array_equal(ro, oracle_hnd[0]) and np.array_equal(rl, oracle_hnd[1])
    for chunk in (0, 1):
        out, lse = fpd.fp8_paged_decode_attention(dev["q"], kh, vh, dev["block_table"],
                                                  dev["seq_lens"], wl.k_scale, wl.v_scale,
                                                  wl.sm_scale, window_left=window,
                                                  sinks=dev["sinks"], chunk_pages_override=chunk,
                                                  kv_layout="HND")
        torch.cuda.synchronize()
        compare(wl, out, lse, ro, rl, f"HND {shape} window {window} chunk {chunk}")
        # the same call on token-major pages gives the same bits
        o2, l2 = fpd.fp8_paged_decode_attention(dev["q"], dev["k_cache"], dev["v_cache"],
                                                dev["block_table"], dev["seq_lens"], wl.k_scale,
                                                wl.v_scale, wl.sm_scale, window_left=window,
                                                sinks=dev["sinks"], chunk_pages_override=chunk)
        torch.cuda.synchronize()
        assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_hnd_invalid_page_reads_zeros():
    """A block-table entry past the pool is flagged and read as zeros in HND too."""
    wl = W.make_custom(B=2, Hq=8, Hkv=4, D=128, block_tokens=16, seq_lens=[40, 64], seed=91)
    dev = to_device(wl)
    kh = torch.from_numpy(to_hnd(wl.k_cache)).cuda()
    vh = torch.from_numpy(to_hnd(wl.v_cache)).cuda()
    bad = dev["block_table"].clone()
    bad[1, 2] = wl.num_blocks + 5
    ws = torch.zeros(fpd.fp8_paged_decode_workspace_bytes(2, 8, 4, 128, 16, wl.max_blocks) + 256,
                     dtype=torch.uint8, device="cuda")
    out, lse = fpd.fp8_paged_decode_attention(dev["q"], kh, vh, bad, dev["seq_lens"], wl.k_scale,
                                              wl.v_scale, wl.sm_scale, workspace=ws,
                                              kv_layout="HND")
    assert fpd.fp8_paged_decode_check_status(ws) & fpd.FPD_DEVERR_BLOCK_TABLE
    assert torch.isfinite(out.float()).all()
    # sequence 0 is untouched by the bad entry
    ro, rl = ref(wl)
    assert_parity(out[:1].float().cpu().numpy().astype(np.float64),
                  lse[:1].cpu().numpy().astype(np.float64), ro[:1], rl[:1], what="HND row 0")


@pytest.mark.parametrize("Q", [1, 3])
def test_strided_q_and_out(Q):
    """q a slice of a fused QKV buffer, out a slice of a wider buffer; the bytes
    around the output slice stay untouched."""
    Hq, Hkv, D = 32, 8, 128
    wl = W.make_custom(B=5, Hq=Hq, Hkv=Hkv, D=D, block_tokens=16, seq_lens=[3, 100, 900, 17, 2048],
                       sinks=True, seed=92 + Q, sm_scale=0.09, q_len=Q)
    dev = to_device(wl)
    T = wl.B * Q
    qkv = torch.randn(T, (Hq + 2 * Hkv) * D, device="cuda").to(torch.bfloat16)
    qkv[:, :Hq * D] = dev["q"].reshape(T, Hq * D)
    qv = qkv[:, :Hq * D].view(*wl.q.shape[:-2], Hq, D)
    assert qv.data_ptr() == qkv.data_ptr() and not qv.is_contiguous()
    obuf = torch.full((T, Hq * D + 72), 7.0, dtype=torch.bfloat16, device="cuda")
    ov = obuf[:, :Hq * D].view(*wl.q.shape[:-2], Hq, D)
    ro, rl = ref(wl)
    for chunk in (0, 4):
        out, lse = fpd.fp8_paged_decode_attention(qv, dev["k_cache"], dev["v_cache"],
                                                  dev["block_table"], dev["seq_lens"], wl.k_scale,
                                                  wl.v_scale, wl.sm_scale, sinks=dev["sinks"],
                                                  out=ov, chunk_pages_override=chunk)
        torch.cuda.synchronize()
        assert out.data_ptr() == obuf.data_ptr()
        compare(wl, out, lse, ro, rl, f"strided q/out q_len {Q} chunk {chunk}")
        assert (obuf[:, Hq * D:] == 7.0).all(), "bytes outside the output slice were written"


def test_device_scales_and_graph_replay():
    """Scales read from device memory; a captured graph replayed after the
    scale tensors change uses the new scales."""
    wl = W.make_custom(B=4, Hq=32, Hkv=8, D=128, block_tokens=16, seq_lens=[2000, 10, 700, 4000],
                       sinks=True, seed=93)
    dev = to_device(wl)
    ks = torch.tensor([wl.k_scale], dtype=torch.float32, device="cuda")
    vs = torch.tensor([wl.v_scale], dtype=torch.float32, device="cuda")
    need = fpd.fp8_paged_decode_workspace_bytes(4, 32, 8, 128, 16, wl.max_blocks)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")
    out = torch.empty((4, 32, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((4, 32), dtype=torch.float32, device="cuda")
    args = (dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"], ks, vs,
            wl.sm_scale)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fpd.fp8_paged_decode_attention(*args, sinks=dev["sinks"], out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    ro, rl = ref(wl)
    compare(wl, out, lse, ro, rl, "device scales")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fpd.fp8_paged_decode_attention(*args, sinks=dev["sinks"], out=out, lse=lse, workspace=ws)
    # new scales within a small factor of the ones the codes were quantised with
    # (values then stay in the data's range, as in a real cache; scales 100x
    # larger make |v| ~ 500, where the f16 rounding of P alone exceeds 1e-2)
    for kx, vx in ((wl.k_scale * 2, wl.v_scale * 0.5), (wl.k_scale * 0.5, wl.v_scale * 3),
                   (wl.k_scale * 1.3, wl.v_scale * 0.7)):
        ks.fill_(kx)
        vs.fill_(vx)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        ro, rl = ref(wl, k_scale=np.float32(kx), v_scale=np.float32(vx))
        compare(wl, out, lse, ro, rl, f"graph replay with scales {kx}, {vx}")
    # a scale written by a kernel just before the call (same stream) is seen
    kx = np.float32(wl.k_scale * 0.75)
    with torch.cuda.stream(s):
        ks.fill_(float(kx))
        vs.copy_(ks * 2)
        fpd.fp8_paged_decode_attention(*args, sinks=dev["sinks"], out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    ro, rl = ref(wl, k_scale=kx, v_scale=np.float32(kx * np.float32(2)))
    compare(wl, out, lse, ro, rl, "scale written just before")


@pytest.mark.parametrize("Q", [1, 2, 5])
def test_all_variants_together(Q):
    Hq, Hkv, D, bt = 16, 4, 128, 32
    wl = W.make_custom(B=6, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt,
                       seq_lens=[1, 4, 33, 500, 1200, 64], sinks=True, window_left=100,
                       seed=94 + Q, sm_scale=0.1, q_len=Q)
    q16 = f16_query(wl, 2)
    T = wl.B * Q
    wide = torch.zeros(T, Hq * D + 256, dtype=torch.float16, device="cuda")
    wide[:, 128:128 + Hq * D] = torch.from_numpy(q16.view(np.int16)).view(torch.float16).cuda() \
        .reshape(T, Hq * D)
    qv = wide[:, 128:128 + Hq * D].view(*wl.q.shape[:-2], Hq, D)
    dev = to_device(wl)
    kh = torch.from_numpy(to_hnd(wl.k_cache)).cuda()
    vh = torch.from_numpy(to_hnd(wl.v_cache)).cuda()
    ks = torch.tensor([wl.k_scale], dtype=torch.float32, device="cuda")
    obuf = torch.zeros(T, Hq * D + 8, dtype=torch.bfloat16, device="cuda")
    ov = obuf[:, :Hq * D].view(*wl.q.shape[:-2], Hq, D)
    ro, rl = ref(wl, q=q16, q_dtype="f16")
    for chunk in (0, 2):
        out, lse = fpd.fp8_paged_decode_attention(qv, kh, vh, dev["block_table"], dev["seq_lens"],
                                                  ks, wl.v_scale, wl.sm_scale,
                                                  window_left=wl.window_left, sinks=dev["sinks"],
                                                  out=ov, chunk_pages_override=chunk,
                                                  kv_layout="HND")
        torch.cuda.synchronize()
        compare(wl, out, lse, ro, rl, f"all variants q_len {Q} chunk {chunk}")


def test_cache_write_hnd_bit_exact():
    rng = np.random.default_rng(95)
    for Hkv, D, bt, T in ((2, 128, 16, 70), (8, 64, 32, 300), (4, 128, 64, 129)):
        nb = (T + bt - 1) // bt + 3
        key = torch.from_numpy((rng.standard_normal((T, Hkv, D)) * 2).astype(np.float32)) \
            .to(torch.bfloat16)
        value = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)) \
            .to(torch.bfloat16)
        slots = rng.permutation(nb * bt)[:T].astype(np.int64)
        slots[::11] = -1
        kc0 = rng.integers(0, 256, (nb, Hkv, bt, D), dtype=np.uint8)
        vc0 = rng.integers(0, 256, (nb, Hkv, bt, D), dtype=np.uint8)
        kc, vc = torch.from_numpy(kc0.copy()).cuda(), torch.from_numpy(vc0.copy()).cuda()
        fpd.fp8_paged_decode_cache_write(key.cuda(), value.cuda(), torch.from_numpy(slots).cuda(),
                                         kc, vc, 0.01, 0.004, kv_layout="HND")
        torch.cuda.synchronize()
        wk, wv = kc0.copy(), vc0.copy()
        kb = key.view(torch.int16).numpy().view(np.uint16)
        vb = value.view(torch.int16).numpy().view(np.uint16)
        oracle.cache_write(kb, vb, slots, wk, wv, k_scale=0.01, v_scale=0.004, kv_layout="HND")
        gk, gv = kc.cpu().numpy(), vc.cpu().numpy()
        for got, want, what in ((gk, wk, "K"), (gv, wv, "V")):
            nan = (want & 0x7F) == 0x7F
            assert np.array_equal(nan, (got & 0x7F) == 0x7F), f"{what}: NaN codes differ"
            assert np.array_equal(got[~nan], want[~nan]), f"HND {what} codes differ ({Hkv},{D},{bt})"
