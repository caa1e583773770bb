"""Pins that tie the CPU oracle to things other than itself.

Each ``pin_*`` function takes a loaded oracle library (ctypes handle) and raises
AssertionError when the oracle disagrees with

* a library routine that computes the same thing (torch's float8_e4m3fn and
  bfloat16 casts; torch's scaled_dot_product_attention in float64 with GQA,
  the sink given as an extra zero-valued key whose additive mask is the sink
  logit; scipy's logsumexp over numpy-matmul scores),
* a closed form (K == 0 gives the mean of the attended values and lse = ln n;
  a window of 0 keeps one key; constant value rows return that constant times
  the non-sink probability mass; the E4M3 format's extreme values), or
* an invariant (physical-page permutation, window >= L - 1, a -inf sink,
  k_scale <-> sm_scale exchange, v_scale linearity, identical query rows).

``tests/test_oracle_pins.py`` runs them against the oracle; the mutation test
runs them against deliberately broken copies of the oracle and requires every
copy to fail at least one pin.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from fp8_paged_decode_b200 import workloads as W


# ---------------------------------------------------------------- helpers --

def e4m3_library(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes -> float64 by torch's float8_e4m3fn cast (library routine)."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def bf16_library(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def f16_library(bits: np.ndarray) -> np.ndarray:
    """IEEE fp16 bit patterns -> float64 by numpy's float16 (library routine)."""
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def run(lib, wl, **kw):
    return oracle.decode_workload(wl, lib=lib, threads=4, **kw)


def library_attention(wl, qf=None):
    """Dense attention from the generator's per-sequence dense codes, by torch SDPA
    (out) and scipy logsumexp (lse), in float64.  qf: the query values (default:
    wl.q decoded as bf16)."""
    assert wl.k_dense is not None
    B, Hq, Hkv, D = wl.B, wl.Hq, wl.Hkv, wl.D
    g = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    qf = bf16_library(wl.q) if qf is None else qf
    for b in range(B):
        L = int(wl.seq_lens[b])
        start = max(0, L - 1 - wl.window_left) if wl.window_left >= 0 else 0
        K = e4m3_library(wl.k_dense[b][start:L]) * wl.k_scale   # [n, Hkv, D]
        V = e4m3_library(wl.v_dense[b][start:L]) * wl.v_scale
        n = L - start
        sig = None if wl.sinks is None else wl.sinks.astype(np.float64)
        if n == 0 and sig is None:
            out[b] = 0.0
            lse[b] = -np.inf
            continue
        extra = 0 if sig is None else 1
        Kt = torch.zeros((1, Hkv, n + extra, D), dtype=torch.float64)
        Vt = torch.zeros((1, Hkv, n + extra, D), dtype=torch.float64)
        Kt[0, :, :n] = torch.from_numpy(K).permute(1, 0, 2)
        Vt[0, :, :n] = torch.from_numpy(V).permute(1, 0, 2)
        mask = torch.zeros((1, Hq, 1, n + extra), dtype=torch.float64)
        if sig is not None:
            mask[0, :, 0, n] = torch.from_numpy(sig)
        qt = torch.from_numpy(qf[b]).reshape(1, Hq, 1, D)
        o = F.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=mask, scale=wl.sm_scale,
                                           enable_gqa=True)
        out[b] = o[0, :, 0, :].numpy()
        # scores by numpy matmul, lse by scipy
        Kh = np.repeat(K, g, axis=1)                     # [n, Hq, D], head h -> kv head h // g
        s = wl.sm_scale * np.einsum("hd,nhd->hn", qf[b], Kh)
        if sig is not None:
            s = np.concatenate([s, sig[:, None]], axis=1)
        lse[b] = scipy.special.logsumexp(s, axis=1)
    return out, lse


def close(a, b, rtol=1e-12, atol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    same_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        ok = same_inf | (np.abs(a - b) <= atol + rtol * np.abs(b))
    if not ok.all():
        i = np.argwhere(~ok)[0]
        raise AssertionError(f"{what}: mismatch at {tuple(i)}: {a[tuple(i)]!r} vs {b[tuple(i)]!r}")


def small_cases():
    """Small shapes covering GQA 1..16, D 64/128, page sizes 16/32/64, windows, sinks,
    ragged lengths (1, bt-1, bt, bt+1, multi-page) and an empty sequence."""
    return [
        W.make_custom(B=2, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[37, 300], seed=0,
                      keep_dense=True, sm_scale=1 / math.sqrt(128), name="tiny-like"),
        W.make_custom(B=5, Hq=4, Hkv=4, D=64, block_tokens=16, seq_lens=[1, 15, 16, 17, 70],
                      seed=11, keep_dense=True),
        W.make_custom(B=3, Hq=16, Hkv=2, D=64, block_tokens=32, seq_lens=[200, 33, 64],
                      window_left=40, sinks=True, sm_scale=0.125, seed=12, keep_dense=True),
        W.make_custom(B=3, Hq=32, Hkv=2, D=128, block_tokens=64, seq_lens=[129, 5, 64],
                      window_left=3, sinks=True, sm_scale=0.1, sigma=2.0, seed=13, keep_dense=True),
        W.make_custom(B=2, Hq=4, Hkv=2, D=128, block_tokens=16, seq_lens=[0, 23],
                      sinks=True, seed=14, keep_dense=True),
    ]


# ------------------------------------------------------------------- pins --

def pin_e4m3_codes(lib):
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([lib.fpd_oracle_e4m3_to_f64(int(c)) for c in codes])
    ref = e4m3_library(codes)
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all(), "NaN codes differ"
    assert (mine[~nan] == ref[~nan]).all(), "E4M3 values differ from torch.float8_e4m3fn"
    # format facts: only 0x7F / 0xFF are NaN; max finite 448 at 0x7E; smallest
    # normal 2^-6 at 0x08; smallest subnormal 2^-9 at 0x01; sign symmetry.
    assert set(np.flatnonzero(np.isnan(mine)).tolist()) == {0x7F, 0xFF}
    assert mine[0x7E] == 448.0 and mine[0x08] == 2.0 ** -6 and mine[0x01] == 2.0 ** -9
    assert (mine[0x80:0xFF] == -mine[0x00:0x7F]).all()
    pos = mine[0x00:0x7F]
    assert (np.diff(pos) > 0).all(), "positive codes must increase monotonically"


def pin_bf16(lib):
    rng = np.random.default_rng(7)
    bits = np.concatenate([rng.integers(0, 1 << 16, 4000, dtype=np.uint32).astype(np.uint16),
                           np.array([0x0000, 0x8000, 0x3F80, 0xBF80, 0x0001, 0x7F7F], np.uint16)])
    ref = bf16_library(bits)
    mine = np.array([lib.fpd_oracle_bf16_to_f64(int(x)) for x in bits])
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all()
    assert (mine[~nan] == ref[~nan]).all(), "bf16 decode differs from torch.bfloat16"


def pin_library_attention(lib, cases=None):
    for wl in cases or small_cases():
        out, lse = run(lib, wl)
        ref_out, ref_lse = library_attention(wl)
        close(out, ref_out, rtol=1e-10, atol=1e-12, what=f"out vs SDPA ({wl.name})")
        close(lse, ref_lse, rtol=1e-12, atol=1e-12, what=f"lse vs logsumexp ({wl.name})")


def pin_zero_keys(lib):
    """K == 0: every logit is 0, so out = mean of attended values (times the
    non-sink mass) and lse = ln n (or ln(n + e^sigma))."""
    for sinks, W_ in ((False, -1), (True, 20)):
        wl = W.make_custom(B=3, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[1, 50, 97],
                           window_left=W_, sinks=sinks, seed=21, keep_dense=True)
        wl.k_cache[:] = 0
        out, lse = run(lib, wl)
        for b in range(wl.B):
            L = int(wl.seq_lens[b])
            start = max(0, L - 1 - W_) if W_ >= 0 else 0
            n = L - start
            V = e4m3_library(wl.v_dense[b][start:L]) * wl.v_scale   # [n, Hkv, D]
            for h in range(wl.Hq):
                sig = wl.sinks[h] if sinks else -np.inf
                Z = n + math.exp(sig)
                close(lse[b, h], math.log(Z), what="lse, K=0")
                close(out[b, h], V[:, h // wl.groups, :].sum(0) / Z, atol=1e-13, what="out, K=0")


def pin_window_zero(lib):
    """window_left = 0 keeps only the newest key: out = v_last * p, lse = logaddexp(s, sigma)."""
    wl = W.make_custom(B=3, Hq=4, Hkv=1, D=128, block_tokens=32, seq_lens=[1, 33, 90],
                       window_left=0, sinks=True, seed=22, keep_dense=True)
    out, lse = run(lib, wl)
    qf = bf16_library(wl.q)
    for b in range(wl.B):
        L = int(wl.seq_lens[b])
        k = e4m3_library(wl.k_dense[b][L - 1, 0]) * wl.k_scale
        v = e4m3_library(wl.v_dense[b][L - 1, 0]) * wl.v_scale
        for h in range(wl.Hq):
            s = wl.sm_scale * float(np.dot(qf[b, h], k))
            sig = float(wl.sinks[h])
            l_ref = np.logaddexp(s, sig)
            close(lse[b, h], l_ref, what="lse, W=0")
            close(out[b, h], v * math.exp(s - l_ref), atol=1e-13, what="out, W=0")


def pin_constant_values(lib):
    """Every value row of KV head j equal to c_j: out[h] = c_{h//g} (1 - e^(sigma - lse))."""
    wl = W.make_custom(B=2, Hq=8, Hkv=4, D=64, block_tokens=16, seq_lens=[40, 77],
                       window_left=30, sinks=True, seed=23)
    consts = np.array([0x38, 0xB4, 0x41, 0x02], dtype=np.uint8)   # 1.0, -0.75, 2.25, 2^-8
    for j in range(wl.Hkv):
        wl.v_cache[:, :, j, :] = consts[j]
    out, lse = run(lib, wl)
    cval = e4m3_library(consts) * wl.v_scale
    for b in range(wl.B):
        for h in range(wl.Hq):
            mass = 1.0 - math.exp(float(wl.sinks[h]) - lse[b, h])
            close(out[b, h], np.full(wl.D, cval[h // wl.groups] * mass), rtol=1e-12, atol=1e-15,
                  what="constant V rows")


def pin_invariants(lib):
    wl = W.make_custom(B=3, Hq=8, Hkv=2, D=128, block_tokens=16, seq_lens=[5, 64, 131],
                       sinks=True, seed=24, sm_scale=0.09)
    out, lse = run(lib, wl)

    # physical page permutation (bitwise)
    rng = np.random.default_rng(5)
    perm = rng.permutation(wl.num_blocks)            # new position of each old page
    inv = np.argsort(perm)
    k2 = wl.k_cache[inv]
    v2 = wl.v_cache[inv]
    t2 = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    o2, l2 = oracle.decode(wl.q, k2, v2, t2, wl.seq_lens, k_scale=wl.k_scale, v_scale=wl.v_scale,
                           sm_scale=wl.sm_scale, window_left=-1, sinks=wl.sinks, lib=lib)
    assert np.array_equal(o2, out) and np.array_equal(l2, lse), "page permutation changed the result"

    # a window covering the whole sequence equals no window (bitwise)
    for Wl in (int(wl.seq_lens.max()) - 1, int(wl.seq_lens.max()), 10 ** 6):
        o3, l3 = run(lib, wl, window_left=Wl)
        assert np.array_equal(o3, out) and np.array_equal(l3, lse), f"window {Wl} != no window"

    # a -inf sink equals no sink
    o4, l4 = run(lib, wl, sinks=None)
    o5, l5 = run(lib, wl, sinks=np.full(wl.Hq, -np.inf, np.float32))
    assert np.array_equal(o4, o5) and np.array_equal(l4, l5), "-inf sink != no sink"
    # and a huge sink absorbs all mass
    o6, l6 = run(lib, wl, sinks=np.full(wl.Hq, 1e4, np.float32))
    close(l6, np.full_like(l6, 1e4), what="huge sink lse")
    assert np.abs(o6).max() == 0.0, "huge sink must leave zero output"

    # k_scale * a  <->  sm_scale * a
    a = 1.75
    oa, la = oracle.decode(wl.q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                           k_scale=wl.k_scale * a, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                           sinks=wl.sinks, lib=lib)
    ob, lb = oracle.decode(wl.q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                           k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale * a,
                           sinks=wl.sinks, lib=lib)
    close(oa, ob, rtol=1e-11, atol=1e-14, what="k_scale/sm_scale exchange")
    close(la, lb, rtol=1e-12, what="k_scale/sm_scale exchange (lse)")
    # v_scale is linear (doubling is exact)
    oc, lc = oracle.decode(wl.q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                           k_scale=wl.k_scale, v_scale=wl.v_scale * 2, sm_scale=wl.sm_scale,
                           sinks=wl.sinks, lib=lib)
    assert np.array_equal(oc, 2 * out) and np.array_equal(lc, lse), "v_scale not linear"

    # identical query rows inside one GQA group give identical rows
    q2 = wl.q.copy()
    g = wl.groups
    for j in range(wl.Hkv):
        q2[:, j * g:(j + 1) * g, :] = q2[:, j * g:j * g + 1, :]
    od, ld = oracle.decode(q2, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                           k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                           sinks=np.repeat(wl.sinks[::g], g), lib=lib)
    for j in range(wl.Hkv):
        for h in range(j * g, (j + 1) * g):
            assert np.array_equal(od[:, h], od[:, j * g]) and np.array_equal(ld[:, h], ld[:, j * g])


def pin_softmax_identity(lib):
    """sum_j e^(s_j - lse) + e^(sigma - lse) = 1 with s_j from numpy."""
    wl = W.make_custom(B=2, Hq=4, Hkv=2, D=64, block_tokens=16, seq_lens=[3, 45], sinks=True,
                       sm_scale=0.3, seed=25, keep_dense=True)
    _, lse = run(lib, wl)
    qf = bf16_library(wl.q)
    for b in range(wl.B):
        K = e4m3_library(wl.k_dense[b]) * wl.k_scale
        for h in range(wl.Hq):
            s = wl.sm_scale * K[:, h // wl.groups, :] @ qf[b, h]
            tot = np.exp(s - lse[b, h]).sum() + math.exp(float(wl.sinks[h]) - lse[b, h])
            assert abs(tot - 1.0) < 1e-12, f"probabilities sum to {tot}"


# ----------------------------------------------------- several query tokens --

def pin_multi_token_library(lib):
    """q_len queries per sequence against torch SDPA (float64, an explicit
    causal + window mask, the sink as an extra zero-valued key) and scipy
    logsumexp."""
    # (a first sequence shorter than q_len: its earliest queries sit before the
    # first key and see only the sink)
    for Q, window, L0 in ((3, -1, 3), (4, 20, 4), (2, 0, 2), (5, -1, 2), (4, 1, 1)):
        wl = W.make_custom(B=3, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[L0, 37, 90],
                           sinks=True, window_left=window, seed=51 + Q + L0, sm_scale=0.2,
                           keep_dense=True, q_len=Q)
        q = wl.q
        out, lse = oracle.decode(q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                                 k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                                 window_left=window, sinks=wl.sinks, lib=lib, threads=2)
        qf = bf16_library(q)
        g = wl.Hq // wl.Hkv
        sig = wl.sinks.astype(np.float64)
        for b in range(wl.B):
            L = int(wl.seq_lens[b])
            s0 = max(0, L - Q - window) if window >= 0 else 0   # first key any query sees
            n = L - s0
            K = e4m3_library(wl.k_dense[b][s0:L]) * wl.k_scale
            V = e4m3_library(wl.v_dense[b][s0:L]) * wl.v_scale
            Kt = torch.zeros((1, wl.Hkv, n + 1, wl.D), dtype=torch.float64)
            Vt = torch.zeros_like(Kt)
            Kt[0, :, :n] = torch.from_numpy(K).permute(1, 0, 2)
            Vt[0, :, :n] = torch.from_numpy(V).permute(1, 0, 2)
            mask = torch.full((1, wl.Hq, Q, n + 1), -math.inf, dtype=torch.float64)
            for i in range(Q):
                p = L - Q + i
                if p < 0:
                    continue   # no key at or before this query's position
                lo = max(0, p - window) if window >= 0 else 0
                mask[0, :, i, lo - s0:p + 1 - s0] = 0.0
            mask[0, :, :, n] = torch.from_numpy(sig)[:, None]
            qt = torch.from_numpy(qf[b]).permute(1, 0, 2).unsqueeze(0)   # [1, Hq, Q, D]
            o = F.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=mask, scale=wl.sm_scale,
                                               enable_gqa=True)
            close(out[b], o[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12,
                  what=f"multi-token out (Q={Q}, window {window})")
            Kh = np.repeat(K, g, axis=1)
            sc = wl.sm_scale * np.einsum("ihd,nhd->ihn", qf[b], Kh)
            sc = np.where(mask[0, :, :, :n].permute(1, 0, 2).numpy() == 0, sc, -np.inf)
            sc = np.concatenate([sc, np.broadcast_to(sig[None, :, None], (Q, wl.Hq, 1))], axis=2)
            close(lse[b], scipy.special.logsumexp(sc, axis=2), rtol=1e-12, atol=1e-12,
                  what="multi-token lse")


def pin_multi_token_prefix(lib):
    """Query i of q_len equals a one-query decode of the sequence cut after
    position L - q_len + i (what a causal query sees), with and without a
    window."""
    for window in (-1, 7):
        Q = 5
        wl = W.make_custom(B=2, Hq=4, Hkv=4, D=128, block_tokens=32, seq_lens=[50, 200],
                           sinks=False, window_left=window, seed=53, sm_scale=0.1, q_len=Q)
        q = wl.q
        out, lse = oracle.decode(q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                                 k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                                 window_left=window, lib=lib, threads=2)
        for i in range(Q):
            lens = wl.seq_lens - Q + i + 1
            o1, l1 = oracle.decode(np.ascontiguousarray(q[:, i]), wl.k_cache, wl.v_cache,
                                   wl.block_table, lens, k_scale=wl.k_scale,
                                   v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                                   window_left=window, lib=lib, threads=2)
            assert np.array_equal(out[:, i], o1) and np.array_equal(lse[:, i], l1), \
                f"query {i} differs from the truncated single-query decode"


# ------------------------------------------------------------ cache write --

def e4m3_encode_library(x: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 codes by torch's float8_e4m3fn cast (round to nearest
    even; defined by torch for |x| <= 448 only)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def pin_e4m3_encode_library(lib):
    """Random float32 values, every code value and every midpoint between
    neighbouring codes, against torch's cast."""
    rng = np.random.default_rng(40)
    vals = [rng.standard_normal(4000) * s for s in (0.003, 0.1, 1.0, 30.0, 200.0)]
    codes = np.arange(256, dtype=np.uint8)
    real = e4m3_library(codes)
    finite = np.sort(np.unique(real[np.isfinite(real)]))
    mids = (finite[1:] + finite[:-1]) / 2                         # exact in float32
    x = np.concatenate(vals + [finite, mids, -mids]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    want = e4m3_encode_library(x)
    got = np.array([oracle.f64_to_e4m3(float(v), lib=lib) for v in x], dtype=np.uint8)
    bad = np.flatnonzero(want != got)
    assert bad.size == 0, f"{bad.size} codes differ, e.g. x={x[bad[0]]!r}: {got[bad[0]]:#x} vs {want[bad[0]]:#x}"


def pin_e4m3_encode_closed(lib):
    """Closed forms of the encoder: every non-NaN code round-trips, ties go to
    the even code, +-inf and anything past 448 saturate, signs (and the sign of
    zero) are kept, NaN stays NaN."""
    enc = lambda v: oracle.f64_to_e4m3(v, lib=lib)
    for c in range(256):
        if c & 0x7F == 0x7F:
            continue
        v = oracle.e4m3_to_f64(c, lib=lib)
        assert enc(v) == c, f"code {c:#x} ({v}) does not round-trip"
    assert enc(1.0 + 1 / 16) == 0x38 and enc(1.0 + 3 / 16) == 0x3A        # ties to even
    assert enc(2.0 ** -10) == 0x00 and enc(3 * 2.0 ** -10) == 0x02         # subnormal ties
    assert enc(2.0 ** -10 * 1.0001) == 0x01
    for v in (448.0, 449.0, 464.0, 1e30, math.inf):
        assert enc(v) == 0x7E and enc(-v) == 0xFE, f"{v} does not saturate"
    assert enc(0.0) == 0x00 and enc(-0.0) == 0x80 and enc(-1e-9) == 0x80
    assert enc(math.nan) & 0x7F == 0x7F


def cache_write_library(key, value, slots, k_cache, v_cache, k_scale, v_scale):
    """The cache write with torch: float32 product with the float32 reciprocal of
    the scale, clamp to +-448, torch's float8 cast, numpy scatter."""
    kc, vc = k_cache.copy(), v_cache.copy()
    nb, bt, H, D = kc.shape
    for src, scale, dst in ((key, k_scale, kc), (value, v_scale, vc)):
        x = torch.from_numpy(np.ascontiguousarray(src).view(np.int16)).view(torch.bfloat16).float()
        y = x * (torch.tensor(1.0, dtype=torch.float32) / torch.tensor(scale, dtype=torch.float32))
        codes = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        flat = dst.reshape(nb * bt, H, D)
        for t, sl in enumerate(slots):
            if 0 <= sl < nb * bt:
                flat[sl] = codes[t]
    return kc, vc


def pin_cache_write_library(lib):
    """Scatter with negative (skipped) slots and a strided key, bit-exact
    against the torch version."""
    rng = np.random.default_rng(41)
    nb, bt, H, D, T = 7, 16, 3, 64, 40
    wide = rng.standard_normal((T, H * D * 2)).astype(np.float32) * 3
    kbits = torch.from_numpy(wide).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    key = kbits[:, : H * D].reshape(T, H, D)            # token stride 2*H*D: a slice
    value = torch.from_numpy(rng.standard_normal((T, H, D)).astype(np.float32) * 50).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    slots[slots == 0] = slots[0]
    slots[0] = 0                                        # the first slot of the pool is used
    slots[[3, 17, 30]] = -1                             # padded tokens
    kc0 = rng.integers(0, 256, (nb, bt, H, D), dtype=np.uint8)
    vc0 = rng.integers(0, 256, (nb, bt, H, D), dtype=np.uint8)
    for ks, vs in ((0.02, 0.5), (1.0, 1.0), (3.7, 0.013)):
        kc, vc = kc0.copy(), vc0.copy()
        assert oracle.cache_write(key, value, slots, kc, vc, k_scale=ks, v_scale=vs, lib=lib) == 0
        wk, wv = cache_write_library(key, value, slots, kc0, vc0, ks, vs)
        assert np.array_equal(kc, wk), "K cache differs"
        assert np.array_equal(vc, wv), "V cache differs"


def pin_cache_write_invariants(lib):
    """Permuting tokens together with their slots changes nothing; an
    out-of-range slot is reported and skipped; a cache read back through the
    decoder returns the (scaled) values when they are exact E4M3 values."""
    rng = np.random.default_rng(42)
    nb, bt, H, D, T = 5, 32, 2, 128, 50
    key = torch.from_numpy(rng.standard_normal((T, H, D)).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    value = key[::-1].copy()
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    kc = np.zeros((nb, bt, H, D), np.uint8)
    vc = np.zeros_like(kc)
    oracle.cache_write(key, value, slots, kc, vc, k_scale=0.25, v_scale=2.0, lib=lib)
    perm = rng.permutation(T)
    kc2, vc2 = np.zeros_like(kc), np.zeros_like(vc)
    oracle.cache_write(np.ascontiguousarray(key[perm]), np.ascontiguousarray(value[perm]),
                       slots[perm], kc2, vc2, k_scale=0.25, v_scale=2.0, lib=lib)
    assert np.array_equal(kc, kc2) and np.array_equal(vc, vc2)
    bad = slots.copy()
    bad[5] = nb * bt
    kc3, vc3 = np.zeros_like(kc), np.zeros_like(vc)
    assert oracle.cache_write(key, value, bad, kc3, vc3, k_scale=0.25, v_scale=2.0, lib=lib) == 1
    assert not kc3.reshape(-1, H, D)[slots[5]].any(), "the skipped token was written"
    # exact values: codes decoded and scaled back are the inputs
    codes = rng.integers(0, 0x7F, (T, H, D)).astype(np.uint8)
    exact = e4m3_library(codes) * 0.5                   # bf16 holds these exactly
    xb = torch.from_numpy(exact).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kc4, vc4 = np.zeros_like(kc), np.zeros_like(vc)
    oracle.cache_write(xb, xb, slots, kc4, vc4, k_scale=0.5, v_scale=0.5, lib=lib)
    back = e4m3_library(kc4.reshape(-1, H, D)[slots]) * 0.5
    assert np.array_equal(back, exact)


# ---------------------------------------------------- interface variants --

def pin_f16_codes(lib):
    """All 65536 fp16 bit patterns against numpy's float16 (NaN as NaN)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = f16_library(bits)
    got = np.array([lib.fpd_oracle_f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan), "fp16 NaN patterns differ"
    assert np.array_equal(got[~nan], want[~nan]), "fp16 decode differs from numpy float16"


def pin_f16_query_library(lib):
    """An fp16 query against torch SDPA / scipy logsumexp on the same values."""
    for wl in small_cases()[:4]:
        rng = np.random.default_rng(61)
        q16 = (rng.standard_normal(wl.q.shape) * 3.0).astype(np.float16)
        q16.reshape(-1)[::7] *= np.float16(1e-3)         # small and subnormal-range values
        bits = q16.view(np.uint16)
        out, lse = oracle.decode(bits, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                                 k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                                 window_left=wl.window_left, sinks=wl.sinks, lib=lib, threads=2,
                                 q_dtype="f16")
        ref_out, ref_lse = library_attention(wl, qf=f16_library(bits))
        close(out, ref_out, rtol=1e-10, atol=1e-12, what=f"{wl.name} fp16-q out")
        close(lse, ref_lse, rtol=1e-12, atol=1e-12, what=f"{wl.name} fp16-q lse")


def to_hnd(cache: np.ndarray) -> np.ndarray:
    """[num_blocks, bt, Hkv, D] -> [num_blocks, Hkv, bt, D] (numpy transpose)."""
    return np.ascontiguousarray(cache.transpose(0, 2, 1, 3))


def pin_hnd_layout(lib):
    """Head-major pages hold the same elements at other addresses: decoding the
    transposed caches as HND equals the token-major decode bitwise, for one and
    several queries; and the cache write into HND pages equals the token-major
    write transposed."""
    cases = small_cases()
    cases.append(W.make_custom(B=3, Hq=8, Hkv=4, D=64, block_tokens=32, seq_lens=[3, 40, 99],
                               sinks=True, window_left=10, seed=62, q_len=3))
    for wl in cases:
        kw = dict(k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                  window_left=wl.window_left, sinks=wl.sinks, lib=lib, threads=2)
        o1, l1 = oracle.decode(wl.q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens, **kw)
        o2, l2 = oracle.decode(wl.q, to_hnd(wl.k_cache), to_hnd(wl.v_cache), wl.block_table,
                               wl.seq_lens, kv_layout="HND", **kw)
        assert np.array_equal(o1, o2, equal_nan=True) and np.array_equal(l1, l2, equal_nan=True), \
            f"{wl.name}: HND decode differs from the token-major decode"
    rng = np.random.default_rng(63)
    T, Hkv, D, bt, nb = 40, 2, 64, 16, 4
    key = bf16_bits_of(rng.standard_normal((T, Hkv, D)))
    value = bf16_bits_of(rng.standard_normal((T, Hkv, D)))
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    slots[::9] = -1
    kc = rng.integers(0, 256, (nb, bt, Hkv, D), dtype=np.uint8)
    vc = rng.integers(0, 256, (nb, bt, Hkv, D), dtype=np.uint8)
    kh, vh = to_hnd(kc), to_hnd(vc)
    oracle.cache_write(key, value, slots, kc, vc, k_scale=0.02, v_scale=0.01, lib=lib)
    oracle.cache_write(key, value, slots, kh, vh, k_scale=0.02, v_scale=0.01, lib=lib,
                       kv_layout="HND")
    assert np.array_equal(kh, to_hnd(kc)) and np.array_equal(vh, to_hnd(vc)), \
        "HND cache write differs from the token-major write"


def bf16_bits_of(x: np.ndarray) -> np.ndarray:
    """float -> bf16 bit patterns by torch's bfloat16 cast (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ NVFP4 --

def e2m1_library(codes: np.ndarray) -> np.ndarray:
    """E2M1 codes (low 4 bits) -> float64 by ml_dtypes' float4_e2m1fn (library)."""
    import ml_dtypes
    return np.ascontiguousarray(codes, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn) \
        .astype(np.float64)


def nvfp4_dense(wl, side):
    """Dense [num_blocks, Hkv, bt, D] real values (without the per-tensor scale)
    of one side of an NVFP4 workload's pages, by numpy views of the page bytes,
    ml_dtypes' E2M1 and torch's E4M3 decoding."""
    lay = oracle.nvfp4_page_layout(wl.Hkv, wl.block_tokens, wl.D)
    nb, Hkv, bt, D = wl.num_blocks, wl.Hkv, wl.block_tokens, wl.D
    d0 = lay["k_data" if side == 0 else "v_data"]
    s0 = lay["k_sf" if side == 0 else "v_sf"]
    data = wl.kv_cache[:, d0:d0 + Hkv * bt * D // 2].reshape(nb, Hkv, bt, D // 2)
    sf = wl.kv_cache[:, s0:s0 + Hkv * bt * D // 16].reshape(nb, Hkv, bt, D // 16)
    codes = np.empty((nb, Hkv, bt, D), dtype=np.uint8)
    codes[..., 0::2] = data & 0xF
    codes[..., 1::2] = data >> 4
    return e2m1_library(codes) * np.repeat(e4m3_library(sf), 16, axis=-1)


def nvfp4_cases():
    return [
        W.make_custom_nvfp4(B=3, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[1, 40, 100],
                            sinks=True, seed=71),
        W.make_custom_nvfp4(B=2, Hq=16, Hkv=4, D=128, block_tokens=32, seq_lens=[70, 129],
                            window_left=50, sinks=True, seed=72, sm_scale=0.1, q_len=3),
        W.make_custom_nvfp4(B=2, Hq=4, Hkv=4, D=128, block_tokens=64, seq_lens=[0, 200],
                            seed=73),
    ]


def pin_e2m1_codes(lib):
    """All 16 E2M1 codes against ml_dtypes."""
    codes = np.arange(16, dtype=np.uint8)
    got = np.array([lib.fpd_oracle_e2m1_to_f64(int(c)) for c in codes])
    want = e2m1_library(codes)
    assert np.array_equal(got, want) and np.array_equal(np.signbit(got), np.signbit(want)), \
        "E2M1 decode differs from ml_dtypes"


def pin_e2m1_encode_library(lib):
    """Nearest-even, saturating E2M1 encoding against ml_dtypes' cast, on ties,
    overflow, tiny values and random values of both signs."""
    import ml_dtypes
    rng = np.random.default_rng(74)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    x = np.concatenate([ties, -ties, [0.0, -0.0, 6.0, 6.5, 7.0, 1e9, -1e9, np.inf, -np.inf,
                                      1e-30, -1e-30], rng.standard_normal(4000) * 3,
                        rng.uniform(-8, 8, 4000)])
    got = np.array([lib.fpd_oracle_f64_to_e2m1(float(v)) for v in x], dtype=np.uint8)
    want = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(got, want), \
        f"E2M1 encode differs at {x[np.argmax(got != want)]!r}"


def pin_nvfp4_decode_library(lib):
    """NVFP4 decode against torch SDPA and scipy logsumexp on the pages'
    values decoded by numpy views, ml_dtypes and torch (float64)."""
    for wl in nvfp4_cases():
        out, lse = oracle.decode_nvfp4_workload(wl, lib=lib, threads=2)
        Kd, Vd = nvfp4_dense(wl, 0), nvfp4_dense(wl, 1)
        Q = wl.q_len
        qf = bf16_library(wl.q).reshape(wl.B, Q, wl.Hq, wl.D)
        g = wl.Hq // wl.Hkv
        sig = wl.sinks.astype(np.float64) if wl.sinks is not None else None
        ro = np.zeros((wl.B, Q, wl.Hq, wl.D))
        rl = np.zeros((wl.B, Q, wl.Hq))
        for b in range(wl.B):
            L = int(wl.seq_lens[b])
            j = np.arange(L)
            pages = wl.block_table[b, j // wl.block_tokens]
            K = Kd[pages, :, j % wl.block_tokens] * wl.k_scale    # [L, Hkv, D]
            V = Vd[pages, :, j % wl.block_tokens] * wl.v_scale
            for i in range(Q):
                p = L - Q + i
                lo = max(0, p - wl.window_left) if wl.window_left >= 0 else 0
                n = max(0, p + 1 - lo)
                Kt = torch.zeros((1, wl.Hkv, n + 1, wl.D), dtype=torch.float64)
                Vt = torch.zeros_like(Kt)
                if n:
                    Kt[0, :, :n] = torch.from_numpy(K[lo:p + 1]).permute(1, 0, 2)
                    Vt[0, :, :n] = torch.from_numpy(V[lo:p + 1]).permute(1, 0, 2)
                mask = torch.zeros((1, wl.Hq, 1, n + 1), dtype=torch.float64)
                mask[0, :, 0, n] = torch.from_numpy(sig) if sig is not None else -math.inf
                if n == 0 and sig is None:
                    ro[b, i] = 0.0
                    rl[b, i] = -np.inf
                    continue
                qt = torch.from_numpy(qf[b, i]).reshape(1, wl.Hq, 1, wl.D)
                o = F.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=mask,
                                                   scale=wl.sm_scale, enable_gqa=True)
                ro[b, i] = o[0, :, 0].numpy()
                sc = wl.sm_scale * np.einsum("hd,nhd->hn", qf[b, i],
                                             np.repeat(K[lo:p + 1], g, axis=1))
                if sig is not None:
                    sc = np.concatenate([sc, sig[:, None]], axis=1)
                rl[b, i] = scipy.special.logsumexp(sc, axis=1)
        close(out.reshape(ro.shape), ro, rtol=1e-10, atol=1e-12, what=f"{wl.name} NVFP4 out")
        close(lse.reshape(rl.shape), rl, rtol=1e-12, atol=1e-12, what=f"{wl.name} NVFP4 lse")


def pin_nvfp4_page_strides(lib):
    """The four page regions as separate arrays (their own page strides) give
    the bits of the combined page layout."""
    for wl in nvfp4_cases():
        lay = oracle.nvfp4_page_layout(wl.Hkv, wl.block_tokens, wl.D)
        nb, shp = wl.num_blocks, (wl.num_blocks, wl.Hkv, wl.block_tokens)
        db, sb = wl.Hkv * wl.block_tokens * wl.D // 2, wl.Hkv * wl.block_tokens * wl.D // 16
        reg = tuple(np.ascontiguousarray(wl.kv_cache[:, lay[k]:lay[k] + n]).reshape(shp + (n // (shp[1] * shp[2]),))
                    for k, n in (("k_data", db), ("k_sf", sb), ("v_data", db), ("v_sf", sb)))
        kw = dict(Hkv=wl.Hkv, block_tokens=wl.block_tokens, k_scale=wl.k_scale,
                  v_scale=wl.v_scale, sm_scale=wl.sm_scale, window_left=wl.window_left,
                  sinks=wl.sinks, lib=lib, threads=2)
        o1, l1 = oracle.decode_nvfp4(wl.q, wl.kv_cache, wl.block_table, wl.seq_lens, **kw)
        o2, l2 = oracle.decode_nvfp4(wl.q, None, wl.block_table, wl.seq_lens, regions=reg, **kw)
        assert np.array_equal(o1, o2, equal_nan=True) and np.array_equal(l1, l2, equal_nan=True), \
            "separate page regions differ from the combined page"
        del nb


def nvfp4_writer_library(key_bits, value_bits, k_scale, v_scale):
    """The writer's codes by library roundings: torch's E4M3 cast for the block
    scale, ml_dtypes' E2M1 cast for the elements, numpy float32 products."""
    import ml_dtypes
    T, Hkv, D = key_bits.shape
    res = []
    for bits, scale in ((key_bits, k_scale), (value_bits, v_scale)):
        x = bf16_library(bits).astype(np.float32).reshape(T, Hkv, D // 16, 16)
        gs = np.float32(1.0) / np.float32(scale)
        amax = np.abs(x).max(axis=-1)
        sf_f = (amax * (np.float32(1.0) / np.float32(6.0))) * gs
        sfc = torch.from_numpy(sf_f.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sfv = e4m3_library(sfc).astype(np.float32)
        with np.errstate(divide="ignore"):
            osc = np.where(sfv == 0, np.float32(0),
                           np.float32(1.0) / (sfv * (np.float32(1.0) / gs))).astype(np.float32)
        y = (x * osc[..., None]).astype(np.float32)
        codes = y.astype(np.float64).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
        res.append((codes.reshape(T, Hkv, D), sfc))
    return res


def pin_nvfp4_writer_library(lib):
    """The NVFP4 cache writer's codes and block scales against the same
    recipe computed with library roundings; slots land in the page layout."""
    rng = np.random.default_rng(75)
    for Hkv, D, bt, T in ((2, 64, 16, 40), (4, 128, 32, 70)):
        x = rng.standard_normal((2, T, Hkv, D)).astype(np.float32) * 2
        x[:, ::7, :, :16] *= 1e-3
        x[:, 3, 0, 16:32] = 0.0                          # an all-zero block
        kb, vb = (torch.from_numpy(x[i]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
                  for i in range(2))
        nb = T // bt + 3
        lay = oracle.nvfp4_page_layout(Hkv, bt, D)
        kv = np.zeros((nb, lay["page_bytes"]), dtype=np.uint8)
        slots = rng.permutation(nb * bt)[:T].astype(np.int64)
        slots[::5] = -1
        ks, vs = 0.05, 0.03
        assert oracle.cache_write_nvfp4(kb, vb, slots, kv, block_tokens=bt, k_scale=ks,
                                        v_scale=vs, lib=lib) == 0
        (kc, ksf), (vc, vsf) = nvfp4_writer_library(kb, vb, np.float32(ks), np.float32(vs))
        for side, (codes, sfc) in enumerate(((kc, ksf), (vc, vsf))):
            d0 = lay["k_data" if side == 0 else "v_data"]
            s0 = lay["k_sf" if side == 0 else "v_sf"]
            data = kv[:, d0:d0 + Hkv * bt * D // 2].reshape(nb, Hkv, bt, D // 2)
            sf = kv[:, s0:s0 + Hkv * bt * D // 16].reshape(nb, Hkv, bt, D // 16)
            for t in range(T):
                if slots[t] < 0:
                    continue
                pg, off = divmod(int(slots[t]), bt)
                got = np.empty((Hkv, D), dtype=np.uint8)
                got[:, 0::2] = data[pg, :, off] & 0xF
                got[:, 1::2] = data[pg, :, off] >> 4
                assert np.array_equal(got, codes[t]), f"side {side} token {t}: codes differ"
                assert np.array_equal(sf[pg, :, off], sfc[t]), f"side {side} token {t}: scales differ"


def pin_nvfp4_round_trip(lib):
    """Closed forms of the write -> decode round trip: values c * s * k_scale
    with c an E2M1 value, max |c| = 6 per block, s a power of two and k_scale a
    power of two come back exactly; an all-zero block gives scale code 0; on
    random data every element is within one block step (scale * k_scale) of
    its input."""
    rng = np.random.default_rng(76)
    Hkv, D, bt, T = 2, 64, 16, 20
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    c = vals[rng.integers(0, 8, (T, Hkv, D // 16, 16))] * rng.choice([-1.0, 1.0], (T, Hkv, D // 16, 16))
    c[..., 0] = 6.0
    s = 2.0 ** rng.integers(-4, 5, (T, Hkv, D // 16, 1))
    k_scale = 0.125
    x = (c * s * k_scale).reshape(T, Hkv, D)
    x[0, 1, :16] = 0.0
    bits = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_library(bits), x)
    nb = T // bt + 2
    lay = oracle.nvfp4_page_layout(Hkv, bt, D)
    kv = np.zeros((nb, lay["page_bytes"]), dtype=np.uint8)
    slots = np.arange(T, dtype=np.int64)
    oracle.cache_write_nvfp4(bits, bits, slots, kv, block_tokens=bt, k_scale=k_scale,
                             v_scale=k_scale, lib=lib)
    wl = W.Workload(name="rt", seed=0, B=1, Hq=Hkv, Hkv=Hkv, D=D, block_tokens=bt, num_blocks=nb,
                    max_blocks=nb, q=np.zeros((1, Hkv, D), np.uint16), k_cache=None, v_cache=None,
                    block_table=np.arange(nb, dtype=np.int32)[None], seq_lens=np.array([T], np.int32),
                    k_scale=k_scale, v_scale=k_scale, sm_scale=1.0, window_left=-1, sinks=None,
                    kv_format="nvfp4", kv_cache=kv)
    dense = nvfp4_dense(wl, 0).transpose(0, 2, 1, 3).reshape(nb * bt, Hkv, D)[:T] * k_scale
    assert np.array_equal(dense, x), "exactly representable blocks do not round-trip"
    sf = kv[:, lay["k_sf"]:lay["k_sf"] + Hkv * bt * D // 16].reshape(nb, Hkv, bt, D // 16)
    assert sf[0, 1, 0, 0] == 0, "an all-zero block must get scale code 0"
    # random data: within one block step
    y = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    yb = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kv2 = np.zeros_like(kv)
    oracle.cache_write_nvfp4(yb, yb, slots, kv2, block_tokens=bt, k_scale=0.02, v_scale=0.02,
                             lib=lib)
    wl.kv_cache, wl.k_scale = kv2, 0.02
    d2 = nvfp4_dense(wl, 0).transpose(0, 2, 1, 3).reshape(nb * bt, Hkv, D)[:T] * 0.02
    sf2 = kv2[:, lay["k_sf"]:lay["k_sf"] + Hkv * bt * D // 16].reshape(nb, Hkv, bt, D // 16)
    step = np.repeat(e4m3_library(sf2).transpose(0, 2, 1, 3).reshape(nb * bt, Hkv, D // 16)[:T],
                     16, axis=-1) * 0.02
    assert (np.abs(d2 - bf16_library(yb)) <= step + 1e-12).all(), "round-trip error above one step"


def _page_split(table, lens, bt, parts, r):
    """Part r of `parts` of every sequence's pages: a contiguous run of whole pages."""
    pages = -(-lens // bt)
    t = np.zeros_like(table)
    l = np.zeros_like(lens)
    for b in range(len(lens)):
        p0, p1 = r * pages[b] // parts, (r + 1) * pages[b] // parts
        t[b, :p1 - p0] = table[b, p0:p1]
        l[b] = max(0, min(p1 * bt, lens[b]) - p0 * bt)
    return t, l


def pin_merge_library(lib):
    """The merge of partial results over disjoint key sets (context-parallel
    decode): the oracle's decodes of each part's keys, without the sink,
    merged with the sink, equal dense attention over all keys by torch SDPA
    and scipy logsumexp.  Parts from 1 to 5, some of them empty."""
    for wl in small_cases():
        if wl.window_left >= 0:
            continue   # windows and positions are not part of the merge
        for parts in (1, 2, 3, 5):
            o_p, l_p = [], []
            for r in range(parts):
                t, l = _page_split(wl.block_table, wl.seq_lens, wl.block_tokens, parts, r)
                o, ls = oracle.decode(wl.q, wl.k_cache, wl.v_cache, t, l, k_scale=wl.k_scale,
                                      v_scale=wl.v_scale, sm_scale=wl.sm_scale, sinks=None,
                                      threads=4, lib=lib)
                o_p.append(o)
                l_p.append(ls)
            out, lse = oracle.merge(np.stack(o_p), np.stack(l_p), wl.Hq, wl.sinks, lib=lib)
            ref_out, ref_lse = library_attention(wl)
            close(out, ref_out, rtol=1e-10, atol=1e-12, what=f"merged out ({wl.name}, {parts})")
            close(lse, ref_lse, rtol=1e-12, atol=1e-12, what=f"merged lse ({wl.name}, {parts})")


ALL_PINS = [pin_e4m3_codes, pin_bf16, pin_library_attention, pin_zero_keys, pin_window_zero,
            pin_constant_values, pin_invariants, pin_softmax_identity, pin_e4m3_encode_library,
            pin_e4m3_encode_closed, pin_cache_write_library, pin_cache_write_invariants,
            pin_multi_token_library, pin_multi_token_prefix, pin_f16_codes,
            pin_f16_query_library, pin_hnd_layout, pin_e2m1_codes, pin_e2m1_encode_library,
            pin_nvfp4_decode_library, pin_nvfp4_page_strides, pin_nvfp4_writer_library,
            pin_nvfp4_round_trip, pin_merge_library]
