"""Seeded synthetic inputs for paged FP8 decode attention.

This module is the one piece of code shared by the CUDA path's tests/bench and
the CPU oracle: it draws the inputs and holds none of the attention arithmetic.
It builds, for a decode step,

* ``q``            bf16 ``[B, Hq, D]`` (stored as raw uint16 bit patterns),
* ``k_cache``      E4M3 codes ``[num_blocks, block_tokens, Hkv, D]`` (uint8),
* ``v_cache``      same shape as ``k_cache``,
* ``block_table``  int32 ``[B, max_blocks]`` (-1 in unused slots),
* ``seq_lens``     int32 ``[B]``,
* per-tensor ``k_scale`` / ``v_scale`` (float32 values), ``sm_scale``,
  ``window_left`` and optional per-head ``sinks`` (float32 ``[Hq]``).

Layout follows the paged-KV convention of the serving stacks the pages describe
(FlashInfer/SGLang "paged KV" with a per-sequence block table; the cache page
is token-major, "NHD", as in the NVFP4 KV-cache gist, section on the cache
writer's layout detection).  Physical pages are a seeded random permutation of
the pool, so a kernel that ignores the block table reads the wrong data.

Quantisation recipe of every configuration (K, V ~ N(0, sigma), per-tensor
scale amax/448, round-to-nearest-even into E4M3, saturated to +-448) is done
with ``torch.float8_e4m3fn`` casts, a library routine; the decode side (E4M3 ->
real) lives separately in the oracle and in the CUDA kernels.

Pool slots that the decode must not read (tokens before the sliding-window
start, tokens past ``seq_len`` in a sequence's last page, the spare pages) are
filled with the E4M3 NaN code 0x7F when ``fill="nan"`` (the default), so any
leak shows up as NaN in the result.  ``fill="data"`` writes ordinary quantised
N(0, sigma) samples there instead.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import List, Optional, Sequence

import numpy as np
import torch

E4M3_NAN_CODE = 0x7F
E4M3_MAX = 448.0

# Generation is chunked with spawned child seeds so the stream does not depend
# on how many threads draw it.
_CHUNK = 1 << 22


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    block_tokens: int
    num_blocks: int
    max_blocks: int
    q: np.ndarray            # uint16 [B, Hq, D], or [B, q_len, Hq, D] (bf16 bit patterns)
    k_cache: np.ndarray      # uint8  [num_blocks, block_tokens, Hkv, D]
    v_cache: np.ndarray      # uint8  [num_blocks, block_tokens, Hkv, D]
    block_table: np.ndarray  # int32  [B, max_blocks]
    seq_lens: np.ndarray     # int32  [B]
    k_scale: float
    v_scale: float
    sm_scale: float
    window_left: int
    sinks: Optional[np.ndarray]  # float32 [Hq] or None
    # Dense per-sequence copies of the stored codes, token order, [L_b, Hkv, D];
    # kept only when requested (small cases) for brute-force checks.
    k_dense: Optional[List[np.ndarray]] = None
    v_dense: Optional[List[np.ndarray]] = None
    # Query tokens per sequence (the newest q_len positions, causal).
    q_len: int = 1
    # "e4m3" (k_cache / v_cache) or "nvfp4": then kv_cache holds the pages,
    # uint8 [num_blocks, page_bytes], each [K data | K scales | V data | V scales]
    # with data [Hkv][bt][D/2] (E2M1 pairs) and scales [Hkv][bt][D/16] (E4M3).
    kv_format: str = "e4m3"
    kv_cache: Optional[np.ndarray] = None

    @property
    def groups(self) -> int:
        return self.Hq // self.Hkv

    def attended(self) -> np.ndarray:
        """Number of keys each sequence's queries attend together (window-capped)."""
        L = self.seq_lens.astype(np.int64)
        if self.window_left >= 0:
            return np.minimum(L, self.window_left + self.q_len)
        return L

    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode call must read (NVFP4: the E2M1 data
        and the E4M3 block scales, D/2 + D/16 bytes per token and head and side)."""
        per = self.D if self.kv_format == "e4m3" else self.D // 2 + self.D // 16
        return int(self.attended().sum()) * self.Hkv * per * 2

    def io_bytes(self) -> int:
        """q in, out and lse out: B*q_len*Hq*(2D + 2D + 4) bytes."""
        return self.B * self.q_len * self.Hq * (2 * self.D + 2 * self.D + 4)


# The five synthetic workloads (shapes, distributions and scales as specified
# for this op).  Seeds 0..4 in this order.
CONFIGS = {
    "tiny": dict(B=2, Hq=8, Hkv=2, D=128, block_tokens=16, lens=("fixed", [37, 300]),
                 sm_scale=1.0 / math.sqrt(128), window_left=-1, sinks=False, sigma=1.0, seed=0),
    "llama3_8b": dict(B=32, Hq=32, Hkv=8, D=128, block_tokens=16, lens=("uniform", 1024, 8192),
                      sm_scale=1.0 / math.sqrt(128), window_left=-1, sinks=False, sigma=1.0, seed=1),
    "swa_sinks": dict(B=64, Hq=64, Hkv=8, D=64, block_tokens=16, lens=("uniform", 2048, 16384),
                      sm_scale=0.125, window_left=128, sinks=True, sigma=1.0, seed=2),
    "long_context": dict(B=4, Hq=32, Hkv=8, D=128, block_tokens=64, lens=("fixed", [131072] * 4),
                         sm_scale=1.0 / math.sqrt(128), window_left=-1, sinks=False, sigma=1.0, seed=3),
    "large_mixed": dict(B=256, Hq=64, Hkv=8, D=128, block_tokens=32,
                        lens=("lognormal", 2048.0, 1.0, 1, 32768),
                        sm_scale=0.1, window_left=4096, sinks=True, sigma=2.0, seed=4),
}

CONFIG_ORDER = ["tiny", "llama3_8b", "swa_sinks", "long_context", "large_mixed"]


def describe(name: str) -> str:
    c = CONFIGS[name]
    return (f"{name}: B={c['B']} Hq={c['Hq']} Hkv={c['Hkv']} D={c['D']} "
            f"block_tokens={c['block_tokens']} lens={c['lens']} window_left={c['window_left']} "
            f"sinks={c['sinks']} sm_scale={c['sm_scale']:.6g} sigma={c['sigma']}")


def _draw_lens(rng: np.random.Generator, B: int, spec) -> np.ndarray:
    kind = spec[0]
    if kind == "fixed":
        lens = np.asarray(spec[1], dtype=np.int64)
        assert lens.shape == (B,)
    elif kind == "uniform":
        lens = rng.integers(spec[1], spec[2] + 1, size=B, dtype=np.int64)
    elif kind == "lognormal":
        median, sigma, lo, hi = spec[1], spec[2], spec[3], spec[4]
        z = rng.standard_normal(B)
        lens = np.clip(np.rint(np.exp(math.log(median) + sigma * z)), lo, hi).astype(np.int64)
    else:
        raise ValueError(spec)
    return lens.astype(np.int32)


def _normal_f32(seed_seq: np.random.SeedSequence, n: int, sigma: float, threads: int = 0) -> np.ndarray:
    """n samples of N(0, sigma) as float32, drawn in fixed chunks of child seeds."""
    out = np.empty(n, dtype=np.float32)
    nchunks = max(1, -(-n // _CHUNK))
    kids = seed_seq.spawn(nchunks)

    def fill(i):
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        np.random.default_rng(kids[i]).standard_normal(out=out[lo:hi], dtype=np.float32)

    if nchunks == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(threads or min(16, nchunks)) as ex:
            list(ex.map(fill, range(nchunks)))
    if sigma != 1.0:
        out *= np.float32(sigma)
    return out


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def quantize_e4m3(x: np.ndarray, scale: float) -> np.ndarray:
    """codes = RNE_e4m3(clamp(x / scale, +-448)); the generator's encoder (torch cast)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = (t / torch.tensor(scale, dtype=torch.float32)).clamp_(-E4M3_MAX, E4M3_MAX)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def make_custom(*, B: int, Hq: int, Hkv: int, D: int, block_tokens: int,
                seq_lens: Sequence[int], window_left: int = -1, sinks: bool = False,
                sm_scale: Optional[float] = None, sigma: float = 1.0, seed: int = 0,
                spare_blocks: int = 16, max_blocks: Optional[int] = None,
                fill: str = "nan", keep_dense: bool = False, name: str = "custom",
                q_sigma: float = 1.0, sink_sigma: float = 1.0, q_len: int = 1) -> Workload:
    """Build one decode step of the given shape (see module docstring).  With
    q_len > 1 each sequence has q_len query tokens (q is [B, q_len, Hq, D]) and
    the stored range covers every query's window."""
    assert Hq % Hkv == 0 and fill in ("nan", "data")
    lens = np.asarray(seq_lens, dtype=np.int64)
    assert lens.shape == (B,) and (lens >= 0).all()
    bt = block_tokens
    root = np.random.SeedSequence(seed)
    s_perm, s_q, s_k, s_v, s_fill_k, s_fill_v, s_sink = root.spawn(7)

    pages = -(-lens // bt)
    if max_blocks is None:
        max_blocks = int(max(1, pages.max() if B else 1))
    assert (pages <= max_blocks).all()
    num_blocks = int(pages.sum()) + spare_blocks
    num_blocks = max(num_blocks, 1)
    perm = np.random.default_rng(s_perm).permutation(num_blocks).astype(np.int32)
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, :pages[b]] = perm[off:off + pages[b]]
        off += int(pages[b])

    assert q_len >= 1
    if q_len == 1:
        q = _to_bf16_bits(_normal_f32(s_q, B * Hq * D, q_sigma).reshape(B, Hq, D))
    else:
        q = _to_bf16_bits(_normal_f32(s_q, B * q_len * Hq * D, q_sigma).reshape(B, q_len, Hq, D))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)

    W = window_left
    starts = np.maximum(0, lens - q_len - W) if W >= 0 else np.zeros_like(lens)
    n_att = lens - starts
    tot = int(n_att.sum())
    row = Hkv * D

    # Flat row index (physical page * bt + in-page offset) of every attended token.
    tok_rows = []
    for b in range(B):
        j = np.arange(starts[b], lens[b], dtype=np.int64)
        tok_rows.append(table[b, j // bt].astype(np.int64) * bt + j % bt)
    tok_rows = np.concatenate(tok_rows) if B else np.zeros(0, np.int64)

    def build(seed_seq, seed_fill):
        x = _normal_f32(seed_seq, tot * row, sigma)
        amax = float(np.abs(x).max()) if tot else 1.0
        scale = float(np.float32(amax / E4M3_MAX)) if amax > 0 else 1.0
        codes = quantize_e4m3(x, scale).reshape(tot, Hkv, D)
        del x
        cache = np.full((num_blocks * bt, Hkv, D), E4M3_NAN_CODE, dtype=np.uint8)
        if fill == "data":
            filler = quantize_e4m3(_normal_f32(seed_fill, num_blocks * bt * row, sigma), scale)
            cache[:] = filler.reshape(num_blocks * bt, Hkv, D)
        cache[tok_rows] = codes
        return cache.reshape(num_blocks, bt, Hkv, D), scale

    k_cache, k_scale = build(s_k, s_fill_k)
    v_cache, v_scale = build(s_v, s_fill_v)

    sinks_arr = None
    if sinks:
        sinks_arr = _normal_f32(s_sink, Hq, sink_sigma)

    k_dense = v_dense = None
    if keep_dense:
        k_dense, v_dense = [], []
        kf = k_cache.reshape(num_blocks * bt, Hkv, D)
        vf = v_cache.reshape(num_blocks * bt, Hkv, D)
        for b in range(B):
            j = np.arange(0, lens[b], dtype=np.int64)
            rows = table[b, j // bt].astype(np.int64) * bt + j % bt
            k_dense.append(kf[rows].copy())
            v_dense.append(vf[rows].copy())

    return Workload(name=name, seed=seed, B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt,
                    num_blocks=num_blocks, max_blocks=max_blocks, q=q, k_cache=k_cache,
                    v_cache=v_cache, block_table=table, seq_lens=lens.astype(np.int32),
                    k_scale=k_scale, v_scale=v_scale, sm_scale=float(np.float32(sm_scale)),
                    window_left=int(W), sinks=sinks_arr, k_dense=k_dense, v_dense=v_dense,
                    q_len=int(q_len))


def make_workload(name: str, *, seed: Optional[int] = None, fill: str = "nan",
                  keep_dense: bool = False, B: Optional[int] = None,
                  q_len: int = 1) -> Workload:
    """One of the five named workloads.  ``B`` may shrink the batch (keeps the
    first B sequences' length draws); ``q_len`` > 1 gives each sequence that
    many query tokens (speculative decode of the same shape)."""
    c = CONFIGS[name]
    s = c["seed"] if seed is None else seed
    rng = np.random.default_rng(np.random.SeedSequence([s, 0x5EED]))
    lens = _draw_lens(rng, c["B"], c["lens"])
    nb = c["B"] if B is None else B
    lens = lens[:nb]
    bt = c["block_tokens"]
    # The pool's table width is the configuration's maximum length in pages.
    spec = c["lens"]
    if spec[0] == "fixed":
        max_len = max(spec[1])
    elif spec[0] == "uniform":
        max_len = spec[2]
    else:
        max_len = spec[4]
    max_blocks = -(-max_len // bt)
    return make_custom(B=nb, Hq=c["Hq"], Hkv=c["Hkv"], D=c["D"], block_tokens=bt,
                       seq_lens=lens, window_left=c["window_left"], sinks=c["sinks"],
                       sm_scale=c["sm_scale"], sigma=c["sigma"], seed=s, fill=fill,
                       keep_dense=keep_dense, max_blocks=max_blocks, name=name, q_len=q_len)


# ------------------------------------------------------------------ NVFP4 --

# Magnitude distribution of the synthetic E2M1 codes (values 0, 0.5, 1, 1.5,
# 2, 3, 4, 6): a bell shape like block-scaled normal data, in 1/128 steps.
NVFP4_CODE_WEIGHTS = (12, 22, 22, 19, 17, 18, 12, 6)
E4M3_SF_EXPONENTS = (5, 6, 7, 8)   # block scales 0.25 .. 3.75


def _nibble_lut() -> np.ndarray:
    """Random byte -> E2M1 code: bits 0..6 pick the magnitude by the weights,
    bit 7 the sign."""
    mag = np.repeat(np.arange(8, dtype=np.uint8), NVFP4_CODE_WEIGHTS)
    assert mag.size == 128
    lut = np.empty(256, dtype=np.uint8)
    lut[:128] = mag
    lut[128:] = mag | 0x8
    return lut


def _random_nvfp4_bytes(rng: np.random.Generator, n: int) -> np.ndarray:
    """n bytes of two independent synthetic E2M1 codes each."""
    lut = _nibble_lut()
    r = rng.integers(0, 1 << 16, size=n, dtype=np.uint16)
    return (lut[r & 0xFF] | (lut[r >> 8] << 4)).astype(np.uint8)


def _random_sf_codes(rng: np.random.Generator, n: int) -> np.ndarray:
    e = rng.choice(np.asarray(E4M3_SF_EXPONENTS, dtype=np.uint8), size=n)
    m = rng.integers(0, 8, size=n, dtype=np.uint8)
    return ((e << 3) | m).astype(np.uint8)


def nvfp4_page_bytes(Hkv: int, bt: int, D: int) -> int:
    return 2 * Hkv * bt * (D // 2 + D // 16)


def make_custom_nvfp4(*, B: int, Hq: int, Hkv: int, D: int, block_tokens: int,
                      seq_lens: Sequence[int], window_left: int = -1, sinks: bool = False,
                      sm_scale: Optional[float] = None, seed: int = 0, spare_blocks: int = 16,
                      max_blocks: Optional[int] = None, name: str = "custom-nvfp4",
                      q_sigma: float = 1.0, sink_sigma: float = 1.0, q_len: int = 1,
                      k_scale: float = 0.2, v_scale: float = 0.2) -> Workload:
    """One decode step over NVFP4 pages (head-major, the page layout of
    ``Workload.kv_cache``).  The E2M1 codes follow ``NVFP4_CODE_WEIGHTS`` with
    random signs and the block scales are E4M3 values 0.25 .. 3.75; no
    quantisation arithmetic is involved.  Every block scale of a slot the decode
    must not read (before the window, past seq_len, spare pages) is the E4M3 NaN
    code, so a leak shows up as NaN."""
    assert Hq % Hkv == 0 and D % 16 == 0
    lens = np.asarray(seq_lens, dtype=np.int64)
    assert lens.shape == (B,) and (lens >= 0).all()
    bt = block_tokens
    root = np.random.SeedSequence([seed, 0xF4])
    s_perm, s_q, s_data, s_sf, s_sink = root.spawn(5)
    pages = -(-lens // bt)
    if max_blocks is None:
        max_blocks = int(max(1, pages.max() if B else 1))
    assert (pages <= max_blocks).all()
    num_blocks = max(int(pages.sum()) + spare_blocks, 1)
    perm = np.random.default_rng(s_perm).permutation(num_blocks).astype(np.int32)
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, :pages[b]] = perm[off:off + pages[b]]
        off += int(pages[b])
    shape = (B, Hq, D) if q_len == 1 else (B, q_len, Hq, D)
    q = _to_bf16_bits(_normal_f32(s_q, int(np.prod(shape)), q_sigma).reshape(shape))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)

    data_b, sf_b = Hkv * bt * D // 2, Hkv * bt * D // 16
    page_bytes = 2 * (data_b + sf_b)
    kv = np.empty((num_blocks, page_bytes), dtype=np.uint8)
    rd, rs = np.random.default_rng(s_data), np.random.default_rng(s_sf)
    for side in range(2):
        base = side * (data_b + sf_b)
        kv[:, base:base + data_b] = _random_nvfp4_bytes(rd, num_blocks * data_b).reshape(
            num_blocks, data_b)
        kv[:, base + data_b:base + data_b + sf_b] = _random_sf_codes(
            rs, num_blocks * sf_b).reshape(num_blocks, sf_b)
    # slots the decode must not read: NaN block scales
    W = int(window_left)
    starts = np.maximum(0, lens - q_len - W) if W >= 0 else np.zeros_like(lens)
    valid = np.zeros((num_blocks, bt), dtype=bool)
    for b in range(B):
        j = np.arange(starts[b], lens[b], dtype=np.int64)
        valid[table[b, j // bt], j % bt] = True
    for side in range(2):
        base = side * (data_b + sf_b) + data_b
        sf = kv[:, base:base + sf_b].reshape(num_blocks, Hkv, bt, D // 16)
        sf[np.broadcast_to(~valid[:, None, :, None], sf.shape)] = E4M3_NAN_CODE
    sinks_arr = _normal_f32(s_sink, Hq, sink_sigma) if sinks else None
    return Workload(name=name, seed=seed, B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt,
                    num_blocks=num_blocks, max_blocks=max_blocks, q=q, k_cache=None,
                    v_cache=None, block_table=table, seq_lens=lens.astype(np.int32),
                    k_scale=float(np.float32(k_scale)), v_scale=float(np.float32(v_scale)),
                    sm_scale=float(np.float32(sm_scale)), window_left=W, sinks=sinks_arr,
                    q_len=int(q_len), kv_format="nvfp4", kv_cache=kv)


def make_workload_nvfp4(name: str, *, seed: Optional[int] = None, B: Optional[int] = None,
                        q_len: int = 1) -> Workload:
    """A named workload's shape, lengths, window and sinks over NVFP4 pages."""
    c = CONFIGS[name]
    s = c["seed"] if seed is None else seed
    rng = np.random.default_rng(np.random.SeedSequence([s, 0x5EED]))
    lens = _draw_lens(rng, c["B"], c["lens"])
    nb = c["B"] if B is None else B
    lens = lens[:nb]
    bt = c["block_tokens"]
    spec = c["lens"]
    max_len = max(spec[1]) if spec[0] == "fixed" else (spec[2] if spec[0] == "uniform" else spec[4])
    return make_custom_nvfp4(B=nb, Hq=c["Hq"], Hkv=c["Hkv"], D=c["D"], block_tokens=bt,
                             seq_lens=lens, window_left=c["window_left"], sinks=c["sinks"],
                             sm_scale=c["sm_scale"], seed=s, max_blocks=-(-max_len // bt),
                             name=name + "-nvfp4", q_len=q_len)
