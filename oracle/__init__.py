"""CPU oracle for paged FP8 (E4M3) decode attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the bench's CPU-baseline /
reference leg may import this package.  The CUDA product path never calls it
and shares no code with it.

The arithmetic lives in ``fpd_oracle.c`` (plain C, fp64, one (sequence, head)
row at a time, the definition written out).  This module builds that file with
gcc into ``libfpd_oracle.so`` next to it and exposes it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fpd_oracle.c")
_LIB = os.path.join(_HERE, "libfpd_oracle.so")
_lock = threading.Lock()
_lib = None


def build(src: str = _SRC, out: str = _LIB, extra_flags: Sequence[str] = ()) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math: IEEE fp64)."""
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", *extra_flags,
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    u8p = ctypes.POINTER(ctypes.c_uint8)
    lib.fpd_oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.fpd_oracle_e4m3_to_f64.restype = ctypes.c_double
    lib.fpd_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.fpd_oracle_bf16_to_f64.restype = ctypes.c_double
    vp = ctypes.c_void_p
    ci, cd = ctypes.c_int, ctypes.c_double
    lib.fpd_oracle_decode.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci,
                                      cd, cd, cd, ci, vp, vp, vp, vp, ci, ci]
    lib.fpd_oracle_decode.restype = ci
    lib.fpd_oracle_decode_q.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci,
                                        cd, cd, cd, ci, vp, vp, vp, vp, ci, ci]
    lib.fpd_oracle_decode_q.restype = ci
    lib.fpd_oracle_decode_x.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, ci,
                                        cd, cd, cd, ci, vp, vp, vp, vp, ci, ci, ci, ci]
    lib.fpd_oracle_decode_x.restype = ci
    lib.fpd_oracle_merge.argtypes = [vp, vp, ci, ctypes.c_long, ci, ci, vp, vp, vp]
    lib.fpd_oracle_merge.restype = None
    lib.fpd_oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.fpd_oracle_f16_to_f64.restype = ctypes.c_double
    lib.fpd_oracle_e2m1_to_f64.argtypes = [ctypes.c_uint8]
    lib.fpd_oracle_e2m1_to_f64.restype = ctypes.c_double
    lib.fpd_oracle_f64_to_e2m1.argtypes = [ctypes.c_double]
    lib.fpd_oracle_f64_to_e2m1.restype = ctypes.c_uint8
    cl = ctypes.c_long
    lib.fpd_oracle_decode_nvfp4.argtypes = [vp, vp, vp, vp, vp, cl, cl, vp, vp, ci, ci, ci, ci, ci,
                                            ci, ci, ci, cd, cd, cd, ci, vp, vp, vp, vp, ci, ci,
                                            ci]
    lib.fpd_oracle_decode_nvfp4.restype = ci
    lib.fpd_oracle_cache_write_nvfp4.argtypes = [vp, vp, vp, ci, ci, ci, cl, cl, ctypes.c_float,
                                                 ctypes.c_float, vp, vp, vp, vp, cl, cl, ci, ci]
    lib.fpd_oracle_cache_write_nvfp4.restype = ci
    lib.fpd_oracle_f64_to_e4m3.argtypes = [ctypes.c_double]
    lib.fpd_oracle_f64_to_e4m3.restype = ctypes.c_uint8
    lib.fpd_oracle_cache_write.argtypes = [vp, vp, vp, ci, ci, ci, ctypes.c_long, ctypes.c_long,
                                           ctypes.c_float, ctypes.c_float, vp, vp, ci, ci]
    lib.fpd_oracle_cache_write.restype = ci
    lib.fpd_oracle_cache_write_x.argtypes = lib.fpd_oracle_cache_write.argtypes + [ci]
    lib.fpd_oracle_cache_write_x.restype = ci
    del u8p
    return lib


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
            if stale:
                build()
            _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def e4m3_to_f64(code: int, lib=None) -> float:
    return (lib or load()).fpd_oracle_e4m3_to_f64(int(code))


def bf16_to_f64(bits: int, lib=None) -> float:
    return (lib or load()).fpd_oracle_bf16_to_f64(int(bits))


def f16_to_f64(bits: int, lib=None) -> float:
    return (lib or load()).fpd_oracle_f16_to_f64(int(bits))


def f64_to_e4m3(x: float, lib=None) -> int:
    """Nearest E4M3 code, ties to even, saturating at +-448 (NaN -> S.1111.111)."""
    return int((lib or load()).fpd_oracle_f64_to_e4m3(float(x)))


def cache_write(key, value, slot_mapping, k_cache, v_cache, *, k_scale, v_scale, lib=None,
                kv_layout="NHD") -> int:
    """FP8 KV-cache write into ``k_cache``/``v_cache`` (uint8 [num_blocks, bt, Hkv, D],
    or [num_blocks, Hkv, bt, D] with ``kv_layout="HND"``; modified in place) of
    bf16 ``key``/``value`` (uint16 bits [num_tokens, Hkv, D], any token stride) at
    ``slot_mapping`` (int64 [num_tokens], negative = skip).  Returns the number
    of out-of-range slots (skipped)."""
    lib = lib or load()
    assert key.dtype == np.uint16 and value.dtype == np.uint16
    assert k_cache.dtype == np.uint8 and k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert kv_layout in ("NHD", "HND")
    if kv_layout == "HND":
        num_blocks, Hkv, bt, D = k_cache.shape
    else:
        num_blocks, bt, Hkv, D = k_cache.shape
    T = key.shape[0]
    assert key.shape[1:] == (Hkv, D) and value.shape[1:] == (Hkv, D)
    for a in (key, value):
        assert a.strides[2] == 2 and a.strides[1] == 2 * D, "rows must be contiguous per token"
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert slot_mapping.shape == (T,)
    st = lib.fpd_oracle_cache_write_x(key.ctypes.data_as(ctypes.c_void_p),
                                      value.ctypes.data_as(ctypes.c_void_p), _ptr(slot_mapping),
                                      T, Hkv, D, key.strides[0] // 2, value.strides[0] // 2,
                                      float(k_scale), float(v_scale), _ptr(k_cache),
                                      _ptr(v_cache), num_blocks, bt,
                                      1 if kv_layout == "HND" else 0)
    if st < 0:
        raise ValueError("oracle rejected the cache-write arguments")
    return st


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def decode(q, k_cache, v_cache, block_table, seq_lens, *, k_scale, v_scale, sm_scale,
           window_left=-1, sinks=None, rows=None, threads=None, lib=None, q_dtype="bf16",
           kv_layout="NHD") -> Tuple[np.ndarray, np.ndarray]:
    """fp64 decode attention.

    Arrays are numpy: q uint16 (bf16 bits, or fp16 bits with ``q_dtype="f16"``)
    [B,Hq,D], or [B,q_len,Hq,D] for q_len query tokens per sequence (positions
    L - q_len .. L - 1, causal); k/v_cache uint8 E4M3 codes
    [num_blocks, bt, Hkv, D] (``kv_layout="HND"``: [num_blocks, Hkv, bt, D]); block_table int32
    [B, max_blocks]; seq_lens int32 [B]; sinks float32 [Hq] or None.  ``rows``
    optionally lists flat ``(b * q_len + i) * Hq + h`` rows to compute (others
    are left NaN).  Returns (out float64 [B, (q_len,) Hq, D], lse float64
    [B, (q_len,) Hq]) with q's leading shape.
    """
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint8)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint8)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    lead = q.shape[:-2]
    if q.ndim == 3:
        B, Hq, D = q.shape
        Q = 1
    else:
        B, Q, Hq, D = q.shape
    assert q_dtype in ("bf16", "f16") and kv_layout in ("NHD", "HND")
    if kv_layout == "HND":
        num_blocks, Hkv, bt, D2 = k_cache.shape
    else:
        num_blocks, bt, Hkv, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape
    assert block_table.shape[0] == B and seq_lens.shape == (B,)
    max_blocks = block_table.shape[1]
    if sinks is not None:
        sinks = np.ascontiguousarray(sinks, dtype=np.float32)
        assert sinks.shape == (Hq,)
    out = np.full(lead + (Hq, D), np.nan, dtype=np.float64)
    lse = np.full(lead + (Hq,), np.nan, dtype=np.float64)
    rows_arr = None
    n_rows = 0
    if rows is not None:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int32)
        n_rows = int(rows_arr.size)
    if threads is None:
        threads = os.cpu_count() or 1
    st = lib.fpd_oracle_decode_x(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                 _ptr(seq_lens), B, Q, Hq, Hkv, D, num_blocks, bt, max_blocks,
                                 float(k_scale), float(v_scale), float(sm_scale),
                                 int(window_left), _ptr(sinks), _ptr(out), _ptr(lse),
                                 _ptr(rows_arr), n_rows, int(threads),
                                 1 if q_dtype == "f16" else 0, 1 if kv_layout == "HND" else 0)
    if st != 0:
        raise ValueError(f"oracle rejected the inputs (status {st})")
    return out, lse


def decode_workload(wl, rows=None, threads=None, lib=None, window_left=None, sinks="keep"):
    """Oracle on a ``workloads.Workload``."""
    return decode(wl.q, wl.k_cache, wl.v_cache, wl.block_table, wl.seq_lens,
                  k_scale=wl.k_scale, v_scale=wl.v_scale, sm_scale=wl.sm_scale,
                  window_left=wl.window_left if window_left is None else window_left,
                  sinks=wl.sinks if isinstance(sinks, str) else sinks,
                  rows=rows, threads=threads, lib=lib)


# ----------------------------------------------------------------- NVFP4 --

def e2m1_to_f64(code: int, lib=None) -> float:
    return (lib or load()).fpd_oracle_e2m1_to_f64(int(code))


def f64_to_e2m1(x: float, lib=None) -> int:
    """Nearest E2M1 code, ties to even, saturating at +-6."""
    return int((lib or load()).fpd_oracle_f64_to_e2m1(float(x)))


def nvfp4_page_layout(Hkv: int, bt: int, D: int) -> dict:
    """Byte offsets inside one NVFP4 page [K data | K scales | V data | V scales]
    (data [Hkv][bt][D/2], scales [Hkv][bt][D/16] per side) and its size."""
    data = Hkv * bt * D // 2
    sf = Hkv * bt * D // 16
    return dict(k_data=0, k_sf=data, v_data=data + sf, v_sf=2 * data + sf,
                page_bytes=2 * (data + sf))


def _page_ptrs(kv_cache, Hkv, bt, D):
    lay = nvfp4_page_layout(Hkv, bt, D)
    assert kv_cache.dtype == np.uint8 and kv_cache.flags.c_contiguous
    assert kv_cache.ndim == 2 and kv_cache.shape[1] == lay["page_bytes"]
    base = kv_cache.ctypes.data
    return [ctypes.c_void_p(base + lay[k]) for k in ("k_data", "k_sf", "v_data", "v_sf")], \
        lay["page_bytes"]


def decode_nvfp4(q, kv_cache, block_table, seq_lens, *, Hkv, block_tokens, k_scale, v_scale,
                 sm_scale, window_left=-1, sinks=None, rows=None, threads=None, lib=None,
                 q_dtype="bf16", regions=None) -> Tuple[np.ndarray, np.ndarray]:
    """fp64 decode attention over NVFP4 pages.  ``kv_cache`` is uint8
    [num_blocks, page_bytes] with each page laid out as ``nvfp4_page_layout``;
    or ``kv_cache`` None and ``regions`` = (k_data, k_sf, v_data, v_sf), four
    contiguous uint8 arrays [num_blocks, Hkv, bt, D/2] and [num_blocks, Hkv, bt,
    D/16] (separate page strides for data and scales).  Other arguments as
    ``decode``."""
    lib = lib or load()
    q = np.ascontiguousarray(q, dtype=np.uint16)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    lead = q.shape[:-2]
    if q.ndim == 3:
        B, Hq, D = q.shape
        Q = 1
    else:
        B, Q, Hq, D = q.shape
    if regions is None:
        ptrs, page_bytes = _page_ptrs(kv_cache, Hkv, block_tokens, D)
        data_stride = sf_stride = page_bytes
        num_blocks = kv_cache.shape[0]
    else:
        kd, ks, vd, vs = regions
        num_blocks = kd.shape[0]
        for a, last in ((kd, D // 2), (ks, D // 16), (vd, D // 2), (vs, D // 16)):
            assert a.dtype == np.uint8 and a.flags.c_contiguous
            assert a.shape == (num_blocks, Hkv, block_tokens, last)
        ptrs = [ctypes.c_void_p(a.ctypes.data) for a in (kd, ks, vd, vs)]
        data_stride = Hkv * block_tokens * D // 2
        sf_stride = Hkv * block_tokens * D // 16
    max_blocks = block_table.shape[1]
    if sinks is not None:
        sinks = np.ascontiguousarray(sinks, dtype=np.float32)
    out = np.full(lead + (Hq, D), np.nan, dtype=np.float64)
    lse = np.full(lead + (Hq,), np.nan, dtype=np.float64)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n_rows = 0 if rows_arr is None else int(rows_arr.size)
    st = lib.fpd_oracle_decode_nvfp4(_ptr(q), ptrs[0], ptrs[1], ptrs[2], ptrs[3], data_stride,
                                     sf_stride, _ptr(block_table), _ptr(seq_lens), B, Q, Hq,
                                     Hkv, D, num_blocks, block_tokens, max_blocks,
                                     float(k_scale), float(v_scale), float(sm_scale),
                                     int(window_left), _ptr(sinks), _ptr(out), _ptr(lse),
                                     _ptr(rows_arr), n_rows, int(threads or os.cpu_count() or 1),
                                     1 if q_dtype == "f16" else 0)
    if st != 0:
        raise ValueError(f"oracle rejected the inputs (status {st})")
    return out, lse


def decode_nvfp4_workload(wl, rows=None, threads=None, lib=None):
    """Oracle on an NVFP4 ``workloads.Workload`` (``wl.kv_cache`` set)."""
    return decode_nvfp4(wl.q, wl.kv_cache, wl.block_table, wl.seq_lens, Hkv=wl.Hkv,
                        block_tokens=wl.block_tokens, k_scale=wl.k_scale, v_scale=wl.v_scale,
                        sm_scale=wl.sm_scale, window_left=wl.window_left, sinks=wl.sinks,
                        rows=rows, threads=threads, lib=lib)


def cache_write_nvfp4(key, value, slot_mapping, kv_cache, *, block_tokens, k_scale, v_scale,
                      lib=None) -> int:
    """NVFP4 KV-cache write of bf16 ``key``/``value`` (uint16 bits
    [num_tokens, Hkv, D], any token stride) into ``kv_cache`` (uint8
    [num_blocks, page_bytes], ``nvfp4_page_layout``; modified in place) at
    ``slot_mapping`` (negative = skip).  Returns the count of out-of-range slots."""
    lib = lib or load()
    T, Hkv, D = key.shape
    for a in (key, value):
        assert a.dtype == np.uint16 and a.strides[2] == 2 and a.strides[1] == 2 * D
    ptrs, page_bytes = _page_ptrs(kv_cache, Hkv, block_tokens, D)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    st = lib.fpd_oracle_cache_write_nvfp4(key.ctypes.data_as(ctypes.c_void_p),
                                          value.ctypes.data_as(ctypes.c_void_p),
                                          _ptr(slot_mapping), T, Hkv, D, key.strides[0] // 2,
                                          value.strides[0] // 2, float(k_scale), float(v_scale),
                                          ptrs[0], ptrs[1], ptrs[2], ptrs[3], page_bytes,
                                          page_bytes, kv_cache.shape[0], block_tokens)
    if st < 0:
        raise ValueError("oracle rejected the NVFP4 cache-write arguments")
    return st


def merge(o_parts, lse_parts, Hq: int, sinks=None, lib=None):
    """The merge of R partial results of disjoint key sets (``fpd_oracle_merge``):
    ``o_parts`` [R, *lead, Hq, D] and ``lse_parts`` [R, *lead, Hq] (natural log,
    -inf for a part with no key), ``sinks`` [Hq] or None.  Returns fp64
    (out [*lead, Hq, D], lse [*lead, Hq])."""
    lib = lib or load()
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    l = np.ascontiguousarray(lse_parts, dtype=np.float64)
    R, D = o.shape[0], o.shape[-1]
    lead = o.shape[1:-1]
    rows = int(np.prod(lead))
    if l.shape != (R,) + tuple(lead) or lead[-1] != Hq:
        raise ValueError("o_parts / lse_parts shapes disagree")
    s = None if sinks is None else np.ascontiguousarray(sinks, dtype=np.float32)
    out = np.zeros(tuple(lead) + (D,), dtype=np.float64)
    lse = np.zeros(tuple(lead), dtype=np.float64)
    lib.fpd_oracle_merge(_ptr(o), _ptr(l), R, rows, D, Hq, _ptr(s), _ptr(out), _ptr(lse))
    return out, lse
