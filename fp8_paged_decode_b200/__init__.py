"""Paged E4M3 (FP8) decode attention for B200 (sm_100a).

A thin ctypes binding of ``libfp8_paged_decode.so`` (the C ABI declared in
``include/fp8_paged_decode.h``).  The functions carry the C names and only
marshal arguments: torch tensors become raw device pointers and the current
CUDA stream is passed along.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback.  If the shared library is
missing, calling any function raises immediately (build it with
``python -m fp8_paged_decode_b200.build``).

Layouts (all contiguous, on one CUDA device):
  q            bfloat16 [B, Hq, D]
  k_cache      uint8 or float8_e4m3fn [num_blocks, block_tokens, Hkv, D]
  v_cache      same as k_cache
  block_table  int32 [B, max_blocks]
  seq_lens     int32 [B]
  sinks        float32 [Hq] or None
  out          bfloat16 [B, Hq, D]; lse float32 [B, Hq] (optional)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

__all__ = [
    "FPD_OK", "FPD_ERR_INVALID_ARG", "FPD_ERR_UNSUPPORTED", "FPD_ERR_WORKSPACE_TOO_SMALL",
    "FPD_ERR_CUDA", "FPD_DEVERR_SEQ_LEN", "FPD_DEVERR_BLOCK_TABLE", "FPD_DEVERR_TIMEOUT",
    "FpdError", "library_path", "load_library", "fp8_paged_decode_make_plan",
    "fp8_paged_decode_make_plan_qlen", "FPD_MAX_Q_LEN", "FPD_KV_NHD", "FPD_KV_HND",
    "FPD_Q_BF16", "FPD_Q_F16", "fpd_decode_args", "fp8_paged_decode_cache_write_layout",
    "FPD_KV_E4M3", "FPD_KV_NVFP4", "FPD_OUT_BF16", "FPD_OUT_F32", "fp8_paged_decode_cp_merge",
    "fp8_paged_decode_cp_merge_wait",
    "nvfp4_page_layout", "fp8_paged_decode_attention_nvfp4",
    "fp8_paged_decode_cache_write_nvfp4", "fp8_paged_decode_workspace_bytes_args",
    "fp8_paged_decode_plan", "fp8_paged_decode_workspace_bytes",
    "fp8_paged_decode_workspace_bytes_ex", "fp8_paged_decode_attention_profiled",
    "fp8_paged_decode_attention", "fp8_paged_decode_attention_ex",
    "fp8_paged_decode_check_status", "fp8_paged_decode_workspace_init",
    "fp8_paged_decode_cache_write", "fp8_paged_decode_plan_qlen",
    "fp8_paged_decode_workspace_bytes_qlen",
    "fp8_paged_decode_status_string", "fp8_paged_decode_version", "EXPORTED_SYMBOLS",
]

FPD_OK = 0
FPD_ERR_INVALID_ARG = 1
FPD_ERR_UNSUPPORTED = 2
FPD_ERR_WORKSPACE_TOO_SMALL = 3
FPD_ERR_CUDA = 4
FPD_DEVERR_SEQ_LEN = 0x1
FPD_DEVERR_BLOCK_TABLE = 0x2
FPD_DEVERR_TIMEOUT = 0x4
FPD_DEVERR_SLOT = 0x8
FPD_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
FPD_MAX_Q_LEN = 64
FPD_KV_NHD = 0
FPD_KV_HND = 1
FPD_Q_BF16 = 0
FPD_Q_F16 = 1
FPD_KV_E4M3 = 0
FPD_KV_NVFP4 = 1
FPD_OUT_BF16 = 0
FPD_OUT_F32 = 1

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libfp8_paged_decode.so"
_lock = threading.Lock()
_lib = None

# Every entry point declared in include/fp8_paged_decode.h.
EXPORTED_SYMBOLS = (
    "fp8_paged_decode_make_plan",
    "fp8_paged_decode_make_plan_qlen",
    "fp8_paged_decode_plan",
    "fp8_paged_decode_workspace_bytes",
    "fp8_paged_decode_workspace_bytes_ex",
    "fp8_paged_decode_attention",
    "fp8_paged_decode_attention_ex",
    "fp8_paged_decode_attention_profiled",
    "fp8_paged_decode_attention_noalloc",
    "fp8_paged_decode_check_status",
    "fp8_paged_decode_workspace_init",
    "fp8_paged_decode_cache_write",
    "fp8_paged_decode_attention_qlen",
    "fp8_paged_decode_attention_args",
    "fp8_paged_decode_attention_args_profiled",
    "fp8_paged_decode_plan_args",
    "fp8_paged_decode_workspace_bytes_args",
    "fp8_paged_decode_cache_write_layout",
    "fp8_paged_decode_cache_write_nvfp4",
    "fp8_paged_decode_plan_qlen",
    "fp8_paged_decode_workspace_bytes_qlen",
    "fp8_paged_decode_cp_merge",
    "fp8_paged_decode_cp_merge_wait",
    "fp8_paged_decode_status_string",
    "fp8_paged_decode_version",
)


class FpdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)} ({status})")


class fpd_plan(ctypes.Structure):
    _fields_ = [("chunk_pages", ctypes.c_int), ("max_splits", ctypes.c_int),
                ("heads_per_stage", ctypes.c_int), ("stage_tokens", ctypes.c_int),
                ("stages", ctypes.c_int), ("header_slots", ctypes.c_int),
                ("ctas", ctypes.c_int), ("smem_bytes", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t), ("q_per_item", ctypes.c_int),
                ("q_chunks", ctypes.c_int), ("adapt_chunk_pages", ctypes.c_int)]


class fpd_decode_args(ctypes.Structure):
    """Mirror of the C struct fpd_decode_args (field order and types)."""
    _fields_ = [("q", ctypes.c_void_p), ("q_dtype", ctypes.c_int),
                ("q_token_stride", ctypes.c_int64),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("kv_layout", ctypes.c_int),
                ("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("B", ctypes.c_int), ("q_len", ctypes.c_int), ("Hq", ctypes.c_int),
                ("Hkv", ctypes.c_int), ("D", ctypes.c_int), ("num_blocks", ctypes.c_int),
                ("block_tokens", ctypes.c_int), ("max_blocks", ctypes.c_int),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
                ("k_scale_dev", ctypes.c_void_p), ("v_scale_dev", ctypes.c_void_p),
                ("sm_scale", ctypes.c_float), ("window_left", ctypes.c_int),
                ("sinks", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("out_token_stride", ctypes.c_int64), ("lse", ctypes.c_void_p),
                ("chunk_pages_override", ctypes.c_int), ("kv_format", ctypes.c_int),
                ("k_scales", ctypes.c_void_p), ("v_scales", ctypes.c_void_p),
                ("kv_page_stride", ctypes.c_int64), ("sf_page_stride", ctypes.c_int64),
                ("out_dtype", ctypes.c_int),
                ("cp_gather", ctypes.c_void_p), ("cp_flags", ctypes.c_void_p),
                ("cp_ranks", ctypes.c_int), ("cp_rank", ctypes.c_int),
                ("cp_epoch", ctypes.c_uint32), ("cp_block_floats", ctypes.c_int64)]


def library_path() -> str:
    return os.path.join(_PKG, _LIB_NAME)


def _bind(lib):
    ci, cf, cz, vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p
    lib.fp8_paged_decode_make_plan.argtypes = [ci] * 10 + [ctypes.POINTER(fpd_plan)]
    lib.fp8_paged_decode_make_plan.restype = ci
    lib.fp8_paged_decode_make_plan_qlen.argtypes = [ci] * 11 + [ctypes.POINTER(fpd_plan)]
    lib.fp8_paged_decode_make_plan_qlen.restype = ci
    lib.fp8_paged_decode_plan.argtypes = [ci] * 8 + [ctypes.POINTER(fpd_plan)]
    lib.fp8_paged_decode_plan.restype = ci
    lib.fp8_paged_decode_workspace_bytes.argtypes = [ci] * 7
    lib.fp8_paged_decode_workspace_bytes.restype = cz
    lib.fp8_paged_decode_workspace_bytes_ex.argtypes = [ci] * 8
    lib.fp8_paged_decode_workspace_bytes_ex.restype = cz
    attn = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, cf, cf, ci, vp, vp, vp, vp, cz, vp]
    lib.fp8_paged_decode_attention.argtypes = attn
    lib.fp8_paged_decode_attention.restype = ci
    lib.fp8_paged_decode_attention_ex.argtypes = attn + [ci]
    lib.fp8_paged_decode_attention_ex.restype = ci
    lib.fp8_paged_decode_attention_profiled.argtypes = attn[:6] + [ci] + attn[6:] + [ci, vp, vp, vp]
    lib.fp8_paged_decode_attention_profiled.restype = ci
    lib.fp8_paged_decode_attention_noalloc.argtypes = attn[:19] + [vp]
    lib.fp8_paged_decode_attention_qlen.argtypes = attn[:6] + [ci] + attn[6:] + [ci]
    lib.fp8_paged_decode_attention_qlen.restype = ci
    lib.fp8_paged_decode_attention_args.argtypes = [ctypes.POINTER(fpd_decode_args), vp, cz, vp]
    lib.fp8_paged_decode_attention_args.restype = ci
    lib.fp8_paged_decode_attention_args_profiled.argtypes = [ctypes.POINTER(fpd_decode_args), vp,
                                                             cz, vp, vp, vp, vp]
    lib.fp8_paged_decode_attention_args_profiled.restype = ci
    lib.fp8_paged_decode_plan_args.argtypes = [ctypes.POINTER(fpd_decode_args),
                                               ctypes.POINTER(fpd_plan)]
    lib.fp8_paged_decode_plan_args.restype = ci
    lib.fp8_paged_decode_workspace_bytes_args.argtypes = [ctypes.POINTER(fpd_decode_args)]
    lib.fp8_paged_decode_workspace_bytes_args.restype = cz
    i64 = ctypes.c_int64
    lib.fp8_paged_decode_cache_write_nvfp4.argtypes = [vp, vp, vp, ci, ci, ci, i64, i64, cf, cf,
                                                       vp, vp, vp, vp, i64, i64, ci, ci, vp, vp]
    lib.fp8_paged_decode_cache_write_nvfp4.restype = ci
    lib.fp8_paged_decode_cp_merge.argtypes = [vp, ci, i64, i64, ci, ci, vp, vp, i64, vp, vp]
    lib.fp8_paged_decode_cp_merge.restype = ci
    lib.fp8_paged_decode_cp_merge_wait.argtypes = [vp, ci, i64, i64, ci, ci, vp, vp, i64, vp, vp,
                                                   ctypes.c_uint32, ctypes.c_uint64, vp, vp]
    lib.fp8_paged_decode_cp_merge_wait.restype = ci
    lib.fp8_paged_decode_plan_qlen.argtypes = [ci] * 9 + [ctypes.POINTER(fpd_plan)]
    lib.fp8_paged_decode_plan_qlen.restype = ci
    lib.fp8_paged_decode_workspace_bytes_qlen.argtypes = [ci] * 9
    lib.fp8_paged_decode_workspace_bytes_qlen.restype = cz
    lib.fp8_paged_decode_attention_noalloc.restype = ci
    lib.fp8_paged_decode_check_status.argtypes = [vp, vp, ctypes.POINTER(ci), ci]
    lib.fp8_paged_decode_check_status.restype = ci
    lib.fp8_paged_decode_cache_write.argtypes = [vp, vp, vp, ci, ci, ci, ctypes.c_int64,
                                                 ctypes.c_int64, cf, cf, vp, vp, ci, ci, vp, vp]
    lib.fp8_paged_decode_cache_write.restype = ci
    lib.fp8_paged_decode_cache_write_layout.argtypes = (
        lib.fp8_paged_decode_cache_write.argtypes[:14] + [ci, vp, vp])
    lib.fp8_paged_decode_cache_write_layout.restype = ci
    lib.fp8_paged_decode_workspace_init.argtypes = [vp, cz, vp]
    lib.fp8_paged_decode_workspace_init.restype = ci
    lib.fp8_paged_decode_status_string.argtypes = [ci]
    lib.fp8_paged_decode_status_string.restype = ctypes.c_char_p
    lib.fp8_paged_decode_version.argtypes = []
    lib.fp8_paged_decode_version.restype = ctypes.c_char_p
    return lib


def load_library(path: Optional[str] = None):
    """Load the CUDA library (no CUDA call happens at load time)."""
    global _lib
    with _lock:
        if _lib is None or path is not None:
            p = path or library_path()
            if not os.path.exists(p):
                raise RuntimeError(
                    f"{p} is missing: the CUDA extension has not been built "
                    "(python -m fp8_paged_decode_b200.build); there is no fallback path")
            lib = _bind(ctypes.CDLL(p))
            if path is not None:
                return lib
            _lib = lib
    return _lib


def _status_name(status: int) -> str:
    try:
        return load_library().fp8_paged_decode_status_string(int(status)).decode()
    except Exception:  # noqa: BLE001 - naming only
        return f"status {status}"


def _check(status: int, where: str):
    if status != FPD_OK:
        raise FpdError(status, where)


def fp8_paged_decode_status_string(status: int) -> str:
    return load_library().fp8_paged_decode_status_string(int(status)).decode()


def fp8_paged_decode_version() -> str:
    return load_library().fp8_paged_decode_version().decode()


def fp8_paged_decode_make_plan(B, Hq, Hkv, D, block_tokens, max_blocks, window_left, num_sms,
                               ctas_per_sm, chunk_pages_override=0) -> dict:
    """Host-only split planner (no CUDA call)."""
    plan = fpd_plan()
    st = load_library().fp8_paged_decode_make_plan(
        int(B), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks), int(window_left),
        int(num_sms), int(ctas_per_sm), int(chunk_pages_override), ctypes.byref(plan))
    _check(st, "fp8_paged_decode_make_plan")
    return {f: getattr(plan, f) for f, _ in fpd_plan._fields_}


def fp8_paged_decode_make_plan_qlen(B, q_len, Hq, Hkv, D, block_tokens, max_blocks, window_left,
                                    num_sms, ctas_per_sm, chunk_pages_override=0) -> dict:
    """Host-only split planner for q_len query tokens per sequence (no CUDA call)."""
    plan = fpd_plan()
    st = load_library().fp8_paged_decode_make_plan_qlen(
        int(B), int(q_len), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks),
        int(window_left), int(num_sms), int(ctas_per_sm), int(chunk_pages_override),
        ctypes.byref(plan))
    _check(st, "fp8_paged_decode_make_plan_qlen")
    return {f: getattr(plan, f) for f, _ in fpd_plan._fields_}


def fp8_paged_decode_plan(B, Hq, Hkv, D, block_tokens, max_blocks, window_left=-1,
                          chunk_pages_override=0) -> dict:
    """The plan used on the current CUDA device."""
    plan = fpd_plan()
    st = load_library().fp8_paged_decode_plan(
        int(B), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks), int(window_left),
        int(chunk_pages_override), ctypes.byref(plan))
    _check(st, "fp8_paged_decode_plan")
    return {f: getattr(plan, f) for f, _ in fpd_plan._fields_}


def fp8_paged_decode_workspace_bytes(B, Hq, Hkv, D, block_tokens, max_blocks, window_left=-1):
    return int(load_library().fp8_paged_decode_workspace_bytes(
        int(B), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks), int(window_left)))


def fp8_paged_decode_plan_qlen(B, q_len, Hq, Hkv, D, block_tokens, max_blocks, window_left=-1,
                               chunk_pages_override=0) -> dict:
    """The plan used on the current CUDA device for q_len queries per sequence."""
    plan = fpd_plan()
    st = load_library().fp8_paged_decode_plan_qlen(
        int(B), int(q_len), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks),
        int(window_left), int(chunk_pages_override), ctypes.byref(plan))
    _check(st, "fp8_paged_decode_plan_qlen")
    return {f: getattr(plan, f) for f, _ in fpd_plan._fields_}


def fp8_paged_decode_workspace_bytes_qlen(B, q_len, Hq, Hkv, D, block_tokens, max_blocks,
                                          window_left=-1, chunk_pages_override=0) -> int:
    return int(load_library().fp8_paged_decode_workspace_bytes_qlen(
        int(B), int(q_len), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks),
        int(window_left), int(chunk_pages_override)))


def fp8_paged_decode_workspace_bytes_ex(B, Hq, Hkv, D, block_tokens, max_blocks, window_left=-1,
                                        chunk_pages_override=0):
    return int(load_library().fp8_paged_decode_workspace_bytes_ex(
        int(B), int(Hq), int(Hkv), int(D), int(block_tokens), int(max_blocks), int(window_left),
        int(chunk_pages_override)))


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_ptr(t, name, dtypes, shape=None):
    import torch
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype in {dtypes}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _token_rows(t, name, lead, Hq, D):
    """Element stride between consecutive query tokens of a [*lead, Hq, D] view
    whose (Hq, D) rows are contiguous; raises otherwise."""
    if tuple(t.shape) != tuple(lead) + (Hq, D):
        raise ValueError(f"{name} must have shape {tuple(lead) + (Hq, D)}, got {tuple(t.shape)}")
    if (D > 1 and t.stride(-1) != 1) or (Hq > 1 and t.stride(-2) != D):
        raise ValueError(f"{name} must have contiguous [Hq, D] rows")
    if len(lead) == 1:
        return t.stride(0) if lead[0] > 1 else Hq * D
    B, Q = lead
    if Q == 1:
        return t.stride(0) if B > 1 else Hq * D
    tok = t.stride(1)
    if B > 1 and t.stride(0) != Q * tok:
        raise ValueError(f"{name}: the query tokens of all sequences must be equally spaced")
    return tok


def _scale_arg(x, name):
    """(host value, device pointer) of a scale given as a number or a CUDA tensor."""
    import torch
    if isinstance(x, torch.Tensor):
        if not x.is_cuda or x.dtype != torch.float32 or x.numel() != 1:
            raise TypeError(f"{name} as a tensor must be one float32 on the GPU")
        return 1.0, ctypes.c_void_p(x.data_ptr())
    return float(x), None


def fp8_paged_decode_attention(q, k_cache, v_cache, block_table, seq_lens, k_scale, v_scale,
                               sm_scale, window_left=-1, sinks=None, out=None, lse=None,
                               workspace=None, stream=None, chunk_pages_override=0,
                               return_lse=True, kv_layout="NHD", out_dtype="bf16",
                               cp_publish=None):
    """Enqueue one decode call on ``stream`` (default: torch's current stream).

    ``q`` is [B, Hq, D] (one query token per sequence) or [B, q_len, Hq, D]
    (the q_len newest tokens of each sequence, causal), bf16 or fp16; its
    [Hq, D] rows must be contiguous, the tokens may be spaced further apart
    (a slice of a fused QKV buffer).  ``out`` (q's shape, same rule; bf16, or
    float32 for the partial result of a context-parallel rank) and ``lse``
    (float32, contiguous) are allocated when not given, ``out`` with
    ``out_dtype`` ("bf16" or "f32").  ``cp_publish``: the descriptor's
    (cp_gather, cp_flags, cp_ranks, cp_rank, cp_epoch, cp_block_floats) for a
    context-parallel rank whose rows go to every rank's gather buffer (see
    ``cp.CpExchange``); out and lse are then neither allocated nor written and
    (None, None) is returned.  The caches are
    E4M3 (uint8 or float8_e4m3fn) [num_blocks, block_tokens, Hkv, D], or
    [num_blocks, Hkv, block_tokens, D] with ``kv_layout="HND"``.  ``k_scale`` /
    ``v_scale`` are numbers or one-element float32 CUDA tensors (read on the
    GPU when the call runs, e.g. for CUDA-graph replay with new scales).
    Allocates ``out``/``lse``/``workspace`` with torch when not given (pass
    them in to keep a call allocation-free).  Returns ``(out, lse)``.
    """
    import torch
    if q.dim() == 3:
        B, Hq, D = q.shape
        q_len = 1
    else:
        B, q_len, Hq, D = q.shape
    lead = tuple(q.shape[:-2])
    if kv_layout not in ("NHD", "HND"):
        raise ValueError("kv_layout must be 'NHD' or 'HND'")
    if kv_layout == "HND":
        num_blocks, Hkv, bt, D2 = k_cache.shape
    else:
        num_blocks, bt, Hkv, D2 = k_cache.shape
    if D2 != D:
        raise ValueError("q and the caches disagree on head_dim")
    max_blocks = block_table.shape[1]
    dev = q.device
    if cp_publish is not None:
        out, lse, out_dtype = None, None, "f32"
    else:
        out, lse = _alloc_outputs(out, lse, lead, Hq, D, dev, out_dtype, return_lse)
    for name, t in (("q", q),) + ((("out", out),) if out is not None else ()):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor")
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("q must be bf16 or fp16")
    a = fpd_decode_args()
    a.q = q.data_ptr()
    a.q_dtype = FPD_Q_F16 if q.dtype == torch.float16 else FPD_Q_BF16
    a.q_token_stride = _token_rows(q, "q", lead, Hq, D)
    kv_types = (torch.uint8, torch.float8_e4m3fn)
    a.k_cache = _dev_ptr(k_cache, "k_cache", kv_types).value
    a.v_cache = _dev_ptr(v_cache, "v_cache", kv_types, tuple(k_cache.shape)).value
    a.kv_layout = FPD_KV_HND if kv_layout == "HND" else FPD_KV_NHD
    a.block_table = _dev_ptr(block_table, "block_table", (torch.int32,), (B, max_blocks)).value
    a.seq_lens = _dev_ptr(seq_lens, "seq_lens", (torch.int32,), (B,)).value
    a.B, a.q_len, a.Hq, a.Hkv, a.D = B, q_len, Hq, Hkv, D
    a.num_blocks, a.block_tokens, a.max_blocks = num_blocks, bt, max_blocks
    a.k_scale, a.k_scale_dev = _scale_arg(k_scale, "k_scale")
    a.v_scale, a.v_scale_dev = _scale_arg(v_scale, "v_scale")
    a.sm_scale = float(sm_scale)
    a.window_left = int(window_left)
    sp = _dev_ptr(sinks, "sinks", (torch.float32,), (Hq,))
    a.sinks = sp.value if sp is not None else None
    if cp_publish is not None:
        (a.cp_gather, a.cp_flags, a.cp_ranks, a.cp_rank, a.cp_epoch,
         a.cp_block_floats) = cp_publish
        a.out_dtype = FPD_OUT_F32
    else:
        a.out = out.data_ptr()
        a.out_token_stride = _token_rows(out, "out", lead, Hq, D)
        lp = _dev_ptr(lse, "lse", (torch.float32,), lead + (Hq,))
        a.lse = lp.value if lp is not None else None
        a.out_dtype = _out_code(out)
    a.chunk_pages_override = int(chunk_pages_override)
    _run_args(a, workspace, dev, stream, "fp8_paged_decode_attention")
    return out, lse


def _alloc_outputs(out, lse, lead, Hq, D, dev, out_dtype, return_lse):
    import torch
    if out_dtype not in ("bf16", "f32"):
        raise ValueError("out_dtype must be 'bf16' or 'f32'")
    if out is None:
        dt = torch.float32 if out_dtype == "f32" else torch.bfloat16
        out = torch.empty(lead + (Hq, D), dtype=dt, device=dev)
    if lse is None and return_lse:
        lse = torch.empty(lead + (Hq,), dtype=torch.float32, device=dev)
    return out, lse


def _out_code(out):
    import torch
    if out.dtype == torch.bfloat16:
        return FPD_OUT_BF16
    if out.dtype == torch.float32:
        return FPD_OUT_F32
    raise TypeError("out must be bf16 or float32")


def _run_args(a, workspace, dev, stream, where):
    """Run a filled descriptor; allocates the workspace it needs when none is given."""
    import torch
    lib = load_library()
    if workspace is None:
        need = int(lib.fp8_paged_decode_workspace_bytes_args(ctypes.byref(a)))
        if need == 0 and a.B > 0:   # surface the planner's own status
            plan = fpd_plan()
            _check(lib.fp8_paged_decode_plan_args(ctypes.byref(a), ctypes.byref(plan)),
                   "fp8_paged_decode_plan_args")
            raise FpdError(FPD_ERR_UNSUPPORTED, "fp8_paged_decode_workspace_bytes_args")
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    st = lib.fp8_paged_decode_attention_args(
        ctypes.byref(a), _dev_ptr(workspace, "workspace", (torch.uint8,)),
        ctypes.c_size_t(workspace.numel()), _stream_handle(stream))
    _check(st, where)


fp8_paged_decode_attention_ex = fp8_paged_decode_attention


def fp8_paged_decode_cache_write(key, value, slot_mapping, k_cache, v_cache, k_scale, v_scale,
                                 status=None, stream=None, kv_layout="NHD"):
    """Enqueue the FP8 KV-cache write on ``stream``: bf16 ``key``/``value``
    [num_tokens, Hkv, D] (rows contiguous; any token stride that is a multiple
    of 8 elements) quantised with the per-tensor scales into ``k_cache``/
    ``v_cache`` [num_blocks, block_tokens, Hkv, D] (or [num_blocks, Hkv,
    block_tokens, D] with ``kv_layout="HND"``; uint8 or float8_e4m3fn) at
    ``slot_mapping`` (int64 [num_tokens], negative = skip).  ``status``: an
    optional int32 CUDA tensor whose first word receives FPD_DEVERR_SLOT."""
    import torch
    T, Hkv, D = key.shape
    if kv_layout not in ("NHD", "HND"):
        raise ValueError("kv_layout must be 'NHD' or 'HND'")
    if kv_layout == "HND":
        num_blocks, Hkv2, bt, D2 = k_cache.shape
    else:
        num_blocks, bt, Hkv2, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or tuple(value.shape) != (T, Hkv, D):
        raise ValueError("key/value and the caches disagree on (Hkv, D)")
    for name, t in (("key", key), ("value", value)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} rows must be contiguous ([num_tokens, Hkv, D], any token stride)")
    kv_types = (torch.uint8, torch.float8_e4m3fn)
    st = load_library().fp8_paged_decode_cache_write_layout(
        ctypes.c_void_p(key.data_ptr()), ctypes.c_void_p(value.data_ptr()),
        _dev_ptr(slot_mapping, "slot_mapping", (torch.int64,), (T,)), T, Hkv, D,
        key.stride(0), value.stride(0), float(k_scale), float(v_scale),
        _dev_ptr(k_cache, "k_cache", kv_types),
        _dev_ptr(v_cache, "v_cache", kv_types, tuple(k_cache.shape)), num_blocks, bt,
        FPD_KV_HND if kv_layout == "HND" else FPD_KV_NHD,
        _dev_ptr(status, "status", (torch.int32,)), _stream_handle(stream))
    _check(st, "fp8_paged_decode_cache_write")


def fp8_paged_decode_check_status(workspace, stream=None, clear=False) -> int:
    """Synchronise ``stream`` and return the workspace's device status bits."""
    import torch
    bits = ctypes.c_int(0)
    st = load_library().fp8_paged_decode_check_status(
        _dev_ptr(workspace, "workspace", (torch.uint8,)), _stream_handle(stream),
        ctypes.byref(bits), int(bool(clear)))
    _check(st, "fp8_paged_decode_check_status")
    return int(bits.value)


def fp8_paged_decode_workspace_init(workspace, stream=None):
    import torch
    st = load_library().fp8_paged_decode_workspace_init(
        _dev_ptr(workspace, "workspace", (torch.uint8,)), ctypes.c_size_t(workspace.numel()),
        _stream_handle(stream))
    _check(st, "fp8_paged_decode_workspace_init")


# ------------------------------------------------------------------ NVFP4 --

def nvfp4_page_layout(Hkv: int, block_tokens: int, D: int) -> dict:
    """Byte offsets inside one NVFP4 page [K data | K scales | V data | V scales]
    (data [Hkv][bt][D/2], scales [Hkv][bt][D/16] per side) and the page size."""
    data = Hkv * block_tokens * D // 2
    sf = Hkv * block_tokens * D // 16
    return dict(k_data=0, k_sf=data, v_data=data + sf, v_sf=2 * data + sf,
                page_bytes=2 * (data + sf))


def _nvfp4_pointers(kv_pages, Hkv, block_tokens, D):
    import torch
    lay = nvfp4_page_layout(Hkv, block_tokens, D)
    if not isinstance(kv_pages, torch.Tensor) or not kv_pages.is_cuda or kv_pages.dtype != torch.uint8:
        raise TypeError("kv_pages must be a uint8 CUDA tensor")
    if kv_pages.dim() != 2 or kv_pages.shape[1] != lay["page_bytes"] or not kv_pages.is_contiguous():
        raise ValueError(f"kv_pages must be contiguous [num_blocks, {lay['page_bytes']}]")
    base = kv_pages.data_ptr()
    return {k: base + lay[k] for k in ("k_data", "k_sf", "v_data", "v_sf")}, lay["page_bytes"]


def fp8_paged_decode_attention_nvfp4(q, kv_pages, block_table, seq_lens, k_scale, v_scale,
                                     sm_scale, *, Hkv, block_tokens, window_left=-1, sinks=None,
                                     out=None, lse=None, workspace=None, stream=None,
                                     chunk_pages_override=0, return_lse=True, out_dtype="bf16"):
    """Decode over NVFP4 pages: ``kv_pages`` uint8 [num_blocks, page_bytes], each
    page [K data | K scales | V data | V scales] (``nvfp4_page_layout``; head-major
    E2M1 pairs, element 2i in the low nibble, and one E4M3 scale per 16
    elements).  An element is e2m1(code) * e4m3(block scale) * k_scale
    (v_scale).  q, out, lse, scales and the rest as ``fp8_paged_decode_attention``."""
    import torch
    if q.dim() == 3:
        B, Hq, D = q.shape
        q_len = 1
    else:
        B, q_len, Hq, D = q.shape
    lead = tuple(q.shape[:-2])
    ptrs, page_bytes = _nvfp4_pointers(kv_pages, Hkv, block_tokens, D)
    num_blocks = kv_pages.shape[0]
    max_blocks = block_table.shape[1]
    dev = q.device
    out, lse = _alloc_outputs(out, lse, lead, Hq, D, dev, out_dtype, return_lse)
    if q.dtype not in (torch.bfloat16, torch.float16):
        raise TypeError("q must be bf16 or fp16")
    a = fpd_decode_args()
    a.q = q.data_ptr()
    a.q_dtype = FPD_Q_F16 if q.dtype == torch.float16 else FPD_Q_BF16
    a.q_token_stride = _token_rows(q, "q", lead, Hq, D)
    a.k_cache, a.v_cache = ptrs["k_data"], ptrs["v_data"]
    a.k_scales, a.v_scales = ptrs["k_sf"], ptrs["v_sf"]
    a.kv_page_stride = a.sf_page_stride = page_bytes
    a.kv_format = FPD_KV_NVFP4
    a.kv_layout = FPD_KV_HND
    a.block_table = _dev_ptr(block_table, "block_table", (torch.int32,), (B, max_blocks)).value
    a.seq_lens = _dev_ptr(seq_lens, "seq_lens", (torch.int32,), (B,)).value
    a.B, a.q_len, a.Hq, a.Hkv, a.D = B, q_len, Hq, Hkv, D
    a.num_blocks, a.block_tokens, a.max_blocks = num_blocks, block_tokens, max_blocks
    a.k_scale, a.k_scale_dev = _scale_arg(k_scale, "k_scale")
    a.v_scale, a.v_scale_dev = _scale_arg(v_scale, "v_scale")
    a.sm_scale = float(sm_scale)
    a.window_left = int(window_left)
    sp = _dev_ptr(sinks, "sinks", (torch.float32,), (Hq,))
    a.sinks = sp.value if sp is not None else None
    a.out = out.data_ptr()
    a.out_token_stride = _token_rows(out, "out", lead, Hq, D)
    lp = _dev_ptr(lse, "lse", (torch.float32,), lead + (Hq,))
    a.lse = lp.value if lp is not None else None
    a.chunk_pages_override = int(chunk_pages_override)
    a.out_dtype = _out_code(out)
    _run_args(a, workspace, dev, stream, "fp8_paged_decode_attention_nvfp4")
    return out, lse


def fp8_paged_decode_workspace_bytes_args(args) -> int:
    return int(load_library().fp8_paged_decode_workspace_bytes_args(ctypes.byref(args)))


def fp8_paged_decode_cp_merge_wait(gather, flags, epoch, out, lse=None, sinks=None,
                                   timeout_ns=1_000_000_000, status=None, stream=None):
    """The merge of a fused exchange: waits (at most ``timeout_ns`` of GPU time)
    until ``flags`` (uint32 CUDA tensor [R], this rank's flag words) all equal
    ``epoch``, then merges ``gather`` (float32 [R, block_floats], the slots the
    ranks' publishing decode calls filled) like ``fp8_paged_decode_cp_merge``.
    A timeout or-s FPD_DEVERR_TIMEOUT into ``status`` (int32 CUDA tensor) and
    leaves ``out`` unwritten."""
    import torch
    if out.dim() not in (3, 4) or out.dtype != torch.bfloat16:
        raise TypeError("out must be bf16 [B, Hq, D] or [B, q_len, Hq, D]")
    Hq, D = out.shape[-2], out.shape[-1]
    lead = tuple(out.shape[:-2])
    R, block = gather.shape
    if flags.dtype not in (torch.int32, torch.uint32) or flags.numel() != R:
        raise ValueError("flags must be R 32-bit words")
    st = load_library().fp8_paged_decode_cp_merge_wait(
        _dev_ptr(gather, "gather", (torch.float32,)), int(R), int(block), int(out.numel() // D),
        int(Hq), int(D), _dev_ptr(sinks, "sinks", (torch.float32,), (Hq,)),
        ctypes.c_void_p(out.data_ptr()), _token_rows(out, "out", lead, Hq, D),
        _dev_ptr(lse, "lse", (torch.float32,), lead + (Hq,)),
        _dev_ptr(flags, "flags", (torch.int32, torch.uint32)), ctypes.c_uint32(int(epoch)),
        ctypes.c_uint64(int(timeout_ns)), _dev_ptr(status, "status", (torch.int32,)),
        _stream_handle(stream))
    _check(st, "fp8_paged_decode_cp_merge_wait")
    return out, lse


def fp8_paged_decode_cp_merge(partials, out, lse=None, sinks=None, stream=None):
    """Enqueue the context-parallel merge: ``partials`` float32 [R, block_floats],
    rank r's row holding its f32 decode output [rows, D] followed by its lse
    [rows] (``cp.partial_views`` lays a buffer out so), rows = out.numel() / D;
    ``out`` bf16 [B, Hq, D] or [B, q_len, Hq, D] ([Hq, D] rows contiguous),
    ``lse`` float32 of out's leading shape or None, ``sinks`` float32 [Hq] or
    None.  Returns ``(out, lse)``."""
    import torch
    if out.dim() not in (3, 4) or out.dtype != torch.bfloat16:
        raise TypeError("out must be bf16 [B, Hq, D] or [B, q_len, Hq, D]")
    Hq, D = out.shape[-2], out.shape[-1]
    lead = tuple(out.shape[:-2])
    rows = out.numel() // D
    if partials.dim() != 2:
        raise ValueError("partials must be [R, block_floats]")
    R, block = partials.shape
    pp = _dev_ptr(partials, "partials", (torch.float32,))
    lp = _dev_ptr(lse, "lse", (torch.float32,), lead + (Hq,))
    sp = _dev_ptr(sinks, "sinks", (torch.float32,), (Hq,))
    st = load_library().fp8_paged_decode_cp_merge(
        pp, int(R), int(block), int(rows), int(Hq), int(D), sp,
        ctypes.c_void_p(out.data_ptr()), _token_rows(out, "out", lead, Hq, D), lp,
        _stream_handle(stream))
    _check(st, "fp8_paged_decode_cp_merge")
    return out, lse


def fp8_paged_decode_cache_write_nvfp4(key, value, slot_mapping, kv_pages, k_scale, v_scale, *,
                                       block_tokens, status=None, stream=None):
    """Enqueue the NVFP4 KV-cache write: bf16 ``key``/``value`` [num_tokens, Hkv,
    D] (rows contiguous, token stride a multiple of 8) quantised per 16-element
    block into ``kv_pages`` (uint8 [num_blocks, page_bytes], ``nvfp4_page_layout``)
    at ``slot_mapping`` (int64, negative = skip)."""
    import torch
    T, Hkv, D = key.shape
    if tuple(value.shape) != (T, Hkv, D):
        raise ValueError("key and value disagree on shape")
    for name, t in (("key", key), ("value", value)):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} rows must be contiguous")
    ptrs, page_bytes = _nvfp4_pointers(kv_pages, Hkv, block_tokens, D)
    vp = ctypes.c_void_p
    st = load_library().fp8_paged_decode_cache_write_nvfp4(
        vp(key.data_ptr()), vp(value.data_ptr()),
        _dev_ptr(slot_mapping, "slot_mapping", (torch.int64,), (T,)), T, Hkv, D, key.stride(0),
        value.stride(0), float(k_scale), float(v_scale), vp(ptrs["k_data"]), vp(ptrs["k_sf"]),
        vp(ptrs["v_data"]), vp(ptrs["v_sf"]), page_bytes, page_bytes, kv_pages.shape[0],
        block_tokens, _dev_ptr(status, "status", (torch.int32,)), _stream_handle(stream))
    _check(st, "fp8_paged_decode_cache_write_nvfp4")
