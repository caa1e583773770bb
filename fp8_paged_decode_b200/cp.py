"""Context-parallel decode: every sequence's KV pages are spread over the ranks
of a process group, one process per GPU.

Each rank runs the decode over its own keys with no sinks and an f32 output,
giving a partial (O_r, lse_r) per (token, head) row; the ranks all-gather those
partials (one NCCL collective over NVLink / NVSwitch); each rank then folds
them, and the sinks, into the attention over all keys with
``fp8_paged_decode_cp_merge``, the split-KV merge of partial O and LSE of
FlashInfer PR #5591 (Summary) with ranks in place of splits.  That page lists
decode context parallelism as unsupported ("Unsupported" section), so the
partition of the keys is the caller's; ``cp_shard`` gives the contiguous,
page-aligned one the tests and the benchmark use.

Supported: one query token per sequence and no sliding window.  Both depend
on a key's absolute position, which a rank holding a middle part of a
sequence does not see: its causal and window masks would be taken relative to
its own last key.

The per-rank buffer is [O (rows * D) | lse (rows) | pad to 4 floats] f32, rows =
B * Hq, so an all-gather of it is already the merge's [R, block] input.

``CpExchange`` and ``fp8_paged_decode_attention_cp_fused`` fuse the exchange
into the decode instead: each rank's combine kernel stores its rows straight
into every rank's gather buffer (peer memory mapped with CUDA IPC) and raises a
flag there, and each rank's merge waits for the flags; no collective runs on
the data path.
"""
from __future__ import annotations

import numpy as np


def partial_block_floats(rows: int, D: int) -> int:
    """Floats of one rank's partial buffer: O, lse, padded to 16 bytes."""
    return rows * D + (rows + 3) // 4 * 4


def partial_views(buf, lead, Hq: int, D: int):
    """(O view [*lead, Hq, D], lse view [*lead, Hq]) of a flat f32 partial buffer."""
    rows = int(np.prod(lead)) * Hq
    if buf.dim() != 1 or buf.numel() < partial_block_floats(rows, D):
        raise ValueError("partial buffer too small")
    o = buf[: rows * D].view(*lead, Hq, D)
    lse = buf[rows * D: rows * D + rows].view(*lead, Hq)
    return o, lse


def cp_shard(block_table, seq_lens, world: int, rank: int, block_tokens: int):
    """Rank ``rank``'s share of every sequence: a contiguous run of whole pages.

    Sequence b of L tokens has P = ceil(L / block_tokens) pages; rank r holds
    pages [floor(r P / world), floor((r + 1) P / world)), so the ranks' page
    counts differ by one at most and only the last holder's final page may be
    partly filled.  Returns (block_table_r [B, max(1, most pages)], seq_lens_r
    [B]) as int32 numpy arrays; block_table_r lists the same physical page
    numbers (unused entries 0), seq_lens_r the rank's key count (0 when it holds
    no page of the sequence).  Host-only."""
    if world < 1 or not 0 <= rank < world or block_tokens < 1:
        raise ValueError("need world >= 1, 0 <= rank < world, block_tokens >= 1")
    table = np.asarray(block_table, dtype=np.int64)
    lens = np.asarray(seq_lens, dtype=np.int64)
    B = lens.shape[0]
    pages = (lens + block_tokens - 1) // block_tokens
    p0 = rank * pages // world
    p1 = (rank + 1) * pages // world
    width = max(1, int((p1 - p0).max()) if B else 1)
    out_table = np.zeros((B, width), dtype=np.int32)
    out_lens = np.zeros(B, dtype=np.int32)
    for b in range(B):
        n = int(p1[b] - p0[b])
        out_table[b, :n] = table[b, p0[b]:p1[b]]
        end = min(int(p1[b]) * block_tokens, int(lens[b]))
        out_lens[b] = max(0, end - int(p0[b]) * block_tokens)
    return out_table, out_lens


def cp_exchange(buf, group=None, gathered=None):
    """All-gather every rank's flat partial buffer: returns [world, numel], row r
    from rank r.  The one collective of the path (NCCL for CUDA tensors, gloo
    for CPU ones)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if gathered is None:
        gathered = torch.empty((world, buf.numel()), dtype=buf.dtype, device=buf.device)
    # a flat output: rank r's buffer lands at [r * numel, (r + 1) * numel)
    dist.all_gather_into_tensor(gathered.view(-1), buf, group=group)
    return gathered


def fp8_paged_decode_attention_cp(q, k_cache, v_cache, block_table, seq_lens, k_scale, v_scale,
                                  sm_scale, *, sinks=None, group=None, out=None, lse=None,
                                  workspace=None, partial=None, gathered=None,
                                  kv_layout="NHD", chunk_pages_override=0):
    """One rank's context-parallel decode on torch's current stream.

    ``block_table`` / ``seq_lens`` describe this rank's keys of each sequence
    (``cp_shard``), over this rank's caches; ``q`` bf16 or fp16 [B, Hq, D] is
    the same on every rank; ``sinks`` float32 [Hq] or None.  Every rank of
    ``group`` must make the call with the same shapes.  ``partial``
    (f32 [partial_block_floats(B * Hq, D)]), ``gathered`` ([world, that]),
    ``workspace``, ``out`` and ``lse`` may be passed in to keep the call
    allocation-free.  Returns ``(out, lse)``, the attention over all ranks'
    keys, on every rank."""
    import torch
    import torch.distributed as dist
    import fp8_paged_decode_b200 as fpd
    if q.dim() != 3:
        raise ValueError("context-parallel decode takes one query token per sequence: q [B, Hq, D]")
    B, Hq, D = q.shape
    rows = B * Hq
    dev = q.device
    if partial is None:
        partial = torch.empty(partial_block_floats(rows, D), dtype=torch.float32, device=dev)
    o_r, lse_r = partial_views(partial, (B,), Hq, D)
    fpd.fp8_paged_decode_attention(q, k_cache, v_cache, block_table, seq_lens, k_scale, v_scale,
                                   sm_scale, window_left=-1, sinks=None, out=o_r, lse=lse_r,
                                   workspace=workspace, kv_layout=kv_layout,
                                   chunk_pages_override=chunk_pages_override)
    if gathered is None:
        gathered = torch.empty((dist.get_world_size(group), partial.numel()),
                               dtype=torch.float32, device=dev)
    cp_exchange(partial, group, gathered)
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    return fpd.fp8_paged_decode_cp_merge(gathered, out, lse, sinks)


# ------------------------------------------------------------ fused exchange --

def _cudart():
    """The CUDA runtime library that torch loads, with the prototypes the
    context-parallel exchange and the benchmark's host loop use: device
    allocation, IPC handles, async copies and event calls."""
    import ctypes
    import ctypes.util
    import os
    import torch
    cands = [os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib",
                          "libcudart.so.12")]
    found = ctypes.util.find_library("cudart")
    if found:
        cands.append(found)
    for c in cands:
        try:
            rt = ctypes.CDLL(c)
            break
        except OSError:
            continue
    else:
        raise RuntimeError("no CUDA runtime library found")

    class Handle(ctypes.Structure):
        _fields_ = [("reserved", ctypes.c_char * 64)]
    vp = ctypes.c_void_p
    rt.cudaMalloc.argtypes = [ctypes.POINTER(vp), ctypes.c_size_t]
    rt.cudaFree.argtypes = [vp]
    rt.cudaMemset.argtypes = [vp, ctypes.c_int, ctypes.c_size_t]
    rt.cudaIpcGetMemHandle.argtypes = [ctypes.POINTER(Handle), vp]
    rt.cudaIpcOpenMemHandle.argtypes = [ctypes.POINTER(vp), Handle, ctypes.c_uint]
    rt.cudaIpcCloseMemHandle.argtypes = [vp]
    rt.cudaMemcpyAsync.argtypes = [vp, vp, ctypes.c_size_t, ctypes.c_int, vp]
    rt.cudaEventRecord.argtypes = [vp, vp]
    rt.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
    rt.Handle = Handle
    return rt


class CpExchange:
    """The buffers of the exchange fused into the decode (``cp_gather`` /
    ``cp_flags`` of the decode descriptor) for one process group, one process
    per GPU.

    Every rank owns one device allocation (cudaMalloc): two gather buffers of
    R slots of ``partial_block_floats(B * Hq, D)`` floats, then two arrays of R
    flag words.  The ranks exchange CUDA IPC handles of their allocations once
    (a gather of small host objects over the process group), so each rank
    holds device pointers to every rank's buffers; its combine kernel stores
    its rows straight into slot ``rank`` of all of them over NVLink and raises
    its flag there, and its merge waits for the R flags of its own buffer.
    Steps alternate between the two buffers by the parity of the epoch: a rank
    may publish step k + 1 while a slower rank still merges step k, but not
    step k + 2, whose merge waits for that rank's step k + 1, which its stream
    runs after its merge of step k.

    ``CpExchange.local(R, ...)`` makes R such buffers in one process, standing
    in for R ranks on one GPU (the publishing calls then run one after another,
    and every flag is set before any merge waits on it)."""

    def __init__(self, B, Hq, D, group=None, _local_ranks=None):
        import ctypes
        import torch
        self.B, self.Hq, self.D = B, Hq, D
        self.block = partial_block_floats(B * Hq, D)
        self._rt = _cudart()
        self._opened = []
        self._own = []
        if _local_ranks is not None:
            self.R, self.rank = _local_ranks, 0
            bases = [self._alloc() for _ in range(self.R)]
            self._own = list(bases)
        else:
            import torch.distributed as dist
            self.R = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
            mine = self._alloc()
            self._own = [mine]
            h = self._rt.Handle()
            self._check(self._rt.cudaIpcGetMemHandle(ctypes.byref(h), ctypes.c_void_p(mine)))
            handles = [None] * self.R
            dist.all_gather_object(handles, bytes(h.reserved), group=group)
            bases = []
            for r, hb in enumerate(handles):
                if r == self.rank:
                    bases.append(mine)
                    continue
                hr = self._rt.Handle()
                ctypes.memmove(hr.reserved, hb, 64)
                p = ctypes.c_void_p()
                self._check(self._rt.cudaIpcOpenMemHandle(ctypes.byref(p), hr, 1))
                self._opened.append(p.value)
                bases.append(p.value)
        self.bases = bases
        dev = torch.device("cuda", torch.cuda.current_device())
        # per parity: every rank's gather buffer and flag array
        self.gather_ptrs = [torch.tensor([self._gather_at(b, par) for b in bases],
                                         dtype=torch.int64, device=dev) for par in (0, 1)]
        self.flag_ptrs = [torch.tensor([self._flags_at(b, par) for b in bases],
                                       dtype=torch.int64, device=dev) for par in (0, 1)]
        self.epoch = 0

    @classmethod
    def local(cls, R, B, Hq, D):
        return cls(B, Hq, D, _local_ranks=R)

    def _check(self, err):
        if err != 0:
            raise RuntimeError(f"CUDA runtime error {err} in the context-parallel exchange")

    def _alloc(self):
        import ctypes
        nbytes = self.R_bytes()
        p = ctypes.c_void_p()
        self._check(self._rt.cudaMalloc(ctypes.byref(p), nbytes))
        self._check(self._rt.cudaMemset(p, 0, nbytes))
        return p.value

    def _flag_stride(self):
        return (self.R * 4 + 255) // 256 * 256

    def R_bytes(self):
        """Bytes of one rank's allocation: two gather buffers of R slots, then
        two arrays of R flag words."""
        return 2 * self.R * self.block * 4 + 2 * self._flag_stride()

    def _gather_at(self, base, parity):
        return base + parity * self.R * self.block * 4

    def _flags_at(self, base, parity):
        return base + 2 * self.R * self.block * 4 + parity * self._flag_stride()

    def gather(self, r=None):
        """Rank r's gather buffer of the current epoch, float32 [R, block]
        (this process's rank by default)."""
        import torch
        base = self.bases[self.rank if r is None else r]
        return _borrowed(self._gather_at(base, self.epoch & 1), (self.R, self.block),
                         torch.float32)

    def flags(self, r=None):
        """Rank r's flag words of the current epoch, int32 [R]."""
        import torch
        base = self.bases[self.rank if r is None else r]
        return _borrowed(self._flags_at(base, self.epoch & 1), (self.R,), torch.int32)

    def next_epoch(self):
        """Advance to the next step: epochs run 1, 2, ..., 2**32 - 2 and wrap to 1,
        so they are never 0 and their parity always alternates."""
        self.epoch = self.epoch % 0xFFFFFFFE + 1
        return self.epoch

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def publish_fields(self, rank=None):
        """(cp_gather, cp_flags, cp_ranks, cp_rank, cp_epoch, cp_block_floats) of
        this rank's publishing decode call at the current epoch."""
        par = self.epoch & 1
        return (self.gather_ptrs[par].data_ptr(), self.flag_ptrs[par].data_ptr(), self.R,
                self.rank if rank is None else rank, self.epoch, self.block)

    def close(self):
        """Unmap the peers' buffers and free this rank's (after the device work
        that uses them has finished); the exchange is unusable afterwards."""
        import ctypes
        for p in self._opened:
            self._rt.cudaIpcCloseMemHandle(ctypes.c_void_p(p))
        for p in self._own:
            self._rt.cudaFree(ctypes.c_void_p(p))
        self._opened, self._own, self.bases = [], [], []


class _CudaArray:
    """Raw device memory described by the CUDA array interface (not owned)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3,
                                         "strides": None}


def _borrowed(ptr, shape, dtype):
    """A torch tensor over device memory that torch neither owns nor frees."""
    import torch
    typestr = {torch.float32: "<f4", torch.int32: "<i4"}[dtype]
    return torch.as_tensor(_CudaArray(ptr, shape, typestr), device="cuda")


def fp8_paged_decode_attention_cp_fused(q, k_cache, v_cache, block_table, seq_lens, k_scale,
                                        v_scale, sm_scale, *, exchange, sinks=None, out=None,
                                        lse=None, workspace=None, timeout_ns=1_000_000_000,
                                        status=None, rank=None, publish=True, merge=True,
                                        kv_layout="NHD", chunk_pages_override=0):
    """One rank's context-parallel decode with the exchange fused into it, on
    torch's current stream: the decode over this rank's keys (``block_table`` /
    ``seq_lens``, as ``fp8_paged_decode_attention_cp``) stores its f32 rows
    into every rank's gather buffer of ``exchange`` (a ``CpExchange``) and
    raises its flag there; the merge then waits for all ranks' flags of the
    current ``exchange.epoch`` (call ``exchange.next_epoch()`` once per step,
    on every rank, before this) and folds the slots and the sinks together.
    ``rank`` (default: the exchange's) and ``publish`` / ``merge`` let one
    process stand in for several ranks.  A flag that does not arrive within
    ``timeout_ns`` or-s FPD_DEVERR_TIMEOUT into ``status`` (int32 CUDA tensor)
    and leaves ``out`` unwritten.  Returns ``(out, lse)``."""
    import torch
    import fp8_paged_decode_b200 as fpd
    if q.dim() != 3:
        raise ValueError("context-parallel decode takes one query token per sequence: q [B, Hq, D]")
    if exchange.epoch == 0:
        raise ValueError("call exchange.next_epoch() before the step")
    B, Hq, D = q.shape
    r = exchange.rank if rank is None else rank
    if publish:
        fpd.fp8_paged_decode_attention(q, k_cache, v_cache, block_table, seq_lens, k_scale,
                                       v_scale, sm_scale, window_left=-1, sinks=None,
                                       workspace=workspace, kv_layout=kv_layout,
                                       chunk_pages_override=chunk_pages_override,
                                       cp_publish=exchange.publish_fields(r))
    if not merge:
        return None, None
    if out is None:
        out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    return fpd.fp8_paged_decode_cp_merge_wait(exchange.gather(r), exchange.flags(r),
                                              exchange.epoch, out, lse, sinks,
                                              timeout_ns=timeout_ns, status=status)
