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
