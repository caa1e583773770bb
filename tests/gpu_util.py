"""Helpers for GPU tests: move a seeded workload to the device, run the CUDA
path through the C ABI binding, compare with the oracle."""
import numpy as np
import torch

import fp8_paged_decode_b200 as fpd

OUT_ATOL = 1e-2
OUT_RTOL = 1e-2
LSE_ATOL = 1e-3


def to_device(wl, device="cuda"):
    t = {}
    t["q"] = torch.from_numpy(wl.q.view(np.int16)).view(torch.bfloat16).to(device)
    t["k_cache"] = torch.from_numpy(wl.k_cache).to(device)
    t["v_cache"] = torch.from_numpy(wl.v_cache).to(device)
    t["block_table"] = torch.from_numpy(wl.block_table).to(device)
    t["seq_lens"] = torch.from_numpy(wl.seq_lens).to(device)
    t["sinks"] = None if wl.sinks is None else torch.from_numpy(wl.sinks).to(device)
    return t


def run_cuda(wl, dev=None, chunk_pages=0, window_left=None, workspace=None, out=None, lse=None):
    dev = dev or to_device(wl)
    o, l = fpd.fp8_paged_decode_attention(
        dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"], dev["seq_lens"],
        wl.k_scale, wl.v_scale, wl.sm_scale,
        window_left=wl.window_left if window_left is None else window_left,
        sinks=dev["sinks"], chunk_pages_override=chunk_pages, workspace=workspace, out=out,
        lse=lse)
    torch.cuda.synchronize()
    return o.float().cpu().numpy().astype(np.float64), l.cpu().numpy().astype(np.float64)


def assert_parity(out, lse, ref_out, ref_lse, rows=None, what=""):
    """Element-wise: |out - ref| <= 1e-2 + 1e-2 |ref|, |lse - ref| <= 1e-3."""
    if rows is not None:
        B, Hq = ref_lse.shape
        bs, hs = np.divmod(np.asarray(rows), Hq)
        out, lse, ref_out, ref_lse = out[bs, hs], lse[bs, hs], ref_out[bs, hs], ref_lse[bs, hs]
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ref_out)
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} outputs outside tolerance; worst "
                           f"|d|={err.max():.3e}")
    both_inf = np.isinf(lse) & np.isinf(ref_lse) & (np.sign(lse) == np.sign(ref_lse))
    with np.errstate(invalid="ignore"):
        lerr = np.where(both_inf, 0.0, np.abs(lse - ref_lse))
    assert (lerr <= LSE_ATOL).all(), f"{what}: lse worst |d|={np.nanmax(lerr):.3e}"
    return float(err.max()), float(lerr.max())
