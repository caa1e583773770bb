"""FP8 KV-cache write on the GPU vs the CPU oracle: bit-exact on every byte of
both caches (written slots and untouched ones), since the E4M3 code is decided
in fp32 on both sides from the same reciprocal and product."""
import numpy as np
import pytest
import torch

import fp8_paged_decode_b200 as fpd
import oracle
from fp8_paged_decode_b200 import workloads as W
from tests.gpu_util import assert_parity, run_cuda, to_device

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU hosts, never run there
    pytest.skip("needs a CUDA device", allow_module_level=True)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def kv_values(rng, shape, scale):
    """Mixed magnitudes: typical values, values past the E4M3 range (saturate)
    and values near and under the smallest subnormal."""
    x = rng.standard_normal(shape).astype(np.float32) * scale
    flat = x.reshape(-1)
    n = flat.size
    idx = rng.permutation(n)
    flat[idx[: n // 20]] *= 600.0
    flat[idx[n // 20: n // 10]] *= 1e-4
    return x


def gpu_write(key_bits, value_bits, slots, kc0, vc0, k_scale, v_scale, status=None):
    dev = "cuda"
    key = torch.from_numpy(key_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    value = torch.from_numpy(value_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    kc = torch.from_numpy(kc0.copy()).to(dev)
    vc = torch.from_numpy(vc0.copy()).to(dev)
    sm = torch.from_numpy(slots).to(dev)
    fpd.fp8_paged_decode_cache_write(key, value, sm, kc, vc, k_scale, v_scale, status=status)
    torch.cuda.synchronize()
    return kc.cpu().numpy(), vc.cpu().numpy()


def oracle_write(key_bits, value_bits, slots, kc0, vc0, k_scale, v_scale):
    kc, vc = kc0.copy(), vc0.copy()
    bad = oracle.cache_write(key_bits, value_bits, slots, kc, vc, k_scale=k_scale, v_scale=v_scale)
    return kc, vc, bad


def assert_same_codes(got, want, what):
    nan_w = (want & 0x7F) == 0x7F
    nan_g = (got & 0x7F) == 0x7F
    assert np.array_equal(nan_w, nan_g), f"{what}: NaN codes differ"
    diff = np.flatnonzero((got != want) & ~nan_w)
    assert diff.size == 0, (f"{what}: {diff.size} bytes differ, first at {diff[0]}: "
                            f"{got.reshape(-1)[diff[0]]:#x} vs {want.reshape(-1)[diff[0]]:#x}")


CASES = [(1, 64, 16, 1), (2, 128, 16, 37), (8, 128, 16, 700), (8, 64, 32, 300), (4, 128, 64, 129)]


@pytest.mark.parametrize("Hkv,D,bt,T", CASES, ids=[f"kv{h}-D{d}-bt{b}-T{t}" for h, d, b, t in CASES])
def test_bit_exact(Hkv, D, bt, T):
    rng = np.random.default_rng(1000 + Hkv + D + bt + T)
    nb = (T + bt - 1) // bt + 3
    key = bf16_bits(kv_values(rng, (T, Hkv, D), 2.0))
    value = bf16_bits(kv_values(rng, (T, Hkv, D), 0.5))
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    if T > 5:
        slots[rng.choice(T, T // 5, replace=False)] = -1       # padded tokens
    kc0 = rng.integers(0, 256, (nb, bt, Hkv, D), dtype=np.uint8)  # stale bytes stay untouched
    vc0 = rng.integers(0, 256, (nb, bt, Hkv, D), dtype=np.uint8)
    for ks, vs in ((0.01, 0.003), (1.0, 1.0), (1.7, 0.37)):
        gk, gv = gpu_write(key, value, slots, kc0, vc0, ks, vs)
        wk, wv, bad = oracle_write(key, value, slots, kc0, vc0, ks, vs)
        assert bad == 0
        assert_same_codes(gk, wk, f"K scale {ks}")
        assert_same_codes(gv, wv, f"V scale {vs}")


def test_strided_key_value():
    """key and value as slices of a fused [T, (Hq + 2 Hkv) * D] projection."""
    rng = np.random.default_rng(7)
    T, Hq, Hkv, D, bt, nb = 50, 8, 2, 128, 16, 6
    fused = torch.from_numpy(kv_values(rng, (T, (Hq + 2 * Hkv) * D), 1.0)).to(torch.bfloat16).cuda()
    key = fused[:, Hq * D:(Hq + Hkv) * D].view(T, Hkv, D)
    value = fused[:, (Hq + Hkv) * D:].view(T, Hkv, D)
    assert key.stride(0) == (Hq + 2 * Hkv) * D
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    kc = torch.zeros((nb, bt, Hkv, D), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    fpd.fp8_paged_decode_cache_write(key, value, torch.from_numpy(slots).cuda(), kc, vc, 0.2, 0.3)
    kb = fused.cpu().view(torch.int16).numpy().view(np.uint16)
    wk, wv, _ = oracle_write(kb[:, Hq * D:(Hq + Hkv) * D].reshape(T, Hkv, D),
                             kb[:, (Hq + Hkv) * D:].reshape(T, Hkv, D), slots,
                             np.zeros((nb, bt, Hkv, D), np.uint8),
                             np.zeros((nb, bt, Hkv, D), np.uint8), 0.2, 0.3)
    assert_same_codes(kc.cpu().numpy(), wk, "strided K")
    assert_same_codes(vc.cpu().numpy(), wv, "strided V")


def test_special_values():
    """+-inf saturate to +-448, NaN stays a NaN code, signed zeros keep their sign."""
    T, Hkv, D, bt = 4, 1, 64, 16
    x = np.zeros((T, Hkv, D), np.float32)
    x[0, 0, :8] = [np.inf, -np.inf, np.nan, -0.0, 0.0, 1e-30, -1e-30, 448.0]
    x[1] = 1e6
    x[2] = -1e6
    x[3, 0] = np.linspace(-500, 500, D)
    bits = bf16_bits(x)
    slots = np.array([0, 1, 2, 3], np.int64)
    kc0 = np.zeros((1, bt, Hkv, D), np.uint8)
    gk, gv = gpu_write(bits, bits, slots, kc0, kc0, 1.0, 1.0)
    wk, wv, _ = oracle_write(bits, bits, slots, kc0, kc0, 1.0, 1.0)
    assert_same_codes(gk, wk, "special K")
    assert_same_codes(gv, wv, "special V")
    row = gk[0, 0, 0]
    assert row[0] == 0x7E and row[1] == 0xFE and (row[2] & 0x7F) == 0x7F
    assert row[3] == 0x80 and row[4] == 0x00 and row[6] == 0x80


def test_out_of_range_slot_flagged_and_skipped():
    rng = np.random.default_rng(9)
    T, Hkv, D, bt, nb = 20, 2, 64, 16, 2
    key = bf16_bits(rng.standard_normal((T, Hkv, D)))
    slots = rng.permutation(nb * bt)[:T].astype(np.int64)
    slots[4] = nb * bt          # one past the end
    slots[9] = 10 ** 12
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    kc0 = np.zeros((nb, bt, Hkv, D), np.uint8)
    gk, gv = gpu_write(key, key, slots, kc0, kc0, 0.5, 0.5, status=status)
    wk, wv, bad = oracle_write(key, key, slots, kc0, kc0, 0.5, 0.5)
    assert bad == 2
    assert_same_codes(gk, wk, "K")
    assert int(status[0].item()) & fpd.FPD_DEVERR_SLOT


def test_no_tokens_and_bad_arguments():
    kc = torch.zeros((2, 16, 2, 64), dtype=torch.uint8, device="cuda")
    empty = torch.empty((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    fpd.fp8_paged_decode_cache_write(empty, empty, torch.empty(0, dtype=torch.int64, device="cuda"),
                                     kc, kc.clone(), 1.0, 1.0)
    assert not kc.any()
    key = torch.zeros((3, 2, 64), dtype=torch.bfloat16, device="cuda")
    slots = torch.arange(3, dtype=torch.int64, device="cuda")
    with pytest.raises(fpd.FpdError):
        fpd.fp8_paged_decode_cache_write(key, key, slots, kc, kc.clone(), 0.0, 1.0)
    wide = torch.zeros((3, 2 * 64 + 4), dtype=torch.bfloat16, device="cuda")
    odd = wide[:, :128].view(3, 2, 64)          # token stride 132: not a multiple of 8
    with pytest.raises(fpd.FpdError):
        fpd.fp8_paged_decode_cache_write(odd, odd, slots, kc, kc.clone(), 1.0, 1.0)


def test_write_then_decode():
    """The writer fills a cache from bf16 K/V; decoding it on the GPU matches
    the oracle on the cache the oracle writes (the two caches are identical)."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, bt = 3, 16, 4, 128, 16
    lens = [300, 17, 1000]
    wl = W.make_custom(B=B, Hq=Hq, Hkv=Hkv, D=D, block_tokens=bt, seq_lens=lens, sinks=True,
                       seed=12, sm_scale=0.08)
    # every attended slot is written by the cache write from fresh bf16 rows
    slots = []
    for b, L in enumerate(lens):
        for j in range(L):
            slots.append(int(wl.block_table[b, j // bt]) * bt + j % bt)
    slots = np.array(slots, np.int64)
    T = len(slots)
    key = bf16_bits(rng.standard_normal((T, Hkv, D)) * 3)
    value = bf16_bits(rng.standard_normal((T, Hkv, D)))
    ks, vs = 3 * 4 / 448, 4 / 448
    gk, gv = gpu_write(key, value, slots, wl.k_cache, wl.v_cache, ks, vs)
    wk, wv, _ = oracle_write(key, value, slots, wl.k_cache, wl.v_cache, ks, vs)
    assert_same_codes(gk, wk, "K")
    assert_same_codes(gv, wv, "V")
    wl.k_cache, wl.v_cache, wl.k_scale, wl.v_scale = wk, wv, ks, vs
    ref_out, ref_lse = oracle.decode_workload(wl)
    out, lse = run_cuda(wl, to_device(wl))
    assert_parity(out, lse, ref_out, ref_lse, what="write then decode")
