"""The CPU oracle against library routines, closed forms and invariants (no GPU)."""
import pytest

import oracle
from tests import oracle_pins as P


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_rejects_bad_inputs(lib):
    from fp8_paged_decode_b200 import workloads as W
    wl = W.make_custom(B=1, Hq=2, Hkv=1, D=64, block_tokens=16, seq_lens=[20], seed=3)
    bad = wl.block_table.copy()
    bad[0, 1] = wl.num_blocks          # out-of-range page inside the attended range
    with pytest.raises(ValueError):
        oracle.decode(wl.q, wl.k_cache, wl.v_cache, bad, wl.seq_lens, k_scale=1, v_scale=1,
                      sm_scale=1, lib=lib)
    lens = wl.seq_lens.copy()
    lens[0] = wl.max_blocks * 16 + 1   # longer than the table can hold
    with pytest.raises(ValueError):
        oracle.decode(wl.q, wl.k_cache, wl.v_cache, wl.block_table, lens, k_scale=1, v_scale=1,
                      sm_scale=1, lib=lib)


def test_rows_subset_matches_full(lib):
    from fp8_paged_decode_b200 import workloads as W
    import numpy as np
    wl = W.make_custom(B=3, Hq=8, Hkv=2, D=64, block_tokens=16, seq_lens=[9, 40, 77], seed=4,
                       sinks=True)
    out, lse = oracle.decode_workload(wl, lib=lib)
    rows = [1, 10, 23]
    o2, l2 = oracle.decode_workload(wl, rows=rows, lib=lib)
    for r in rows:
        b, h = divmod(r, wl.Hq)
        assert np.array_equal(o2[b, h], out[b, h]) and l2[b, h] == lse[b, h]
    assert np.isnan(l2[0, 0])
