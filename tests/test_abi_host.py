"""C-ABI library on the host (no GPU): loads, exports every declared symbol, and
its planner / validation logic behave as documented.  No kernel is launched."""
import ctypes
import os
import re

import pytest

import fp8_paged_decode_b200 as fpd
from fp8_paged_decode_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if fbuild.needs_build():
        fbuild.build()
    return fpd.load_library()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(fp8_paged_decode_\w+)\s*\(", text)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 9
    raw = ctypes.CDLL(fpd.library_path())
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/ but not exported"
    assert set(names) == set(fpd.EXPORTED_SYMBOLS)


def test_version_and_status_strings(lib):
    assert "sm_100a" in fpd.fp8_paged_decode_version()
    assert fpd.fp8_paged_decode_version().startswith("0.2")
    assert fpd.fp8_paged_decode_status_string(fpd.FPD_ERR_UNSUPPORTED) == "FPD_ERR_UNSUPPORTED"
    assert fpd.fp8_paged_decode_status_string(99) == "FPD_UNKNOWN_STATUS"


def plan(**kw):
    args = dict(B=32, Hq=32, Hkv=8, D=128, block_tokens=16, max_blocks=512, window_left=-1,
                num_sms=148, ctas_per_sm=2, chunk_pages_override=0)
    args.update(kw)
    return fpd.fp8_paged_decode_make_plan(**args)


def test_planner_fills_the_machine():
    for shape in [dict(B=4, Hq=32, Hkv=8, block_tokens=64, max_blocks=2048),
                  dict(B=32, Hq=32, Hkv=8, block_tokens=16, max_blocks=512),
                  dict(B=256, Hq=64, Hkv=8, block_tokens=32, max_blocks=1024, window_left=4096)]:
        p = plan(**shape)
        # a persistent grid: one CTA per resident slot (148 SMs x 2)
        # Hkv = 8: work items and stages cover KV heads in groups of 4
        assert p["heads_per_stage"] == 4 and p["stage_tokens"] == 16
        units = shape["B"] * shape["Hkv"] // 4
        assert p["ctas"] == min(296, units * p["max_splits"]) == 296
        # enough work items for several per slot on long inputs (about 4 rounds
        # when the items are long, 5 otherwise)
        assert units * p["max_splits"] >= 3 * 296
        # at least 256 (token, KV head) rows per work item
        assert p["chunk_pages"] * shape["block_tokens"] * 4 >= 256


def test_planner_one_head_per_stage():
    # Hkv not a multiple of 4: one KV head per 64-token stage, whole stages per split
    for bt in (16, 32, 64):
        p = plan(Hq=16, Hkv=2, block_tokens=bt, max_blocks=8192 // bt)
        assert p["heads_per_stage"] == 1 and p["stage_tokens"] == 64
        assert p["chunk_pages"] * bt % 64 == 0
        assert p["ctas"] == min(296, 32 * 2 * p["max_splits"])


def test_planner_header_slots():
    # two header slots while an item's query rows fit in 4 KB
    assert plan()["header_slots"] == 2                           # 4 x 4 heads x 128 x 2 B
    assert plan(Hq=64, Hkv=8)["header_slots"] == 1               # 4 x 8 heads
    assert plan(Hq=64, Hkv=8, D=64)["header_slots"] == 2
    assert plan(Hq=32, Hkv=2)["header_slots"] == 2               # 1 x 16 heads


def test_planner_window_caps_splits():
    # a 129-token window spans at most 10 pages: one split.  64 sequences x 2
    # four-head groups leave CTA slots idle, and the planner keeps four heads
    # per stage all the same (128 work items, no combine)
    p = plan(B=64, Hq=64, Hkv=8, D=64, block_tokens=16, max_blocks=1024, window_left=128)
    assert p["heads_per_stage"] == 4 and p["max_splits"] == 1 and p["workspace_bytes"] == 256
    assert p["ctas"] == 128
    # with enough sequences the four-head shape fills the machine by itself
    p4 = plan(B=512, Hq=64, Hkv=8, D=64, block_tokens=16, max_blocks=1024, window_left=128)
    assert p4["heads_per_stage"] == 4 and p4["max_splits"] == 1


def test_planner_override_and_workspace():
    # one KV head per stage: rounded up to whole 64-token (4-page) stages
    p = plan(Hq=8, Hkv=2, chunk_pages_override=5)
    assert p["chunk_pages"] == 8
    assert p["max_splits"] == 512 // 8
    # header + partial O + partial lse
    ws = 256 + 32 * 8 * 64 * 128 * 4 + 32 * 8 * 64 * 4
    assert p["workspace_bytes"] == ws
    # four KV heads per stage: 16-token stages, any page count
    p4 = plan(chunk_pages_override=5)
    assert p4["chunk_pages"] == 5 and p4["max_splits"] == -(-512 // 5)
    p1 = plan(chunk_pages_override=512)
    assert p1["max_splits"] == 1 and p1["workspace_bytes"] == 256


def test_planner_monotone_workspace():
    prev = 0
    for mb in (16, 64, 256, 1024):
        w = plan(max_blocks=mb, chunk_pages_override=4)["workspace_bytes"]
        assert w >= prev
        prev = w


def plan_q(q_len, **kw):
    args = dict(B=32, q_len=q_len, Hq=32, Hkv=8, D=128, block_tokens=16, max_blocks=512,
                window_left=-1, num_sms=148, ctas_per_sm=2, chunk_pages_override=0)
    args.update(kw)
    return fpd.fp8_paged_decode_make_plan_qlen(**args)


@pytest.mark.parametrize("g,q_len,per_item,chunks", [
    (4, 1, 1, 1), (4, 2, 2, 1), (4, 4, 4, 1),      # up to 16 columns: one item per KV range
    (4, 5, 3, 2), (4, 8, 4, 2),                    # near-equal chunks of <= 4 positions
    (8, 2, 2, 1), (8, 3, 2, 2), (8, 8, 2, 4),
    (16, 1, 1, 1), (16, 4, 1, 4),                  # one position per item
    (1, 16, 16, 1), (1, 17, 9, 2), (2, 64, 8, 8),
])
def test_planner_query_chunks(g, q_len, per_item, chunks):
    p = plan_q(q_len, Hq=8 * g)
    assert (p["q_per_item"], p["q_chunks"]) == (per_item, chunks)
    assert p["q_per_item"] * g <= 16 or p["q_per_item"] == 1
    # the partials cover every (sequence, query, head) row
    n_rows = 32 * q_len * 8 * g
    if p["max_splits"] > 1:
        assert p["workspace_bytes"] == 256 + n_rows * p["max_splits"] * (128 * 4 + 4)
    # more work items per KV range: no more splits than with one query
    assert p["max_splits"] <= plan(Hq=8 * g)["max_splits"]


def test_planner_q_len_one_is_the_single_query_plan():
    for shape in [dict(), dict(Hq=64, window_left=4096, block_tokens=32, max_blocks=1024),
                  dict(Hq=16, Hkv=2)]:
        assert plan_q(1, **shape) == plan(**shape)


def test_planner_q_len_limits():
    assert plan_q(fpd.FPD_MAX_Q_LEN)["q_chunks"] == fpd.FPD_MAX_Q_LEN * 4 // 16
    for q_len, status in ((fpd.FPD_MAX_Q_LEN + 1, fpd.FPD_ERR_UNSUPPORTED),
                          (0, fpd.FPD_ERR_INVALID_ARG)):
        with pytest.raises(fpd.FpdError) as e:
            plan_q(q_len)
        assert e.value.status == status


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), fpd.FPD_ERR_UNSUPPORTED),
    (dict(D=256), fpd.FPD_ERR_UNSUPPORTED),
    (dict(Hq=24, Hkv=8), fpd.FPD_ERR_UNSUPPORTED),     # g = 3
    (dict(Hq=30, Hkv=8), fpd.FPD_ERR_INVALID_ARG),     # not a multiple
    (dict(block_tokens=8), fpd.FPD_ERR_UNSUPPORTED),
    (dict(block_tokens=128), fpd.FPD_ERR_UNSUPPORTED),
    (dict(B=-1), fpd.FPD_ERR_INVALID_ARG),
    (dict(max_blocks=0), fpd.FPD_ERR_INVALID_ARG),
    (dict(num_sms=0), fpd.FPD_ERR_INVALID_ARG),
    (dict(chunk_pages_override=-2), fpd.FPD_ERR_INVALID_ARG),
])
def test_planner_rejects(kw, status):
    with pytest.raises(fpd.FpdError) as e:
        plan(**kw)
    assert e.value.status == status


def test_attention_validates_before_any_launch(lib):
    f = lib.fp8_paged_decode_attention
    P = ctypes.c_void_p(4096)   # never dereferenced: validation fails first
    args = [P, P, P, P, P, 2, 8, 2, 128, 10, 16, 4, 1.0, 1.0, 0.1, -1, None, P, None, P, 1 << 20, None]
    bad = list(args); bad[8] = 80                       # D = 80
    assert f(*bad) == fpd.FPD_ERR_UNSUPPORTED
    bad = list(args); bad[0] = None                     # q == NULL
    assert f(*bad) == fpd.FPD_ERR_INVALID_ARG
    bad = list(args); bad[14] = 0.0                     # sm_scale * k_scale must be > 0
    assert f(*bad) == fpd.FPD_ERR_INVALID_ARG
    bad = list(args); bad[12] = float("nan")
    assert f(*bad) == fpd.FPD_ERR_INVALID_ARG
    bad = list(args); bad[0] = ctypes.c_void_p(4100)    # q not 16-byte aligned
    assert f(*bad) == fpd.FPD_ERR_INVALID_ARG
    bad = list(args); bad[9] = 0                        # empty pool
    assert f(*bad) == fpd.FPD_ERR_UNSUPPORTED
    ok = list(args); ok[5] = 0                          # B == 0: nothing to do
    assert f(*ok) == fpd.FPD_OK


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        fpd.load_library(str(tmp_path / "absent.so"))


def base_args(**kw):
    P = 4096   # never dereferenced: validation fails first (or B == 0 returns early)
    a = fpd.fpd_decode_args()
    a.q = a.k_cache = a.v_cache = a.block_table = a.seq_lens = a.out = P
    a.B, a.q_len, a.Hq, a.Hkv, a.D = 2, 1, 8, 2, 128
    a.num_blocks, a.block_tokens, a.max_blocks = 10, 16, 4
    a.k_scale = a.v_scale = 1.0
    a.sm_scale = 0.1
    a.window_left = -1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value", [
    ("q_token_stride", 7), ("q_token_stride", 8 * 128 - 8), ("out_token_stride", 1028),
    ("q_dtype", 2), ("kv_layout", 2), ("sm_scale", 0.0), ("chunk_pages_override", -1),
    ("k_scale", float("inf")),
])
def test_args_entry_validates_each_field(lib, field, value):
    """Each field of the descriptor reaches its check (the C and Python struct
    layouts agree); no CUDA call is made before these checks."""
    f = lib.fp8_paged_decode_attention_args
    ws = ctypes.c_void_p(4096)
    assert f(ctypes.byref(base_args(**{field: value})), ws, 1 << 20, None) == \
        fpd.FPD_ERR_INVALID_ARG
    # a device k_scale lifts the host k_scale check
    if field == "k_scale":
        a = base_args(k_scale=float("inf"), k_scale_dev=4096, B=0)
        assert f(ctypes.byref(a), ws, 1 << 20, None) == fpd.FPD_OK


def test_args_entry_accepts_the_variants(lib):
    f = lib.fp8_paged_decode_attention_args
    ws = ctypes.c_void_p(4096)
    for kw in (dict(), dict(q_dtype=fpd.FPD_Q_F16), dict(kv_layout=fpd.FPD_KV_HND),
               dict(q_token_stride=8 * 128 + 8 * 3 * 128, out_token_stride=8 * 128 + 64),
               dict(q_len=5)):
        assert f(ctypes.byref(base_args(B=0, **kw)), ws, 1 << 20, None) == fpd.FPD_OK
    assert f(None, ws, 1 << 20, None) == fpd.FPD_ERR_INVALID_ARG
    # misaligned q base stays rejected through the descriptor
    assert f(ctypes.byref(base_args(q=4100)), ws, 1 << 20, None) == fpd.FPD_ERR_INVALID_ARG


def test_planner_single_split_for_tiny_calls():
    """A call that cannot fill the machine and whose longest item is a few
    stages gets one split (no combine launch); longer ones keep splitting."""
    p = plan(B=2, Hq=8, Hkv=2, block_tokens=16, max_blocks=19)      # <= 304 tokens, 5 stages
    assert p["max_splits"] == 1 and p["workspace_bytes"] == 256
    p = plan(B=2, Hq=8, Hkv=2, block_tokens=16, max_blocks=40)      # 640 tokens, 10 stages
    assert p["max_splits"] > 1
    p = plan(B=2, Hq=32, Hkv=8, block_tokens=16, max_blocks=6)      # four-head stages: 6 stages
    assert p["max_splits"] == 1
    # overriding the split size still wins
    assert plan(B=2, Hq=8, Hkv=2, block_tokens=16, max_blocks=19,
                chunk_pages_override=4)["max_splits"] == 5


def test_planner_underfilled_calls_split_finer():
    """A call whose minimum-size items cannot fill the machine splits down to
    items of about 48 tokens (two items per SM at most); one that needs no
    split keeps a single one, so no combine kernel runs."""
    p = plan(B=1, max_blocks=256, ctas_per_sm=3)            # one 4096-token sequence
    assert p["chunk_pages"] == 3 and p["adapt_chunk_pages"] == 0
    assert p["max_splits"] == 86 and p["ctas"] == 2 * 86    # two four-head groups
    p = plan(B=1, block_tokens=64, max_blocks=64, ctas_per_sm=3)
    assert p["chunk_pages"] == 1                             # 64-token pages: one page
    p = plan(B=64, Hq=64, Hkv=8, D=64, max_blocks=1024, window_left=128, ctas_per_sm=3)
    assert p["max_splits"] == 1 and p["ctas"] == 128


def test_planner_offers_one_round_split_size():
    """Between one and 2.5 rounds of minimum-size items: the plan keeps the
    minimum split (max_splits, workspace) and offers a larger one for one round
    of about two items per SM, with the grid sized for it."""
    p = plan(B=4, block_tokens=64, max_blocks=256, ctas_per_sm=3)   # 4 x 16384 tokens
    assert p["chunk_pages"] == 4 and p["max_splits"] == 64        # 512 items: 1.15 rounds
    assert p["adapt_chunk_pages"] == 7 and p["ctas"] == 8 * 37    # 296 items
    # one KV head per stage: whole 64-token stages (4 pages)
    p = plan(B=8, Hq=8, Hkv=2, max_blocks=1024, ctas_per_sm=3)
    assert p["heads_per_stage"] == 1 and p["adapt_chunk_pages"] == 56
    assert p["ctas"] == 16 * 19
    # many rounds (Llama-3-8B-shaped, long context): the queue balances them
    for kw in (dict(), dict(B=4, block_tokens=64, max_blocks=2048)):
        p = plan(ctas_per_sm=3, **kw)
        assert p["adapt_chunk_pages"] == 0 and p["ctas"] == 444
    # a forced split size is used as given
    p = plan(B=4, block_tokens=64, max_blocks=256, ctas_per_sm=3, chunk_pages_override=4)
    assert p["adapt_chunk_pages"] == 0 and p["ctas"] == 444


def test_ctypes_structs_match_the_c_header(tmp_path):
    """The Python mirrors of fpd_plan and fpd_decode_args have the C layout:
    every field's offset and the struct sizes, as a C compiler sees the header."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "fp8_paged_decode.h"',
             "int main(void) {"]
    for cname, cls in (("fpd_plan", fpd.fpd_plan), ("fpd_decode_args", fpd.fpd_decode_args)):
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(root, "include"), "-o", str(exe), str(src)], check=True)
    seen = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True,
                               text=True).stdout.splitlines():
        name, field, value = line.split()
        seen[(name, field)] = int(value)
    for cname, cls in (("fpd_plan", fpd.fpd_plan), ("fpd_decode_args", fpd.fpd_decode_args)):
        assert seen[(cname, "size")] == ctypes.sizeof(cls), cname
        for f, _ in cls._fields_:
            assert seen[(cname, f)] == getattr(cls, f).offset, (cname, f)


def test_binding_arguments_match_the_header():
    """Every entry point's ctypes argtypes matches its C prototype: as many
    arguments, pointers where the header has pointers, and scalars of the
    header's size and kind (a wrong one would shift or garble later ones)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "include", "fp8_paged_decode.h")) as f:
        text = re.sub(r"/\*.*?\*/", " ", f.read(), flags=re.S)   # drop comments
    protos = dict(
        (m.group(1), m.group(2))
        for m in re.finditer(r"\b(fp8_paged_decode_\w+)\s*\(([^;{}]*?)\)\s*;", text))
    lib = fpd.load_library()
    # C parameter type -> (is a pointer, size in bytes, is a float)
    scalar = {"int": (4, False), "fpd_status": (4, False), "float": (4, True),
              "size_t": (8, False), "int64_t": (8, False), "uint32_t": (4, False),
              "uint64_t": (8, False)}
    checked = 0
    for name in fpd.EXPORTED_SYMBOLS:
        params = protos[name].strip()
        plist = [] if params in ("", "void") else [x.strip() for x in params.split(",")]
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, name
        assert len(argtypes) == len(plist), (name, len(argtypes), len(plist))
        for decl, at in zip(plist, argtypes):
            is_ptr = "*" in decl
            py_ptr = at in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(at, "_type_") and \
                isinstance(getattr(at, "_type_", None), type)
            assert is_ptr == py_ptr, (name, decl, at)
            if not is_ptr:
                ctype = decl.rsplit(None, 1)[0].replace("const", "").strip()
                size, is_float = scalar[ctype]
                assert ctypes.sizeof(at) == size, (name, decl, at)
                assert (at in (ctypes.c_float, ctypes.c_double)) == is_float, (name, decl, at)
        checked += 1
    assert checked == len(fpd.EXPORTED_SYMBOLS)


def test_planner_invariants_on_random_shapes():
    """For many random supported shapes and machine sizes, the plan is
    self-consistent: splits cover every page, whole stages with one head per
    stage, a grid within the resident slots, a larger offered split size only
    with fewer items, and a workspace that holds every partial."""
    import numpy as np
    rng = np.random.default_rng(2024)
    for _ in range(3000):
        Hkv = int(rng.choice([1, 2, 4, 8, 16]))
        g = int(rng.choice([1, 2, 4, 8, 16]))
        D = int(rng.choice([64, 128]))
        bt = int(rng.choice([16, 32, 64]))
        B = int(rng.integers(1, 300))
        q_len = int(rng.choice([1, 1, 1, 2, 3, 4, 8]))
        max_blocks = int(rng.integers(1, 3000))
        window = int(rng.choice([-1, -1, 0, 5, 128, 4096]))
        sms, occ = int(rng.choice([132, 148, 160])), int(rng.integers(1, 4))
        p = fpd.fp8_paged_decode_make_plan_qlen(B, q_len, g * Hkv, Hkv, D, bt, max_blocks,
                                                window, sms, occ)
        HB = p["heads_per_stage"]
        assert HB == (4 if Hkv % 4 == 0 else 1)
        pages = max_blocks if window < 0 else min(max_blocks, (window + q_len - 1) // bt + 2)
        assert p["chunk_pages"] >= 1 and p["max_splits"] == -(-pages // p["chunk_pages"])
        if HB == 1:
            assert p["chunk_pages"] % (64 // bt) == 0
        units = B * (Hkv // HB) * p["q_chunks"]
        assert 1 <= p["ctas"] <= sms * occ
        assert p["ctas"] <= units * p["max_splits"]
        a = p["adapt_chunk_pages"]
        if a:
            assert a > p["chunk_pages"] and (HB == 4 or a % (64 // bt) == 0)
            assert p["ctas"] == min(sms * occ, units * -(-pages // a))
        parts = B * q_len * g * Hkv * p["max_splits"] if p["max_splits"] > 1 else 0
        assert p["workspace_bytes"] >= 256 + parts * (D + 1) * 4
        assert p["q_per_item"] * g <= 16 or p["q_per_item"] == 1
