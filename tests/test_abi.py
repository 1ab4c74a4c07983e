"""The C-ABI library: builds, loads, exports every entry point the header
declares, and rejects bad arguments on the host without touching a GPU."""
import ctypes
import os
import re

import pytest
import torch

from fp16_kv_cache_b200 import build as hbuild
from fp16_kv_cache_b200 import hyq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hyq.h")
DEBUG_HEADER = os.path.join(ROOT, "include", "hyq_debug.h")


@pytest.fixture(scope="module")
def L():
    hbuild.build()
    return hyq.lib()


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hyq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("hyq_pack", "hyq_prefill", "hyq_append", "hyq_select_vl", "hyq_vl_apply",
              "hyq_decode", "hyq_decode_fp16", "hyq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), n
    assert {n for n, _, _ in hyq.EXPORTS} == set(declared_functions())


def test_debug_library_exports_both_headers():
    hbuild.build_debug()
    D = hyq.debug_lib()
    extra = declared_functions(DEBUG_HEADER)
    assert extra == ["hyq_debug_set_wait"]
    for n in declared_functions() + extra:
        assert hasattr(D, n), n
    assert {n for n, _, _ in hyq.DEBUG_EXPORTS} == set(extra)
    # the release library has no debug entry point
    assert not hasattr(hyq.lib(), "hyq_debug_set_wait")
    assert D.hyq_debug_set_wait(10, 0) == 1  # limit below 1 us: rejected on the host


def test_version_and_status_strings(L):
    assert L.hyq_version() == 100
    for code, text in hyq.STATUS.items():
        assert L.hyq_status_string(code).decode() == text


def _desc(**over):
    c = hyq.hyq_cache()
    c.batch, c.n_q_heads, c.n_kv_heads = 1, 8, 2
    c.head_dim, c.group, c.window, c.capacity, c.vl_capacity = 128, 32, 128, 4096, 64
    fake = 0x10000  # aligned, never dereferenced: validation fails or stops first
    for name in ("blocks", "win_k", "win_v", "vl_k", "vl_v", "vl_pos", "vl_count", "seq_len"):
        setattr(c, name, fake)
        fake += 0x10000
    for k, v in over.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 64, 2), ("group", 64, 2), ("window", 256, 2), ("n_q_heads", 7, 1), ("n_q_heads", 6, 2),
    ("n_q_heads", 24, 2), ("capacity", 4000, 1), ("capacity", 0, 1), ("vl_capacity", 0, 1),
    ("batch", 0, 1), ("blocks", 0, 1), ("vl_pos", 0x10008, 3), ("seq_len", None, 1),
])
def test_decode_rejects_bad_descriptors(L, field, value, code):
    c = _desc(**{field: value})
    rc = L.hyq_decode(ctypes.byref(c), 0x20000000, 0x30000000, None, 0, 0x40000000, 1 << 30, None)
    assert rc == code


def test_decode_requires_workspace(L):
    c = _desc()
    assert L.hyq_decode(ctypes.byref(c), 0x20000000, 0x30000000, None, 8, None, 0, None) == 4
    need = L.hyq_decode_workspace(ctypes.byref(c), 8)
    assert need > 0
    assert L.hyq_decode(ctypes.byref(c), 0x20000000, 0x30000000, None, 8, 0x40000000, need - 1, None) == 4
    assert L.hyq_decode(ctypes.byref(c), 0x20000008, 0x30000000, None, 8, 0x40000000, need, None) == 3


def test_copy_argument_checks(L):
    """hyq_copy's host-side checks come before any CUDA call: null pointers
    and sizes that are not multiples of 16 are invalid, misaligned pointers
    are refused, zero bytes is a no-op; a pointer the CUDA runtime cannot
    describe (no GPU here) is invalid, with nothing enqueued."""
    assert L.hyq_copy(None, 0x2000, 64, None) == 1
    assert L.hyq_copy(0x1000, None, 0, None) == 1      # null even with nothing to copy
    assert L.hyq_copy(0x1000, 0x2000, 0, None) == 0    # nothing to do
    assert L.hyq_copy(0x1000, 0x2000, 40, None) == 1   # not a multiple of 16
    assert L.hyq_copy(0x1008, 0x2000, 64, None) == 3   # misaligned destination
    assert L.hyq_copy(0x1000, 0x2004, 64, None) == 3   # misaligned source
    if not torch.cuda.is_available():
        assert L.hyq_copy(0x1000, 0x2000, 64, None) == 1


def test_pack_argument_checks(L):
    assert L.hyq_pack(0x1000, 0, 128, None, 0x2000, 0x3000, None, None) == 0   # nothing to do
    assert L.hyq_pack(0x1000, -1, 128, None, 0x2000, 0x3000, None, None) == 1
    assert L.hyq_pack(0x1000, 4, 100, None, 0x2000, 0x3000, None, None) == 1
    assert L.hyq_pack(0x1000, 4, 132, None, 0x2000, 0x3000, None, None) == 1
    assert L.hyq_pack(0x1004, 4, 128, None, 0x2000, 0x3000, None, None) == 3
    assert L.hyq_pack(None, 4, 128, None, 0x2000, 0x3000, None, None) == 1


def test_select_and_vl_apply_argument_checks(L):
    c = _desc()
    ws = L.hyq_select_vl_workspace(ctypes.byref(c), 64)
    assert ws > 0
    sel = L.hyq_select_vl
    assert sel(ctypes.byref(c), 0x1000, 0, 0, None, 8, 0x2000, None, 0x4000, ws, None) == 1     # n_q
    assert sel(ctypes.byref(c), 0x1000, 65, 0, None, 8, 0x2000, None, 0x4000, ws, None) == 1    # n_q
    assert sel(ctypes.byref(c), 0x1000, 64, 0, None, 65, 0x2000, None, 0x4000, ws, None) == 1   # k > vl_cap
    assert sel(ctypes.byref(c), 0x1000, 64, 0, None, 8, 0x2000, None, 0x4000, ws - 1, None) == 4
    assert L.hyq_vl_apply(ctypes.byref(c), 0x1000, 65, None, None, None, None) == 1
    assert L.hyq_vl_apply(ctypes.byref(c), 0x1000, 8, 0x2000, None, None, None) == 1  # k_full w/o v_full


def test_append_and_prefill_argument_checks(L):
    c = _desc()
    assert L.hyq_append(ctypes.byref(c), None, 0x2000, None, None, 0, None) == 1
    assert L.hyq_append(ctypes.byref(c), 0x1000, 0x2000, 0x3000, None, 64, None) == 1
    assert L.hyq_append(ctypes.byref(c), 0x1008, 0x2000, None, None, 0, None) == 3
    assert L.hyq_prefill(ctypes.byref(c), None, 0x2000, None) == 1
    assert L.hyq_decode_fp16(0x1000, 0x2000, 0x3000, 0x4000, 1, 6, 2, 4096, 0x5000, None, 0,
                             0x6000, 1 << 20, None, None) == 2


@pytest.mark.parametrize("field,value,code", [("head_dim", 64, 2), ("n_q_heads", 7, 1), ("blocks", 0, 1),
                                              ("vl_pos", 0x10008, 3)])
def test_decode_vl_only_checks_like_decode(L, field, value, code):
    c = _desc(**{field: value})
    args = (0x20000000, 0x30000000, None, 0, 0x40000000, 1 << 30, None)
    assert L.hyq_decode_vl_only(ctypes.byref(c), *args) == code == L.hyq_decode(ctypes.byref(c), *args)


def test_decode_vl_only_requires_workspace(L):
    c = _desc()
    need = L.hyq_decode_workspace(ctypes.byref(c), 8)
    assert L.hyq_decode_vl_only(ctypes.byref(c), 0x20000000, 0x30000000, None, 8, None, 0, None) == 4
    assert L.hyq_decode_vl_only(ctypes.byref(c), 0x20000000, 0x30000000, None, 8, 0x40000000, need - 1, None) == 4
    assert L.hyq_decode_vl_only(ctypes.byref(c), 0x20000000, 0x30000008, None, 8, 0x40000000, need, None) == 3
    assert L.hyq_decode_vl_only(ctypes.byref(c), None, 0x30000000, None, 8, 0x40000000, need, None) == 1


def test_decode_step_argument_checks(L):
    c = _desc()
    step = L.hyq_decode_step
    need = L.hyq_decode_step_workspace(ctypes.byref(c), 8)
    assert need == L.hyq_decode_workspace(ctypes.byref(c), 8) + 256
    q, kn, vn, ring, o, ws = 0x20000000, 0x21000000, 0x22000000, 0x23000000, 0x30000000, 0x40000000
    assert step(ctypes.byref(c), q, None, vn, ring, 64, o, None, 8, ws, need, None) == 1        # k_new
    assert step(ctypes.byref(c), q, kn, vn, ring, 0, o, None, 8, ws, need, None) == 1           # n_q
    assert step(ctypes.byref(c), q, kn, vn, ring, 1025, o, None, 8, ws, need, None) == 1        # n_q
    assert step(ctypes.byref(c), q, kn + 8, vn, ring, 64, o, None, 8, ws, need, None) == 3      # alignment
    assert step(ctypes.byref(c), q, kn, vn, ring + 8, 64, o, None, 8, ws, need, None) == 3
    assert step(ctypes.byref(c), q, kn, vn, ring, 64, o, None, -1, ws, need, None) == 1         # n_ctas
    assert step(ctypes.byref(c), q, kn, vn, ring, 64, o, None, 8, ws, need - 1, None) == 4      # workspace
    assert step(ctypes.byref(c), q, kn, vn, None, 0, o, None, 8, ws, need - 1, None) == 4       # no ring: n_q free
    assert step(ctypes.byref(_desc(window=256)), q, kn, vn, ring, 64, o, None, 8, ws, need, None) == 2


@pytest.mark.parametrize("over,code", [
    (dict(stage_rows=-1), 1), (dict(stage_rows=2000), 1), (dict(stage_rows=64), 1),
    (dict(stage_rows=64, stage_k=0x50008, stage_v=0x60000), 3),
    (dict(stage_rows=64, stage_k=0x50000, stage_v=0x60000), 4),   # valid: stops at the workspace
])
def test_staging_fields_are_checked(L, over, code):
    c = _desc(**over)
    assert L.hyq_decode(ctypes.byref(c), 0x20000000, 0x30000000, None, 8, None, 0, None) == code


def test_vcode_rows_undoes_the_documented_pair_layout():
    """The record's V code area keeps position pairs interleaved by 16 bits
    (include/hyq.h): word h of piece p of slot t has its low 16 bits at byte
    128 i + 16 (p xor 2 (i mod 4)) + 8 h + 2 s, i = t / 2, and its high 16
    bits 4 bytes further, with s = (t mod 2) xor ((t / 4) mod 2).  The
    binding's decoder must give back the plain rows, and the layout must use
    every byte exactly once."""
    import numpy as np

    def off(t, p, h):
        i = t // 2
        return 128 * i + 16 * (p ^ (2 * (i % 4))) + 8 * h + 2 * ((t % 2) ^ ((t // 4) % 2))

    places = sorted(off(t, p, h) + d for t in range(32) for p in range(8) for h in range(2) for d in (0, 1, 4, 5))
    assert places == list(range(2048))
    rng = np.random.default_rng(5)
    rows = rng.integers(0, 256, (2, 3, 32, 64), dtype=np.uint8)
    area = np.zeros((2, 3, 2048), np.uint8)
    for t in range(32):
        for p in range(8):
            for h in range(2):
                o = off(t, p, h)
                word = rows[:, :, t, 8 * p + 4 * h:8 * p + 4 * h + 4]
                area[:, :, o:o + 2] = word[..., 0:2]
                area[:, :, o + 4:o + 6] = word[..., 2:4]
    assert np.array_equal(hyq.vcode_rows(area), rows)
