"""CUDA path vs the CPU oracle, element by element on the same seeded inputs.

Bit-exact: INT4 codes, scale/zero bits, window rows, vertical-line rows,
bitmask, selected positions.  Floating point: decode output within 2e-3 max
abs and 1e-3 relative L2 of the fp64 oracle (the tolerance the hot path is
specified with), log-sum-exp within 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from fp16_kv_cache_b200 import hyq

from gpu_cases import Case, compare_decode, dev, host
from gpu_cases import assert_cache_equal as _assert_cache_equal
from gpu_cases import check_selection as _check_selection
from gpu_cases import select_gpu as _select_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from fp16_kv_cache_b200 import build
    build.build()


def _rows(n, seed):
    rng = np.random.default_rng(seed)
    a, b = n // 3, 2 * n // 3
    rows = rng.standard_normal((n, 128)).astype(np.float32)
    rows[:a, rng.choice(128, 4, replace=False)] *= 8.0
    rows[a:b] *= (10.0 ** rng.uniform(-6, 4, (b - a, 1))).astype(np.float32)
    rows[b:] = rng.integers(-40, 40, (n - b, 128)) * 0.25
    if n > 3:
        rows[0, :32] = 1.5            # constant group
        rows[1, 32:64] = -0.0          # zero group with negative zero
        rows[2, 64:96] = np.linspace(-65504, 65504, 32)
    return rows.astype(np.float16)


# ------------------------------------------------------------------ pack
@pytest.mark.parametrize("n", [1, 2, 17, 1000, 4099])
def test_pack_bitexact(n):
    x = _rows(n, n)
    codes = torch.zeros(n, 64, dtype=torch.uint8, device="cuda")
    sz = torch.zeros(n, 8, dtype=torch.float16, device="cuda")
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    hyq.hyq_pack(dev(x), codes, sz, dev_status=st)
    rc, rs, bad = oracle.pack(x)
    assert bad == 0 and int(st[0]) == 0
    assert np.array_equal(host(codes), rc)
    assert np.array_equal(host(sz).view(np.uint16), rs)


def test_pack_strided_scatter():
    n, stride = 300, 136
    x = np.zeros((n, stride), np.float16)
    x[:, :128] = _rows(n, 77)
    perm = np.random.default_rng(1).permutation(2 * n)[:n].astype(np.int64)
    codes = torch.zeros(2 * n, 64, dtype=torch.uint8, device="cuda")
    sz = torch.zeros(2 * n, 8, dtype=torch.float16, device="cuda")
    hyq.hyq_pack(dev(x), codes, sz, dst_rows=dev(perm))
    rc, rs, _ = oracle.pack(np.ascontiguousarray(x[:, :128]))
    assert np.array_equal(host(codes)[perm], rc)
    assert np.array_equal(host(sz).view(np.uint16)[perm], rs)
    untouched = np.setdiff1d(np.arange(2 * n), perm)
    assert not host(codes)[untouched].any()


def test_pack_flags_non_finite_rows():
    x = _rows(8, 3)
    x[5, 70] = np.inf
    codes = torch.zeros(8, 64, dtype=torch.uint8, device="cuda")
    sz = torch.zeros(8, 8, dtype=torch.float16, device="cuda")
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    hyq.hyq_pack(dev(x), codes, sz, dev_status=st)
    assert int(st[0]) & hyq.DEV_NONFINITE
    rc, rs, _ = oracle.pack(np.delete(x, 5, axis=0))
    assert np.array_equal(np.delete(host(codes), 5, axis=0), rc)


# ------------------------------------------------------------------ cache build
@pytest.mark.parametrize("T,k", [(1, 0), (100, 0), (128, 0), (129, 1), (700, 40), (4096, 64)])
def test_prefill_and_vl_apply_bitexact(T, k):
    cfg = synth.custom(2, 8, 2, T, k, seed=T * 7 + k)
    case = Case(cfg)
    _assert_cache_equal(case)
    assert case.g.status() == 0


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("B,Hq,Hkv,T,k", [
    (1, 8, 2, 1, 0), (1, 8, 2, 17, 0), (2, 8, 2, 128, 0), (2, 8, 2, 129, 1), (1, 8, 8, 200, 5),
    (3, 16, 8, 777, 30), (1, 16, 4, 1000, 60), (2, 64, 8, 2100, 40), (1, 8, 1, 5000, 100),
])
@pytest.mark.parametrize("n_ctas", [0, 1, 7, 1000])
def test_decode_small_shapes(B, Hq, Hkv, T, k, n_ctas):
    cfg = synth.custom(B, Hq, Hkv, T, k, seed=B * 1000 + T + Hq)
    case = Case(cfg)
    q = synth.q(cfg)
    og, lg = case.decode_gpu(q, n_ctas)
    oo, lo = oracle.decode(case.o, q)
    compare_decode(og, lg, oo, lo)
    assert case.g.status() == 0


@pytest.mark.parametrize("B,n_ctas", [(250, 7), (300, 7), (250, 0), (300, 1000)])
def test_decode_many_units_both_block_widths(B, n_ctas):
    """G = 4 with many short units.  2000 units on 7 blocks take the 16-warp
    build (many tiles per block, shared memory fits); 2400 units do not fit
    beside 16 warps' tile rings and take the 12-warp build, as do 2000 units
    on 148 blocks (few tiles per block).  Sampled units (first, last, and
    units inside) against the oracle, plus a bit-exact cache check on them."""
    cfg = synth.custom(B, 32, 8, 200, 8, seed=4000 + B)
    U = cfg.units
    units = [0, 1, U // 3, U // 2 + 5, U - 2, U - 1]
    case = Case(cfg, oracle_units=units)
    q = synth.q(cfg)
    og, lg = case.decode_gpu(q, n_ctas)
    oo, lo = oracle.decode(case.o, q, units=units)
    compare_decode(og, lg, oo, lo, heads=case.heads_of(units))
    _assert_cache_equal(case, units)
    assert case.g.status() == 0


def test_decode_config1_full():
    cfg = synth.config(1)
    case = Case(cfg)
    q = synth.q(cfg)
    og, lg = case.decode_gpu(q)
    oo, lo = oracle.decode(case.o, q)
    compare_decode(og, lg, oo, lo)


def test_decode_config2_full():
    cfg = synth.config(2)
    case = Case(cfg)
    for step in range(2):
        q = synth.q(cfg, step)
        og, lg = case.decode_gpu(q)
        oo, lo = oracle.decode(case.o, q)
        compare_decode(og, lg, oo, lo)


def test_decode_with_every_old_position_fp16_equals_fp16_kernel():
    """Invariant: VL = all of [0, T - W) makes the hybrid decode an exact
    FP16 attention; the FP16 comparator kernel must agree with both."""
    cfg = synth.custom(1, 32, 8, 1500, 1500 - 128, seed=99)
    allpos = np.broadcast_to(np.arange(1500 - 128, dtype=np.int32), (1, 8, 1372)).copy()
    case = Case(cfg, vl=allpos)
    q = synth.q(cfg)
    og, lg = case.decode_gpu(q)
    o16 = torch.empty(1, 32, 128, dtype=torch.float16, device="cuda")
    l16 = torch.empty(1, 32, dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_decode_fp16_workspace(1, 32, 8))
    hyq.hyq_decode_fp16(dev(q), case.Kd, case.Vd, case.g.seq_len, o16, ws, lse=l16)
    torch.cuda.synchronize()
    ref, lref = oracle.decode_fp16(q, case.K, case.V, [1500], 32)
    compare_decode(og, lg, ref, lref)
    compare_decode(host(o16.float()).astype(np.float64), host(l16).astype(np.float64), ref, lref)


@pytest.mark.parametrize("cid", [1, 2])
def test_decode_fp16_comparator(cid):
    cfg = synth.config(cid)
    K, V, _ = synth.kv_full(cfg)
    q = synth.q(cfg)
    seq = torch.full((cfg.B,), cfg.T, dtype=torch.int32, device="cuda")
    o = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.float16, device="cuda")
    lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_decode_fp16_workspace(cfg.B, cfg.Hq, cfg.Hkv))
    hyq.hyq_decode_fp16(dev(q), dev(K), dev(V), seq, o, ws, lse=lse)
    torch.cuda.synchronize()
    ref, lref = oracle.decode_fp16(q, K, V, [cfg.T] * cfg.B, cfg.Hq)
    compare_decode(host(o.float()).astype(np.float64), host(lse).astype(np.float64), ref, lref)


def test_decode_repeated_calls_reuse_workspace():
    cfg = synth.custom(2, 32, 8, 3000, 50, seed=5)
    case = Case(cfg)
    ws = hyq.workspace(hyq.hyq_decode_workspace(case.g, 37))
    for step in range(4):
        q = synth.q(cfg, step)
        qd = dev(q)
        o = torch.empty_like(qd)
        lse = torch.empty(qd.shape[:2], dtype=torch.float32, device="cuda")
        hyq.hyq_decode(case.g, qd, o, ws, lse=lse, n_ctas=37)
        torch.cuda.synchronize()
        oo, lo = oracle.decode(case.o, q)
        compare_decode(host(o.float()).astype(np.float64), host(lse).astype(np.float64), oo, lo)
    counters = host(ws[: 4 * cfg.units].view(torch.int32))
    assert not counters.any(), "tile counters must be left at zero"


# ------------------------------------------------------------------ append
def test_append_stream_matches_oracle():
    cfg = synth.custom(2, 16, 4, 200, 12, seed=17, steps=150)
    case = Case(cfg)
    n_q = 64
    ring = torch.zeros(cfg.B, cfg.Hq, n_q, 128, dtype=torch.float16, device="cuda")
    for step in range(cfg.steps):
        kn, vn = synth.step_kv(cfg, step)
        qn = synth.q(cfg, 1000 + step)
        hyq.hyq_append(case.g, dev(kn), dev(vn), dev(qn), ring)
        case.o.append(kn, vn)
        if step % 37 == 0 or step == cfg.steps - 1:
            og, lg = case.decode_gpu(qn)
            oo, lo = oracle.decode(case.o, qn)
            compare_decode(og, lg, oo, lo)
    torch.cuda.synchronize()
    assert np.array_equal(host(case.g.seq_len), case.o.seq_len)
    case.cfg = synth.custom(2, 16, 4, 350, 12, seed=17)
    _assert_cache_equal(case)
    # the query ring holds the last 64 queries at slot position % 64
    T = 350
    r = host(ring).view(np.uint16)
    for step in range(cfg.steps - 64, cfg.steps):
        pos = 200 + step
        assert np.array_equal(r[:, :, pos % 64], synth.q(cfg, 1000 + step).view(np.uint16))
    assert case.g.status() == 0


def test_append_past_capacity_sets_status():
    cfg = synth.custom(1, 8, 2, 128, 0, seed=1)
    case = Case(cfg)
    kn, vn = synth.step_kv(cfg, 0)
    hyq.hyq_append(case.g, dev(kn), dev(vn))  # 128 -> 129 fits (cap 128)? no: cap == 128
    torch.cuda.synchronize()
    assert case.g.status() & hyq.DEV_BADLEN
    assert int(case.g.seq_len[0]) == 128


# ------------------------------------------------------------------ selection
@pytest.mark.parametrize("B,Hq,Hkv,T,k,n_q", [
    (1, 8, 2, 4096, 64, 64), (2, 16, 8, 700, 20, 64), (1, 8, 1, 300, 10, 64),
    (1, 64, 8, 2000, 40, 64), (1, 4, 4, 500, 16, 8), (2, 32, 8, 1200, 0, 64),
])
def test_select_prefill_mode(B, Hq, Hkv, T, k, n_q):
    cfg = synth.custom(B, Hq, Hkv, T, k, seed=T + k, n_q=n_q)
    case = Case(cfg)
    qs = np.stack([synth.qsel(cfg, b) for b in range(B)])
    pos_g, cs_g = _select_gpu(case, dev(qs), k, k_full=case.Kd)
    pos_o, cs_o, margin = oracle.select_vl(case.o, qs, k, k_full=case.K)
    if k:
        _check_selection(pos_g, cs_g, pos_o, cs_o, margin, T, 128,
                         [(b, h) for b in range(B) for h in range(Hkv)])


def test_select_cache_mode_and_ring_layout():
    cfg = synth.custom(2, 32, 8, 3000, 60, seed=4)
    case = Case(cfg)
    qs = np.stack([synth.qsel(cfg, b) for b in range(2)])
    pos_o, cs_o, margin = oracle.select_vl(case.o, qs, 60)
    # ring layout: row of position p at index p % 64
    T = 3000
    ring = np.zeros_like(qs)
    for i in range(64):
        ring[:, :, (T - 64 + i) % 64] = qs[:, :, i]
    pos_g, cs_g = _select_gpu(case, dev(ring), 60, ring=True)
    _check_selection(pos_g, cs_g, pos_o, cs_o, margin, T, 128, [(b, h) for b in range(2) for h in range(8)])


def test_select_ties_lower_position_wins():
    cfg = synth.custom(1, 8, 2, 600, 0, seed=8)
    K, V, _ = synth.kv_full(cfg, 640)
    qs = synth.qsel(cfg, 0)[None]
    m = qs[0, :4].reshape(-1, 128).astype(np.float64).mean(0)
    dom = (8.0 * np.sqrt(128) * m / np.linalg.norm(m)).astype(np.float16)
    for p in (300, 17, 123):
        K[0, 0, p] = dom
    case = Case(cfg, vl=np.zeros((1, 2, 0), np.int32), cap=640, vl_cap=8)
    kf = dev(K)
    for k, want in ((2, [17, 123]), (3, [17, 123, 300])):
        pos_g, cs_g = _select_gpu(case, dev(qs), k, k_full=kf)
        assert cs_g[0, 0, 17] == cs_g[0, 0, 123] == cs_g[0, 0, 300]
        assert list(pos_g[0, 0]) == want


def test_select_config1_all_units():
    cfg = synth.config(1)
    case = Case(cfg)
    qs = np.stack([synth.qsel(cfg, b) for b in range(cfg.B)])
    pos_g, cs_g = _select_gpu(case, dev(qs), cfg.k, k_full=case.Kd)
    pos_o, cs_o, margin = oracle.select_vl(case.o, qs, cfg.k, k_full=case.K)
    _check_selection(pos_g, cs_g, pos_o, cs_o, margin, cfg.T, 128,
                     [divmod(u, cfg.Hkv) for u in range(cfg.units)])


# ------------------------------------------------------------------ VL apply, cache mode
def test_vl_apply_cache_mode_matches_oracle():
    cfg = synth.custom(2, 16, 4, 900, 30, seed=12)
    case = Case(cfg)
    rng = np.random.default_rng(0)
    new = np.zeros((2, 4, 30), np.int32)
    for b in range(2):
        for h in range(4):
            keep = rng.choice(case.vl[b, h], 18, replace=False)
            fresh = rng.choice(np.setdiff1d(np.arange(900 - 128), case.vl[b, h]), 12, replace=False)
            new[b, h] = np.sort(np.concatenate([keep, fresh]))
    nu = torch.zeros(1, dtype=torch.int32, device="cuda")
    hyq.hyq_vl_apply(case.g, dev(new), n_unpromoted=nu)
    n_o = case.o.apply_vl(new)
    torch.cuda.synchronize()
    assert int(nu[0]) == n_o == 2 * 4 * 12
    _assert_cache_equal(case)
    q = synth.q(cfg, 3)
    og, lg = case.decode_gpu(q)
    oo, lo = oracle.decode(case.o, q)
    compare_decode(og, lg, oo, lo)


def test_select_long_context_cluster_path():
    """More candidates than one block stages (n > 32768): the top-k spreads
    them over the 8 blocks of a cluster and merges its histograms and
    counts through distributed shared memory."""
    cfg = synth.custom(1, 8, 2, 40000, 100, seed=41)
    case = Case(cfg)
    qs = synth.qsel(cfg, 0)[None]
    pos_g, cs_g = _select_gpu(case, dev(qs), cfg.k, k_full=case.Kd)
    pos_o, cs_o, margin = oracle.select_vl(case.o, qs, cfg.k, k_full=case.K)
    _check_selection(pos_g, cs_g, pos_o, cs_o, margin, cfg.T, 128, [(0, 0), (0, 1)])


def test_select_very_long_context_single_block_path():
    """n > 8 x 32768 candidates: more than the cluster's blocks stage, so one
    block per unit runs the radix passes over the column sums in global
    memory."""
    cfg = synth.custom(1, 2, 1, 262400, 60, seed=43)
    case = Case(cfg)
    qs = synth.qsel(cfg, 0)[None]
    pos_g, cs_g = _select_gpu(case, dev(qs), cfg.k, k_full=case.Kd)
    pos_o, cs_o, margin = oracle.select_vl(case.o, qs, cfg.k, k_full=case.K)
    _check_selection(pos_g, cs_g, pos_o, cs_o, margin, cfg.T, 128, [(0, 0)])


@pytest.mark.parametrize("k", [1, 50, 472])
def test_select_mass_ties_take_lowest_positions(k):
    """Every key identical and visible to every selection query: all column
    sums are equal (fixed summation order), so the k lowest positions win;
    k = 472 takes every candidate."""
    cfg = synth.custom(1, 8, 2, 600, 0, seed=9)
    K, V, _ = synth.kv_full(cfg, 640)
    K[:, :, :600] = K[0, 0, 5]
    case = Case(cfg, vl=np.zeros((1, 2, 0), np.int32), cap=640, vl_cap=472)
    qs = synth.qsel(cfg, 0)[None]
    pos_g, cs_g = _select_gpu(case, dev(qs), k, k_full=dev(K))
    n = 600 - 128
    for h in range(2):
        assert np.all(cs_g[0, h, :n] == cs_g[0, h, 0])
        assert list(pos_g[0, h]) == list(range(k))
