"""Paged quantized majority: the cache's 32-position records live in a pool
of pages (a page holds the records of every KV head) and each sequence names
its pages in a block table (include/hyq.h, hyq_cache.block_table).

A paged cache and a contiguous one are built from the same ragged prompt,
the page table a shuffled subset of a larger pool whose pages first hold a
different cache's records (stale codes and stale vertical-line bits, as
recycled pages would).  Every entry point then runs on both: prefill,
selection and vertical-line install (prefill mode), decode, fused decode
steps that cross into fresh pages, a cache-mode re-selection, and the
prefill attention.  The logical records must be equal bit for bit, the
selected positions equal, and the outputs bit-identical (the same kernels
over the same values at the same block count); the decode also matches the
oracle.  Reference: aifromscratch.in explainer, "Key Results & Benchmarks"
(long contexts) and wpnews.pro summary (serving); the paging is this
library's layout, not the pages'."""
import numpy as np
import pytest
import torch

import oracle
import synth
from fp16_kv_cache_b200 import hyq
from gpu_cases import compare_decode, dev, host

pytestmark = pytest.mark.gpu

B, HQ, HKV = 3, 16, 4
TS = [1300, 700, 2049]
CAP = 2304           # positions per sequence (72 blocks)
VL = 24


def _build(seed=3):
    cfg = synth.custom(B, HQ, HKV, max(TS), VL, seed=seed)
    K, V, planted = synth.kv_full(cfg, CAP)
    nb = CAP // 32
    n_pages = B * nb + 40
    rng = np.random.default_rng(seed)
    table = rng.permutation(n_pages)[:B * nb].reshape(B, nb).astype(np.int32)
    gc = hyq.HybridCache(B, HQ, HKV, CAP, VL)
    gp = hyq.HybridCache(B, HQ, HKV, CAP, VL, block_table=table, n_pages=n_pages)
    # stale pool: the records of another prompt, with its vertical lines set
    junk = hyq.HybridCache(B, HQ, HKV, CAP, VL)
    Kj, Vj, pj = synth.kv_full(synth.custom(B, HQ, HKV, max(TS), VL, seed=seed + 100), CAP)
    junk.seq_len.fill_(max(TS))
    hyq.hyq_prefill(junk, dev(Kj), dev(Vj))
    hyq.hyq_vl_apply(junk, dev(pj), dev(Kj), dev(Vj))
    pool = junk.blocks.view(-1, hyq.BLOCK_BYTES)
    gp.blocks.view(-1, hyq.BLOCK_BYTES)[: pool.shape[0]] = pool
    Kd, Vd = dev(K), dev(V)
    # vertical lines below every sequence's window
    vl = np.stack([np.stack([np.sort(rng.choice(min(TS) - 128, VL, replace=False)) for _ in range(HKV)])
                   for _ in range(B)]).astype(np.int32)
    for g in (gc, gp):
        g.seq_len.copy_(torch.tensor(TS, dtype=torch.int32))
        hyq.hyq_prefill(g, Kd, Vd)
        hyq.hyq_vl_apply(g, dev(vl), Kd, Vd)
    torch.cuda.synchronize()
    oc = oracle.OracleCache(B, HQ, HKV, CAP, VL)
    oc.load_prompt(K, V, TS)
    oc.apply_vl(vl, K, V)
    return cfg, K, V, Kd, Vd, gc, gp, oc


def _assert_same_records(gc, gp, T):
    a, b = gc.unpack_blocks(), gp.unpack_blocks()
    for bb in range(B):
        n_old = max(0, int(T[bb]) - 128)
        for x, y in zip(a[:4], b[:4]):  # codes and scale/zero rows of the quantized positions
            assert np.array_equal(x[bb, :, :n_old], y[bb, :, :n_old])
        nw = (n_old + 31) // 32
        assert np.array_equal(a[4][bb, :, :nw], b[4][bb, :, :nw])  # vertical-line bitmask words
    for name in ("win_k", "win_v", "vl_k", "vl_v", "vl_pos", "vl_count", "seq_len"):
        assert torch.equal(getattr(gc, name), getattr(gp, name)), name


def _decode(g, q, n_ctas):
    qd = dev(q)
    o = torch.empty_like(qd)
    lse = torch.empty(B, HQ, dtype=torch.float32, device="cuda")
    hyq.hyq_decode(g, qd, o, hyq.workspace(hyq.hyq_decode_workspace(g, n_ctas)), lse=lse, n_ctas=n_ctas)
    torch.cuda.synchronize()
    return o, lse


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")


def test_paged_prompt_decode_matches_contiguous_and_oracle():
    cfg, K, V, Kd, Vd, gc, gp, oc = _build()
    _assert_same_records(gc, gp, TS)
    q = synth.q(cfg, 4)
    for n_ctas in (0, 7, 300):
        oa, la = _decode(gc, q, n_ctas)
        ob, lb = _decode(gp, q, n_ctas)
        assert torch.equal(oa, ob) and torch.equal(la, lb)
    oo, lo = oracle.decode(oc, q)
    compare_decode(host(ob.float()).astype(np.float64), host(lb).astype(np.float64), oo, lo)
    assert gc.status() == 0 and gp.status() == 0


def test_paged_steps_reselection_and_prefill_attention_match_contiguous():
    cfg, K, V, Kd, Vd, gc, gp, oc = _build(seed=5)
    ring = {id(g): torch.zeros(B, HQ, 64, 128, dtype=torch.float16, device="cuda") for g in (gc, gp)}
    ws = {id(g): hyq.workspace(hyq.hyq_decode_step_workspace(g)) for g in (gc, gp)}
    for step in range(80):  # every sequence crosses at least two 32-position records
        kn, vn = synth.step_kv(cfg, step)
        qd = dev(synth.q(cfg, 50 + step))
        outs = []
        for g in (gc, gp):
            o = torch.empty_like(qd)
            hyq.hyq_decode_step(g, qd, dev(kn), dev(vn), o, ws[id(g)], q_ring=ring[id(g)])
            outs.append(o)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]), step
        oc.append(kn, vn)
    T = [t + 80 for t in TS]
    _assert_same_records(gc, gp, T)
    oo, _ = oracle.decode(oc, synth.q(cfg, 50 + 79))
    err = float(np.abs(host(outs[1].float()).astype(np.float64) - oo).max())
    assert err <= 2e-3, err
    # cache-mode re-selection from the query rings, then its install
    sel = []
    for g in (gc, gp):
        pos = torch.full((B, HKV, VL), -1, dtype=torch.int32, device="cuda")
        hyq.hyq_select_vl(g, ring[id(g)], VL, pos, hyq.workspace(hyq.hyq_select_vl_workspace(g, 64)), q_is_ring=True)
        nu = torch.zeros(1, dtype=torch.int32, device="cuda")
        hyq.hyq_vl_apply(g, pos, n_unpromoted=nu)
        sel.append((pos, nu))
    torch.cuda.synchronize()
    assert torch.equal(sel[0][0], sel[1][0]) and torch.equal(sel[0][1], sel[1][1])
    _assert_same_records(gc, gp, T)
    oa, la = _decode(gc, synth.q(cfg, 7), 0)
    ob, lb = _decode(gp, synth.q(cfg, 7), 0)
    assert torch.equal(oa, ob) and torch.equal(la, lb)
    # the prefill attention reads the vertical-line bitmask through the table
    Q = torch.randn(B, HQ, CAP, 128, device="cuda").half()
    res = []
    for g in (gc, gp):
        o = torch.full((B, HQ, CAP, 128), float("nan"), device="cuda")
        hyq.hyq_prefill_attention(g, Q, Kd, Vd, o, hyq.workspace(hyq.hyq_prefill_attention_workspace(g)))
        res.append(o)
    torch.cuda.synchronize()
    assert torch.equal(res[0].nan_to_num(7.0), res[1].nan_to_num(7.0))
    assert gc.status() == 0 and gp.status() == 0


def test_paged_out_of_range_entry_is_reported():
    """A block-table entry outside the pool that a decode needs raises
    HYQ_DEV_BADLEN; the kernel reads page 0 instead (inside the pool)."""
    cfg, K, V, Kd, Vd, gc, gp, oc = _build(seed=8)
    gp.block_table[1, 3] = gp.n_pages + 5
    gp.clear_status()
    _decode(gp, synth.q(cfg, 1), 0)
    assert gp.status() & hyq.DEV_BADLEN
