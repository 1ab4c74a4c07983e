"""hyq_decode_step: the append and the decode of one step in a single launch.

Its results must be identical, bit for bit, to hyq_append followed by
hyq_decode on the same cache: the outputs, the log-sum-exp, and everything
the append leaves behind (INT4 blocks, window, query ring, seq_len).  The
fused path is also checked against the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import Case, compare_decode, dev, host
from fp16_kv_cache_b200 import hyq

pytestmark = pytest.mark.gpu


def _clone_cache(c):
    d = hyq.HybridCache(c.B, c.Hq, c.Hkv, c.cap, c.vl_cap)
    for name in ("blocks", "win_k", "win_v", "vl_k", "vl_v", "vl_pos", "vl_count", "seq_len"):
        getattr(d, name).copy_(getattr(c, name))
    return d


def _state(c, ring):
    torch.cuda.synchronize()
    return {name: host(getattr(c, name)).view(np.uint8).copy()
            for name in ("blocks", "win_k", "win_v", "vl_pos", "vl_count", "seq_len")} | \
        {"ring": None if ring is None else host(ring).view(np.uint8).copy()}


def _run_both(case, steps, n_q=64, seed_q=500, with_ring=True, n_ctas=0):
    """Advance two copies of the cache: A by append + decode, B by the fused
    step; compare every step's outputs and the final state."""
    cfg = case.cfg
    a_cache, b_cache = case.g, _clone_cache(case.g)
    ring_a = ring_b = None
    if with_ring:
        ring_a = torch.zeros(cfg.B, cfg.Hq, n_q, 128, dtype=torch.float16, device="cuda")
        ring_b = ring_a.clone()
    ws_a = hyq.workspace(hyq.hyq_decode_workspace(a_cache, n_ctas))
    ws_b = hyq.workspace(hyq.hyq_decode_step_workspace(b_cache, n_ctas))
    for step in range(steps):
        kn, vn = synth.step_kv(cfg, step)
        q = dev(synth.q(cfg, seed_q + step))
        kd, vd = dev(kn), dev(vn)
        o_a = torch.full_like(q, float("nan"))
        o_b = torch.full_like(q, float("nan"))
        l_a = torch.full((cfg.B, cfg.Hq), float("nan"), dtype=torch.float32, device="cuda")
        l_b = l_a.clone()
        hyq.hyq_append(a_cache, kd, vd, q if with_ring else None, ring_a)
        hyq.hyq_decode(a_cache, q, o_a, ws_a, lse=l_a, n_ctas=n_ctas)
        hyq.hyq_decode_step(b_cache, q, kd, vd, o_b, ws_b, q_ring=ring_b, lse=l_b, n_ctas=n_ctas)
        torch.cuda.synchronize()
        assert torch.equal(o_a.view(torch.int16), o_b.view(torch.int16)), f"step {step}: outputs differ"
        assert torch.equal(l_a.view(torch.int32), l_b.view(torch.int32)), f"step {step}: lse differs"
    sa, sb = _state(a_cache, ring_a), _state(b_cache, ring_b)
    for k in sa:
        if sa[k] is not None:
            assert np.array_equal(sa[k], sb[k]), f"{k} differs after {steps} steps"
    assert a_cache.status() == 0 and b_cache.status() == 0
    return b_cache


@pytest.mark.parametrize("B,Hq,Hkv,T,k,steps,n_ctas", [
    (1, 8, 2, 100, 0, 40, 0),      # window filling: T_old < 128 for the first 28 steps
    (2, 16, 4, 200, 12, 70, 0),    # exiting rows cross a 32-token block boundary
    (1, 32, 8, 4096, 64, 33, 0),   # tiny-4k shape
    (3, 32, 8, 1000, 30, 20, 7),   # several units per block, odd block count
    (2, 8, 1, 517, 9, 12, 1000),   # more blocks than work
    (1, 64, 8, 700, 20, 10, 0),    # G = 8
])
def test_step_equals_append_then_decode(B, Hq, Hkv, T, k, steps, n_ctas):
    cfg = synth.custom(B, Hq, Hkv, T, k, seed=T + 7 * k, steps=steps)
    case = Case(cfg)
    _run_both(case, steps, n_ctas=n_ctas)


def test_step_without_ring():
    cfg = synth.custom(2, 16, 4, 300, 8, seed=5, steps=6)
    _run_both(Case(cfg), 6, with_ring=False)


def test_step_stream_matches_oracle():
    cfg = synth.custom(2, 16, 4, 150, 10, seed=23, steps=60)
    case = Case(cfg)
    ring = torch.zeros(cfg.B, cfg.Hq, 64, 128, dtype=torch.float16, device="cuda")
    ws = hyq.workspace(hyq.hyq_decode_step_workspace(case.g))
    for step in range(cfg.steps):
        kn, vn = synth.step_kv(cfg, step)
        qn = synth.q(cfg, 2000 + step)
        q = dev(qn)
        o = torch.empty_like(q)
        lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
        hyq.hyq_decode_step(case.g, q, dev(kn), dev(vn), o, ws, q_ring=ring, lse=lse)
        case.o.append(kn, vn)
        if step % 11 == 0 or step == cfg.steps - 1:
            torch.cuda.synchronize()
            oo, lo = oracle.decode(case.o, qn)
            compare_decode(host(o.float()).astype(np.float64), host(lse).astype(np.float64), oo, lo)
    assert np.array_equal(host(case.g.seq_len), case.o.seq_len)
    assert case.g.status() == 0


def test_step_past_capacity_sets_status():
    cfg = synth.custom(1, 8, 2, 128, 0, seed=1)
    case = Case(cfg)  # capacity 128, T = 128: no room for one more token
    before = _state(case.g, None)
    kn, vn = synth.step_kv(cfg, 0)
    q = dev(synth.q(cfg, 3))
    o = torch.full_like(q, float("nan"))
    lse = torch.zeros(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_decode_step_workspace(case.g))
    hyq.hyq_decode_step(case.g, q, dev(kn), dev(vn), o, ws, lse=lse)
    torch.cuda.synchronize()
    assert case.g.status() & hyq.DEV_BADLEN
    after = _state(case.g, None)
    for k in before:
        if before[k] is not None:
            assert np.array_equal(before[k], after[k]), k
    assert torch.all(o == 0) and torch.all(torch.isinf(lse)) and torch.all(lse < 0)


def _graph(fn):
    """Capture fn() in a CUDA graph on a side stream, replay it once."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    del g


def _step_inputs(cfg, steps, seed_q):
    kv = [synth.step_kv(cfg, s) for s in range(steps)]
    return ([dev(k) for k, _ in kv], [dev(v) for _, v in kv], [dev(synth.q(cfg, seed_q + s)) for s in range(steps)])


def test_graph_append_then_decode_equals_fused_step():
    """Inside one CUDA graph a decode starts while the append before it (same
    cache) is still running, so the plan it made from the lengths before the
    wait is stale and is made again; the results must still equal the fused
    step's, bit for bit, step by step."""
    cfg = synth.custom(2, 16, 4, 300, 10, seed=41, steps=24)
    case = Case(cfg)
    a_cache, b_cache, warm = case.g, _clone_cache(case.g), _clone_cache(case.g)
    B, Hq, steps = cfg.B, cfg.Hq, cfg.steps
    rings = [torch.zeros(B, Hq, 64, 128, dtype=torch.float16, device="cuda") for _ in range(3)]
    ws_a = hyq.workspace(hyq.hyq_decode_workspace(a_cache))
    ws_b = hyq.workspace(hyq.hyq_decode_step_workspace(b_cache))
    ws_w = hyq.workspace(hyq.hyq_decode_step_workspace(warm))
    ks, vs, qs = _step_inputs(cfg, steps, 700)
    o_a = [torch.full_like(q, float("nan")) for q in qs]
    o_b = [torch.full_like(q, float("nan")) for q in qs]
    l_a = [torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda") for _ in qs]
    l_b = [x.clone() for x in l_a]
    # every kernel once outside the capture (launch attributes), on a scratch copy
    hyq.hyq_append(warm, ks[0], vs[0], qs[0], rings[2])
    hyq.hyq_decode(warm, qs[0], o_a[0], ws_w, lse=l_a[0])
    hyq.hyq_decode_step(warm, qs[0], ks[0], vs[0], o_b[0], ws_w, q_ring=rings[2], lse=l_b[0])
    torch.cuda.synchronize()

    def body():
        for s in range(steps):
            hyq.hyq_append(a_cache, ks[s], vs[s], qs[s], rings[0])
            hyq.hyq_decode(a_cache, qs[s], o_a[s], ws_a, lse=l_a[s])
            hyq.hyq_decode_step(b_cache, qs[s], ks[s], vs[s], o_b[s], ws_b, q_ring=rings[1], lse=l_b[s])

    _graph(body)
    for s in range(steps):
        assert torch.equal(o_a[s].view(torch.int16), o_b[s].view(torch.int16)), f"step {s}: outputs differ"
        assert torch.equal(l_a[s].view(torch.int32), l_b[s].view(torch.int32)), f"step {s}: lse differs"
    sa, sb = _state(a_cache, rings[0]), _state(b_cache, rings[1])
    for k in sa:
        assert np.array_equal(sa[k], sb[k]), f"{k} differs after {steps} steps"
    assert a_cache.status() == 0 and b_cache.status() == 0


@pytest.mark.parametrize("n_ctas", [7, 0])
def test_graph_consecutive_steps_equal_eager(n_ctas):
    """Fused steps on one cache back to back inside a CUDA graph (with 7
    blocks the next launch starts on idle SMs before the previous one has
    written seq_len) equal the same steps launched one by one."""
    cfg = synth.custom(1, 32, 8, 700, 20, seed=43, steps=20)
    case = Case(cfg)
    g_cache, e_cache = case.g, _clone_cache(case.g)
    B, Hq, steps = cfg.B, cfg.Hq, cfg.steps
    rings = [torch.zeros(B, Hq, 64, 128, dtype=torch.float16, device="cuda") for _ in range(2)]
    ws_g = hyq.workspace(hyq.hyq_decode_step_workspace(g_cache, n_ctas))
    ws_e = hyq.workspace(hyq.hyq_decode_step_workspace(e_cache, n_ctas))
    ks, vs, qs = _step_inputs(cfg, steps, 900)
    o_g = [torch.full_like(q, float("nan")) for q in qs]
    o_e = [torch.full_like(q, float("nan")) for q in qs]
    for s in range(steps):
        hyq.hyq_decode_step(e_cache, qs[s], ks[s], vs[s], o_e[s], ws_e, q_ring=rings[1], n_ctas=n_ctas)
        torch.cuda.synchronize()

    def body():
        for s in range(steps):
            hyq.hyq_decode_step(g_cache, qs[s], ks[s], vs[s], o_g[s], ws_g, q_ring=rings[0], n_ctas=n_ctas)

    _graph(body)
    for s in range(steps):
        assert torch.equal(o_g[s].view(torch.int16), o_e[s].view(torch.int16)), f"step {s}: outputs differ"
    sg, se = _state(g_cache, rings[0]), _state(e_cache, rings[1])
    for k in sg:
        assert np.array_equal(sg[k], se[k]), f"{k} differs after {steps} steps"
    assert g_cache.status() == 0 and e_cache.status() == 0


def test_prepared_step_call_matches_the_wrapper():
    """hyq.DecodeStepCall (arguments marshalled once, reused over steps on
    the same buffers) gives the same bits as hyq_decode_step called anew
    each step, on two copies of the cache."""
    cfg = synth.custom(2, 32, 8, 700, 20, seed=61)
    case = Case(cfg)
    a_cache, b_cache = case.g, _clone_cache(case.g)
    ring_a = torch.zeros(cfg.B, cfg.Hq, 64, 128, dtype=torch.float16, device="cuda")
    ring_b = ring_a.clone()
    ws_a = hyq.workspace(hyq.hyq_decode_step_workspace(a_cache, 0))
    ws_b = hyq.workspace(hyq.hyq_decode_step_workspace(b_cache, 0))
    q = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.float16, device="cuda")
    kd = torch.empty(cfg.B, cfg.Hkv, 128, dtype=torch.float16, device="cuda")
    vd = torch.empty_like(kd)
    o_a, o_b = torch.empty_like(q), torch.empty_like(q)
    l_a = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
    l_b = torch.empty_like(l_a)
    call = hyq.DecodeStepCall(b_cache, q, kd, vd, o_b, ws_b, q_ring=ring_b, lse=l_b)
    for step in range(5):
        kn, vn = synth.step_kv(cfg, step)
        q.copy_(dev(synth.q(cfg, 900 + step)))
        kd.copy_(dev(kn))
        vd.copy_(dev(vn))
        hyq.hyq_decode_step(a_cache, q, kd, vd, o_a, ws_a, q_ring=ring_a, lse=l_a)
        call()
        torch.cuda.synchronize()
        assert torch.equal(o_a.view(torch.int16), o_b.view(torch.int16)), f"step {step}"
        assert torch.equal(l_a.view(torch.int32), l_b.view(torch.int32)), f"step {step}"
    sa, sb = _state(a_cache, ring_a), _state(b_cache, ring_b)
    for k in sa:
        assert np.array_equal(sa[k], sb[k]), k


def test_hyq_copy_moves_bytes_between_pinned_host_and_device():
    """hyq_copy (the end-to-end loop's transfer kernel) copies bit for bit
    from pinned host memory to the device, device to device, and back; it
    refuses, on the host and with nothing enqueued, pageable host memory, a
    misaligned pointer and a size that is not a multiple of 16."""
    import ctypes
    g = torch.Generator().manual_seed(3)
    for nbytes in (16, 12288, (1 << 20) + 16):
        src = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
        d1 = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        d2 = torch.empty_like(d1)
        back = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
        hyq.hyq_copy(d1, src)
        hyq.hyq_copy(d2, d1)
        hyq.hyq_copy(back, d2)
        torch.cuda.synchronize()
        assert torch.equal(d1.cpu(), src), nbytes
        assert torch.equal(back, src), nbytes
    lib = hyq._L()
    d = torch.zeros(256, dtype=torch.uint8, device="cuda")
    pageable = torch.ones(256, dtype=torch.uint8)
    assert not pageable.is_pinned()
    vp = ctypes.c_void_p
    assert lib.hyq_copy(vp(d.data_ptr()), vp(pageable.data_ptr()), 256, None) == 1  # HYQ_ERR_INVALID
    assert lib.hyq_copy(vp(d.data_ptr() + 1), vp(d.data_ptr() + 128), 64, None) == 3  # HYQ_ERR_ALIGN
    assert lib.hyq_copy(vp(d.data_ptr()), vp(d.data_ptr() + 128), 40, None) == 1  # not a multiple of 16
    assert lib.hyq_copy(vp(d.data_ptr()), vp(d.data_ptr() + 128), 0, None) == 0  # nothing to do
    with pytest.raises(ValueError):
        hyq.hyq_copy(d, pageable)
    torch.cuda.synchronize()
    assert int(d.sum()) == 0  # nothing was written


def test_step_fed_through_hyq_copy_matches_device_inputs():
    """The end-to-end loop's path -- inputs staged in pinned host memory and
    copied in with hyq_copy, the step through DecodeStepCall, o copied back
    with hyq_copy -- gives the same bits as the step on device tensors."""
    cfg = synth.custom(1, 32, 8, 900, 20, seed=67)
    case = Case(cfg)
    a_cache, b_cache = case.g, _clone_cache(case.g)
    ws_a = hyq.workspace(hyq.hyq_decode_step_workspace(a_cache, 0))
    ws_b = hyq.workspace(hyq.hyq_decode_step_workspace(b_cache, 0))
    nq, nk = cfg.B * cfg.Hq * 128, cfg.B * cfg.Hkv * 128
    din = torch.empty(nq + 2 * nk, dtype=torch.float16, device="cuda")
    dq = din[:nq].view(cfg.B, cfg.Hq, 128)
    dk = din[nq:nq + nk].view(cfg.B, cfg.Hkv, 128)
    dv = din[nq + nk:].view(cfg.B, cfg.Hkv, 128)
    do = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.float16, device="cuda")
    o_a = torch.empty_like(do)
    call = hyq.DecodeStepCall(b_cache, dq, dk, dv, do, ws_b)
    hin = torch.empty(nq + 2 * nk, dtype=torch.float16).pin_memory()
    hout = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.float16).pin_memory()
    for step in range(4):
        kn, vn = synth.step_kv(cfg, step)
        qh = torch.from_numpy(np.ascontiguousarray(synth.q(cfg, 950 + step)))
        hin.copy_(torch.cat([qh.reshape(-1), torch.from_numpy(kn).reshape(-1), torch.from_numpy(vn).reshape(-1)]))
        hyq.hyq_decode_step(a_cache, dev(synth.q(cfg, 950 + step)), dev(kn), dev(vn), o_a, ws_a)
        hyq.hyq_copy(din, hin)
        call()
        hyq.hyq_copy(hout, do)
        torch.cuda.synchronize()
        assert torch.equal(o_a.cpu().view(torch.int16), hout.view(torch.int16)), f"step {step}"
