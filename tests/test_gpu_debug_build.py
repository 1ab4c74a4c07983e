"""Failure detection of the decode kernels, in the debug build of the
library (libhyq_debug.so, the same sources compiled with -DHYQ_DEBUG).

  * Bounded waits: every wait of a decode warp for its tile's bulk copy is
    bounded in wall time; when it runs out the kernel raises
    HYQ_DEV_TIMEOUT, stops issuing copies, lets the copies in flight land,
    finishes its merges and returns.  The test sets a 200 us limit and makes
    every warp's first wait a wait on a barrier that nothing completes (a
    flag nothing sets), so the waits run out: no fault, no trap, no hang.
    It then checks that the launch returned with the status bit set and
    that the context still works: the next decode, with the default wait,
    matches the oracle.
  * Index checks: on valid inputs the debug build's device-side checks never
    raise HYQ_DEV_OOB, and its results equal the release build's.
"""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import synth
from fp16_kv_cache_b200 import build, hyq
from gpu_cases import Case, compare_decode, dev, host

pytestmark = pytest.mark.gpu

DEFAULT_WAIT_NS = 2_000_000_000


@pytest.fixture(scope="module", autouse=True)
def _debug_lib():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    build.build()
    build.build_debug()
    D = hyq.debug_lib()
    yield D
    assert D.hyq_debug_set_wait(DEFAULT_WAIT_NS, 0) == 0


def _decode(case, q, lib_ctx, n_ctas=0):
    qd = dev(q)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full(qd.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
    with lib_ctx():
        ws = hyq.workspace(hyq.hyq_decode_workspace(case.g, n_ctas))
        hyq.hyq_decode(case.g, qd, o, ws, lse=lse, n_ctas=n_ctas)
    torch.cuda.synchronize()
    return o, lse


def test_wait_that_runs_out_returns_timeout_and_leaves_the_context_usable(_debug_lib):
    cfg = synth.custom(2, 32, 8, 8192, 200, seed=606)
    case = Case(cfg)
    q = synth.q(cfg, 1)
    assert _debug_lib.hyq_debug_set_wait(200_000, 1) == 0
    case.g.clear_status()
    _decode(case, q, hyq.using_debug_library)  # returns: the synchronize above completed
    st = case.g.status()
    assert st & hyq.DEV_TIMEOUT, f"no wait ran out (status {st:#x})"
    assert not st & hyq.DEV_OOB
    # the context is intact: the default limit gives the oracle's result again
    assert _debug_lib.hyq_debug_set_wait(DEFAULT_WAIT_NS, 0) == 0
    case.g.clear_status()
    og, lg = _decode(case, q, hyq.using_debug_library)
    oo, lo = oracle.decode(case.o, q)
    compare_decode(host(og.float()).astype(np.float64), host(lg).astype(np.float64), oo, lo)
    assert case.g.status() == 0
    # and so does the release library
    og2, lg2 = _decode(case, q, contextlib.nullcontext)
    assert torch.equal(og, og2) and torch.equal(lg, lg2)


@pytest.mark.parametrize("B,Hq,Hkv,T,k,n_ctas", [
    (1, 8, 2, 4096, 64, 0), (3, 16, 8, 777, 30, 7), (2, 32, 8, 2100, 40, 1000), (1, 8, 1, 129, 1, 0),
])
def test_index_checks_stay_clear_on_valid_inputs(B, Hq, Hkv, T, k, n_ctas):
    cfg = synth.custom(B, Hq, Hkv, T, k, seed=T + 3 * k)
    case = Case(cfg, cap=((T + 40 + 127) // 128) * 128)
    q = synth.q(cfg, 2)
    case.g.clear_status()
    og, lg = _decode(case, q, hyq.using_debug_library, n_ctas)
    assert case.g.status() == 0
    orl, lrl = _decode(case, q, contextlib.nullcontext, n_ctas)
    assert torch.equal(og, orl) and torch.equal(lg, lrl)
    oo, lo = oracle.decode(case.o, q)
    compare_decode(host(og.float()).astype(np.float64), host(lg).astype(np.float64), oo, lo)
    # the fused step through the debug build, a few tokens past the prompt
    ws = hyq.workspace(hyq.hyq_decode_step_workspace(case.g, n_ctas))
    ring = torch.zeros(B, Hq, 64, 128, dtype=torch.float16, device="cuda")
    with hyq.using_debug_library():
        for step in range(40):
            kn, vn = synth.step_kv(cfg, step)
            qn = synth.q(cfg, 100 + step)
            qd = dev(qn)
            o = torch.empty_like(qd)
            lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
            hyq.hyq_decode_step(case.g, qd, dev(kn), dev(vn), o, ws, q_ring=ring, lse=lse, n_ctas=n_ctas)
            case.o.append(kn, vn)
    torch.cuda.synchronize()
    assert case.g.status() == 0
    oo, lo = oracle.decode(case.o, qn)
    compare_decode(host(o.float()).astype(np.float64), host(lse).astype(np.float64), oo, lo)
