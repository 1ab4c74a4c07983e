"""hyq_decode_vl_only: the vertical-only ablation of the decode (attention
over the vertical-line rows and the window alone, the INT4 majority left
out), checked against the oracle's decode_vl_only and timed."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import Case, compare_decode, host
from fp16_kv_cache_b200 import hyq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,T,k,n_ctas", [
    (1, 8, 2, 700, 40, 0),
    (2, 16, 4, 1000, 0, 0),     # no vertical lines: the window alone
    (3, 32, 8, 100, 0, 7),      # shorter than the window
    (2, 8, 1, 517, 9, 1000),    # more blocks than work
    (1, 64, 8, 2000, 60, 0),    # G = 8
])
def test_vl_only_small_shapes(B, Hq, Hkv, T, k, n_ctas):
    cfg = synth.custom(B, Hq, Hkv, T, k, seed=3 * T + k)
    case = Case(cfg)
    q = synth.q(cfg, 11)
    og, lg = case.decode_gpu(q, n_ctas, decode=hyq.hyq_decode_vl_only)
    oo, lo = oracle.decode_vl_only(case.o, q)
    compare_decode(og, lg, oo, lo)
    assert case.g.status() == 0


def test_vl_only_config2_full_and_timed():
    """Llama-3.1-8B shape at 32K: parity on every head, the cache left as it
    was, and the time of back-to-back launches (printed)."""
    cfg = synth.config(2)
    case = Case(cfg)
    before = [host(t).copy() for t in (case.g.blocks, case.g.vl_k, case.g.win_k, case.g.seq_len)]
    q = synth.q(cfg, 12)
    og, lg = case.decode_gpu(q, decode=hyq.hyq_decode_vl_only)
    oo, lo = oracle.decode_vl_only(case.o, q)
    compare_decode(og, lg, oo, lo)
    after = [host(t) for t in (case.g.blocks, case.g.vl_k, case.g.win_k, case.g.seq_len)]
    assert all(np.array_equal(x, y) for x, y in zip(before, after))
    qd = torch.from_numpy(q).cuda()
    o = torch.empty_like(qd)
    ws = hyq.workspace(hyq.hyq_decode_workspace(case.g))
    for _ in range(3):
        hyq.hyq_decode_vl_only(case.g, qd, o, ws)
    torch.cuda.synchronize()
    reps = 50
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for _ in range(reps):
                hyq.hyq_decode_vl_only(case.g, qd, o, ws)
    torch.cuda.synchronize()
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    us = 1000 * e0.elapsed_time(e1) / reps
    nbytes = cfg.B * cfg.Hkv * (cfg.k + 128) * 512 + cfg.B * cfg.Hq * 512
    print(f"\nvertical-only decode, config 2: {us:.2f} us per launch (CUDA graph, back to back, "
          f"4.6 MB working set in L2), {nbytes / us / 1e3:.1f} GB/s on {nbytes} algorithmic bytes")
    assert case.g.status() == 0
