"""Prefill hybrid-precision attention (hyq_prefill_attention) against the
oracle's prefill_attention, element by element: the output rows within
2e-3 max-abs and 1e-3 relative L2, the log-sum-exp within 1e-3.

Method: aifromscratch.in explainer, "Two Operational Modes / Prefill Stage";
wpnews.pro summary.  Cases: one and several 128-row query tiles with ragged
ends, rows inside and beyond the window, no vertical lines, planted vertical
lines, every old position a vertical line (all pairs FP16), G = 1, 2, 4, 8,
sequences of different lengths in one batch, and the tiny decode workload's
4K prompt in full."""
import numpy as np
import pytest
import torch

import oracle
import synth
from fp16_kv_cache_b200 import hyq
from gpu_cases import MAX_ABS, REL_L2, LSE_ABS, dev, host

pytestmark = pytest.mark.gpu


def _run(B, Hq, Hkv, Ts, k, seed, vl=None):
    """Prompt of max(Ts) positions per sequence (sequence b holds Ts[b]); the
    cache's vertical lines are `vl` (or the planted ones of the synthetic
    keys); returns GPU and oracle outputs."""
    T = max(Ts)
    cap = ((T + 127) // 128) * 128
    cfg = synth.custom(B, Hq, Hkv, T, k, seed=seed)
    K, V, planted = synth.kv_full(cfg, cap)
    rng = np.random.default_rng(seed + 1)
    Q = np.zeros((B, Hq, cap, 128), np.float16)
    Q[:, :, :T] = rng.standard_normal((B, Hq, T, 128)).astype(np.float32).astype(np.float16)
    pos = planted if vl is None else np.asarray(vl, np.int32)
    n = pos.shape[-1]
    if n:
        assert all(pos[b].max() < Ts[b] - 128 for b in range(B)), "vertical lines lie below the window"
    g = hyq.HybridCache(B, Hq, Hkv, cap, max(n, 1))
    g.seq_len.copy_(torch.tensor(Ts, dtype=torch.int32))
    Kd, Vd = dev(K), dev(V)
    hyq.hyq_prefill(g, Kd, Vd)
    if n:
        hyq.hyq_vl_apply(g, dev(pos), Kd, Vd)
    o = torch.full((B, Hq, cap, 128), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, Hq, cap), float("nan"), dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_prefill_attention_workspace(g))
    hyq.hyq_prefill_attention(g, dev(Q), Kd, Vd, o, ws, lse=lse)
    torch.cuda.synchronize()
    assert g.status() == 0, hex(g.status())
    o_ref, lse_ref = oracle.prefill_attention(Q, K, V, Ts, vl=pos if n else None)
    return host(o).astype(np.float64), host(lse).astype(np.float64), o_ref, lse_ref, Ts


def _compare(og, lg, oo, lo, Ts):
    for b, T in enumerate(Ts):
        a, r = og[b, :, :T], oo[b, :, :T]
        assert np.all(np.isfinite(a)), "non-finite output"
        err = float(np.abs(a - r).max())
        rel = float(np.linalg.norm(a - r) / np.linalg.norm(r))
        lerr = float(np.abs(lg[b, :, :T] - lo[b, :, :T]).max())
        assert err <= MAX_ABS, f"batch {b}: max abs {err:.3g}"
        assert rel <= REL_L2, f"batch {b}: rel L2 {rel:.3g}"
        assert lerr <= LSE_ABS, f"batch {b}: lse {lerr:.3g}"
        # rows past T are left untouched
        assert np.all(np.isnan(og[b, :, T:]))


@pytest.mark.parametrize("B,Hq,Hkv,T,k", [
    (1, 8, 2, 1, 0), (1, 8, 2, 100, 0), (1, 8, 2, 128, 0), (1, 8, 2, 129, 1), (1, 4, 4, 300, 10),
    (1, 8, 1, 700, 30), (2, 16, 8, 515, 12), (1, 16, 2, 1500, 40),
])
def test_prefill_attention_small_shapes(B, Hq, Hkv, T, k):
    og, lg, oo, lo, Ts = _run(B, Hq, Hkv, [T] * B, k, seed=T * 3 + Hq)
    _compare(og, lg, oo, lo, Ts)


def test_prefill_attention_ragged_batch():
    Ts = [1000, 257, 640]
    rng = np.random.default_rng(9)
    vl = np.stack([np.stack([np.sort(rng.choice(min(Ts) - 128, 20, replace=False)) for _ in range(2)])
                   for _ in range(3)]).astype(np.int32)
    og, lg, oo, lo, Ts = _run(3, 8, 2, Ts, 0, seed=71, vl=vl)
    _compare(og, lg, oo, lo, Ts)


def test_prefill_attention_every_old_position_fp16_is_exact_attention():
    """Every position below the window a vertical line: every pair is high
    precision, so the operator is causal FP16 attention; the oracle is
    checked against torch's fp64 SDPA here as well."""
    T, Hq, Hkv = 600, 8, 2
    allpos = np.broadcast_to(np.arange(T - 128, dtype=np.int32), (1, Hkv, T - 128)).copy()
    og, lg, oo, lo, Ts = _run(1, Hq, Hkv, [T], 0, seed=5, vl=allpos)
    _compare(og, lg, oo, lo, Ts)


def test_prefill_attention_tiny_workload_prompt():
    cfg = synth.config(1)  # the 4K prompt of the tiny decode workload, its planted vertical lines
    og, lg, oo, lo, Ts = _run(cfg.B, cfg.Hq, cfg.Hkv, [cfg.T], cfg.k, seed=cfg.seed)
    _compare(og, lg, oo, lo, Ts)
