"""hyq_decode_noalloc: the decode entry point that takes no workspace.

It exists for callers that cannot allocate device memory themselves, for
example a plugin whose host application owns the GPU memory budget and
forbids cudaMalloc, or a caller bound to a fixed C interface with no way to
carry a workspace pointer.  Its scratch is an array compiled into the
library.  This file is collected last on purpose, and it builds its own
inputs, so it passes alone in a fresh process as well as after the other
tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from fp16_kv_cache_b200 import build, hyq

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3   # the decode tolerance used by the other GPU tests
REL_L2 = 1e-3


def _cache(cfg):
    """The same prompt and vertical lines in the library's cache (built by
    its own kernels) and in the oracle's."""
    cap = ((cfg.T + 127) // 128) * 128
    K, V, planted = synth.kv_full(cfg, cap)
    Kd, Vd = torch.from_numpy(K).cuda(), torch.from_numpy(V).cuda()
    c = hyq.HybridCache(cfg.B, cfg.Hq, cfg.Hkv, cap, max(cfg.k, 1))
    c.seq_len.fill_(cfg.T)
    hyq.hyq_prefill(c, Kd, Vd)
    oc = oracle.OracleCache(cfg.B, cfg.Hq, cfg.Hkv, cap, max(cfg.k, 1))
    oc.load_prompt(K, V, [cfg.T] * cfg.B)
    if cfg.k:
        hyq.hyq_vl_apply(c, torch.from_numpy(planted).cuda(), Kd, Vd)
        oc.apply_vl(planted, K, V)
    return c, oc


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a))
    assert np.abs(a - b).max() <= MAX_ABS
    assert np.linalg.norm(a - b) / np.linalg.norm(b) <= REL_L2


@pytest.mark.parametrize("cfg", [synth.config(1), synth.custom(3, 32, 8, 5000, 120, seed=77)],
                         ids=["tiny-4k", "b3-5k"])
def test_noalloc_decode_matches_workspace_decode_twice(cfg):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    build.build()
    c, oc = _cache(cfg)
    ws = hyq.workspace(hyq.hyq_decode_workspace(c))
    for step in range(2):  # two calls in a row: the array keeps the last call's contents
        qh = synth.q(cfg, 40 + step)
        q = torch.from_numpy(qh).cuda()
        o_ref = torch.empty_like(q)
        lse_ref = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
        hyq.hyq_decode(c, q, o_ref, ws, lse=lse_ref)
        o = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:2], float("nan"), dtype=torch.float32, device="cuda")
        hyq.hyq_decode_noalloc(c, q, o, lse=lse)
        torch.cuda.synchronize()
        # the same kernel at the same automatic block count over the same
        # inputs: only the scratch differs, so the results are identical
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        # and within the decode tolerance of the fp64 oracle
        o_orc, lse_orc = oracle.decode(oc, qh)
        _close(o, o_orc)
        assert np.abs(lse.cpu().numpy().astype(np.float64) - lse_orc).max() <= 1e-3
    assert c.status() == 0


def test_noalloc_rejects_shapes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required")
    build.build()
    c = hyq.HybridCache(1, 8, 2, 256, 4)
    desc = hyq.hyq_cache.from_buffer_copy(c.desc)
    desc.batch = 2049  # 2049 x 2 kv heads > 4096 units
    q = torch.zeros(1, 8, 128, dtype=torch.float16, device="cuda")
    rc = hyq.lib().hyq_decode_noalloc(ctypes.byref(desc), ctypes.c_void_p(q.data_ptr()),
                                      ctypes.c_void_p(q.data_ptr()), None, None)
    assert rc == 2  # HYQ_ERR_UNSUPPORTED, nothing enqueued
