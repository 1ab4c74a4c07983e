"""Helpers shared by the GPU tests: build the same hybrid cache on both sides
(the CUDA library from its own kernels, the oracle from its own quantizer)
from one seeded synthetic input, and compare results."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from fp16_kv_cache_b200 import hyq

# decode tolerance (fp64 oracle vs fp16 output of fp32 arithmetic)
MAX_ABS = 2e-3
REL_L2 = 1e-3
LSE_ABS = 1e-3


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().cpu().numpy()


def round_cap(t):
    return ((t + 127) // 128) * 128


class Case:
    """One workload: synthetic K/V/q on both sides plus the two caches."""

    def __init__(self, cfg: synth.Config, vl=None, cap=None, oracle_units=None, vl_cap=None):
        self.cfg = cfg
        self.T = cfg.T
        self.cap = cap or round_cap(max(cfg.T + cfg.steps, 1))
        self.K, self.V, planted = synth.kv_full(cfg, self.cap)
        self.vl = planted if vl is None else np.asarray(vl, np.int32)
        self.k = self.vl.shape[-1]
        self.vl_cap = vl_cap or max(self.k, cfg.k, 1)
        self.units = oracle_units
        # GPU side: prefill + vertical lines, all through the library
        self.Kd, self.Vd = dev(self.K), dev(self.V)
        self.g = hyq.HybridCache(cfg.B, cfg.Hq, cfg.Hkv, self.cap, self.vl_cap)
        self.g.seq_len.copy_(torch.full((cfg.B,), cfg.T, dtype=torch.int32))
        hyq.hyq_prefill(self.g, self.Kd, self.Vd)
        if self.k:
            hyq.hyq_vl_apply(self.g, dev(self.vl), self.Kd, self.Vd)
        torch.cuda.synchronize()
        # oracle side
        self.o = oracle.OracleCache(cfg.B, cfg.Hq, cfg.Hkv, self.cap, self.vl_cap)
        self.o.load_prompt(self.K, self.V, [cfg.T] * cfg.B, units=oracle_units)
        if self.k:
            self.o.apply_vl(self.vl, self.K, self.V, units=oracle_units)

    def heads_of(self, units):
        G = self.cfg.G
        out = []
        for u in units:
            b, h = divmod(int(u), self.cfg.Hkv)
            out += [(b, h * G + i) for i in range(G)]
        return out

    def decode_gpu(self, q, n_ctas=0, decode=None):
        """hyq_decode (or another entry with its arguments, e.g. the
        vertical-only hyq_decode_vl_only) on the GPU cache."""
        qd = dev(q)
        o = torch.empty_like(qd)
        lse = torch.empty(qd.shape[:2], dtype=torch.float32, device="cuda")
        ws = hyq.workspace(hyq.hyq_decode_workspace(self.g, n_ctas))
        (decode or hyq.hyq_decode)(self.g, qd, o, ws, lse=lse, n_ctas=n_ctas)
        torch.cuda.synchronize()
        return host(o.float()).astype(np.float64), host(lse).astype(np.float64)


def compare_decode(o_gpu, lse_gpu, o_ref, lse_ref, heads=None):
    if heads is not None:
        bi = np.array([b for b, _ in heads])
        hi = np.array([h for _, h in heads])
        o_gpu, o_ref = o_gpu[bi, hi], o_ref[bi, hi]
        lse_gpu, lse_ref = lse_gpu[bi, hi], lse_ref[bi, hi]
    assert np.all(np.isfinite(o_gpu)), "non-finite output"
    err = float(np.abs(o_gpu - o_ref).max())
    rel = float(np.linalg.norm(o_gpu - o_ref) / max(np.linalg.norm(o_ref), 1e-300))
    lerr = float(np.abs(lse_gpu - lse_ref).max())
    assert err <= MAX_ABS, f"max abs {err:.3g} > {MAX_ABS}"
    assert rel <= REL_L2, f"rel L2 {rel:.3g} > {REL_L2}"
    assert lerr <= LSE_ABS, f"lse abs {lerr:.3g} > {LSE_ABS}"
    return err, rel
