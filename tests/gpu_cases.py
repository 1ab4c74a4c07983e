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


def assert_cache_equal(case, units=None):
    """Bit-exact comparison of the GPU cache with the oracle's on `units`
    (all by default): INT4 codes, scale/zero bits, window rows, vertical-line
    rows, positions and count, and the block bitmask."""
    g, o, cfg = case.g, case.o, case.cfg
    U = cfg.units
    units = range(U) if units is None else units
    T = cfg.T
    n_old = max(0, T - cfg.W)
    kc, ks, vc, vs, mask = g.unpack_blocks()
    kc, vc = kc.reshape(U, case.cap, 64), vc.reshape(U, case.cap, 64)
    ks, vs = ks.reshape(U, case.cap, 8), vs.reshape(U, case.cap, 8)
    mask = mask.reshape(U, case.cap // 32)
    wk = host(g.win_k).view(np.uint16).reshape(U, 128, 128)
    wv = host(g.win_v).view(np.uint16).reshape(U, 128, 128)
    vlk = host(g.vl_k).view(np.uint16).reshape(U, case.vl_cap, 128)
    vlv = host(g.vl_v).view(np.uint16).reshape(U, case.vl_cap, 128)
    vpos = host(g.vl_pos).reshape(U, case.vl_cap)
    vcnt = host(g.vl_count).reshape(U)
    nw = min(T, cfg.W)
    for u in units:
        assert np.array_equal(kc[u, :n_old], o.k_codes[u, :n_old])
        assert np.array_equal(vc[u, :n_old], o.v_codes[u, :n_old])
        assert np.array_equal(ks[u, :n_old], o.k_sz[u, :n_old])
        assert np.array_equal(vs[u, :n_old], o.v_sz[u, :n_old])
        slots = [p % cfg.W for p in range(T - nw, T)]
        assert np.array_equal(wk[u, slots], o.win_k[u, slots])
        assert np.array_equal(wv[u, slots], o.win_v[u, slots])
        c = int(o.vl_count[u])
        assert vcnt[u] == c
        assert np.array_equal(vpos[u, :c], o.vl_pos[u, :c])
        assert np.array_equal(vlk[u, :c], o.vl_k[u, :c])
        assert np.array_equal(vlv[u, :c], o.vl_v[u, :c])
        bits = np.unpackbits(mask[u].view(np.uint8), bitorder="little")
        assert np.array_equal(np.flatnonzero(bits), np.sort(o.vl_pos[u, :c]))


def select_gpu(case, q_sel, k, k_full=None, ring=False):
    cfg = case.cfg
    pos = torch.full((cfg.B, cfg.Hkv, max(k, 1)), -7, dtype=torch.int32, device="cuda")[..., :k].contiguous()
    cs = torch.zeros(cfg.B, cfg.Hkv, case.cap, dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_select_vl_workspace(case.g, q_sel.shape[2]))
    hyq.hyq_select_vl(case.g, q_sel, k, pos, ws, out_colsum=cs, k_full=k_full, q_is_ring=ring)
    torch.cuda.synchronize()
    return host(pos), host(cs).astype(np.float64)


def check_selection(pos_g, cs_g, pos_o, cs_o, margin, T, W, units, min_margin=1e-4):
    """Column sums to fp32 accuracy and the selected positions bit for bit.
    The inputs must leave the k-th column sum clear of the (k+1)-th by more
    than `min_margin` (relative) on every checked unit, so that the fp32
    GPU sums cannot reorder the boundary: that is asserted, not assumed."""
    n = T - W
    for u in units:
        b, h = u
        ref = cs_o[b, h, :n]
        got = cs_g[b, h, :n]
        assert np.allclose(got, ref, rtol=2e-4, atol=1e-6 * ref.max())
        assert margin[b, h] > min_margin, f"unit {u}: oracle top-k margin {margin[b, h]:.3g} is a near-tie"
        assert len(pos_g[b, h]) == len(pos_o[b, h])
        assert np.array_equal(pos_g[b, h], pos_o[b, h]), (u, margin[b, h])
        assert np.all(np.diff(pos_g[b, h]) > 0)
