"""Staged promotion on the GPU: the ring of the most recently quantized FP16
rows (filled by hyq_prefill, hyq_append and hyq_decode_step) and the
cache-mode hyq_vl_apply that promotes newly selected positions from it,
compared bit for bit with the oracle's OracleCache(stage=64), then the
decode over the promoted set."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import compare_decode, dev, host
from fp16_kv_cache_b200 import hyq

pytestmark = pytest.mark.gpu

S = 64


def _setup(B, Hq, Hkv, T0, cap, vl_cap, old_vl, seed):
    cfg = synth.custom(B, Hq, Hkv, cap, 0, seed=seed)
    K, V, _ = synth.kv_full(cfg, cap)
    g = hyq.HybridCache(B, Hq, Hkv, cap, vl_cap, stage_rows=S)
    g.seq_len.fill_(T0)
    Kd, Vd = dev(K), dev(V)
    hyq.hyq_prefill(g, Kd, Vd)
    oc = oracle.OracleCache(B, Hq, Hkv, cap, vl_cap, stage=S)
    oc.load_prompt(K, V, [T0] * B)
    if old_vl is not None:
        pos = np.broadcast_to(np.asarray(old_vl, np.int32), (B, Hkv, len(old_vl))).copy()
        hyq.hyq_vl_apply(g, dev(pos), Kd, Vd)
        oc.apply_vl(pos, K, V)
    torch.cuda.synchronize()
    return cfg, K, V, g, oc


def _assert_ring(g, oc):
    B, Hkv = g.B, g.Hkv
    sk = host(g.stage_k).view(np.uint16).reshape(B * Hkv, S, 128)
    sv = host(g.stage_v).view(np.uint16).reshape(B * Hkv, S, 128)
    for b in range(B):
        n_old = int(oc.seq_len[b]) - 128
        slots = [p % S for p in range(max(0, n_old - S), n_old)]
        for h in range(Hkv):
            u = b * Hkv + h
            assert np.array_equal(sk[u, slots], oc.stage_k[u, slots])
            assert np.array_equal(sv[u, slots], oc.stage_v[u, slots])


def _assert_vl(g, oc):
    U = g.B * g.Hkv
    *_, mask = g.unpack_blocks()
    mask = mask.reshape(U, g.cap // 32)
    vk = host(g.vl_k).view(np.uint16).reshape(U, g.vl_cap, 128)
    vv = host(g.vl_v).view(np.uint16).reshape(U, g.vl_cap, 128)
    vpos = host(g.vl_pos).reshape(U, g.vl_cap)
    vcnt = host(g.vl_count).reshape(U)
    for u in range(U):
        c = int(oc.vl_count[u])
        assert vcnt[u] == c
        assert np.array_equal(vpos[u, :c], oc.vl_pos[u, :c])
        assert np.array_equal(vk[u, :c], oc.vl_k[u, :c]) and np.array_equal(vv[u, :c], oc.vl_v[u, :c])
        bits = np.unpackbits(mask[u].view(np.uint8), bitorder="little")
        assert np.array_equal(np.flatnonzero(bits), oc.vl_pos[u, :c])


def test_ring_follows_prefill_append_and_fused_step():
    B, Hq, Hkv, T0, cap = 2, 16, 4, 300, 512
    cfg, K, V, g, oc = _setup(B, Hq, Hkv, T0, cap, 8, None, seed=31)
    _assert_ring(g, oc)
    for t in range(T0, T0 + 40):
        hyq.hyq_append(g, dev(K[:, :, t]), dev(V[:, :, t]))
        oc.append(K[:, :, t], V[:, :, t])
    torch.cuda.synchronize()
    _assert_ring(g, oc)
    ws = hyq.workspace(hyq.hyq_decode_step_workspace(g))
    for t in range(T0 + 40, T0 + 80):
        q = dev(synth.q(cfg, t))
        o = torch.empty_like(q)
        hyq.hyq_decode_step(g, q, dev(K[:, :, t]), dev(V[:, :, t]), o, ws)
        oc.append(K[:, :, t], V[:, :, t])
    torch.cuda.synchronize()
    _assert_ring(g, oc)
    assert g.status() == 0


@pytest.mark.parametrize("n_appends,new,unpromoted", [
    # the method's cadence: every position quantized since the selection is promotable
    (64, [5, 90, 260, 280, 300, 335], 0),
    # 30 appends: staged range [238, 302) holds the kept 260; the staged 250 is
    # older than it and stays INT4, the staged 280 is promoted
    (30, [5, 250, 260, 280], 1),
])
def test_cache_mode_promotion_matches_oracle(n_appends, new, unpromoted):
    B, Hq, Hkv, T0, cap = 2, 8, 2, 400, 512
    cfg, K, V, g, oc = _setup(B, Hq, Hkv, T0, cap, 16, [5, 40, 90, 150, 260], seed=32)
    for t in range(T0, T0 + n_appends):
        hyq.hyq_append(g, dev(K[:, :, t]), dev(V[:, :, t]))
        oc.append(K[:, :, t], V[:, :, t])
    pos = np.broadcast_to(np.asarray(new, np.int32), (B, Hkv, len(new))).copy()
    nu = torch.zeros(1, dtype=torch.int32, device="cuda")
    hyq.hyq_vl_apply(g, dev(pos), n_unpromoted=nu)
    n_o = oc.apply_vl(pos)
    torch.cuda.synchronize()
    assert int(nu[0]) == n_o == unpromoted * B * Hkv
    _assert_vl(g, oc)
    q = synth.q(cfg, 9)
    qd = dev(q)
    o = torch.empty_like(qd)
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    hyq.hyq_decode(g, qd, o, hyq.workspace(hyq.hyq_decode_workspace(g)), lse=lse)
    torch.cuda.synchronize()
    oo, lo = oracle.decode(oc, q)
    compare_decode(host(o.float()).astype(np.float64), host(lse).astype(np.float64), oo, lo)
    assert g.status() == 0
