"""The streaming workload (Qwen3-8B shape, batch 8, 16,384-token prompt):
decode steps that append as they go (hyq_decode_step), with the detector
re-selecting every 64 tokens in cache mode from the ring of the last 64
decode queries.  Sampled units are checked against the oracle, which follows
the same steps: selection indices (bit-exact, on units whose oracle top-k
margin is asserted to exceed 1e-4), the vertical-line rows after each cache-mode apply, the count of
unpromoted positions, and decode outputs along the way."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import Case, compare_decode, dev, host
from fp16_kv_cache_b200 import hyq

pytestmark = pytest.mark.gpu

UNITS = [0, 37]  # (b, h) = (0, 0) and (4, 5)
STEPS = 130      # two re-selections (after steps 63 and 127)


def _selection_ok(pos_g, pos_o, cs_o, margin, b, h, n):
    """Bit-exact selection on a unit whose oracle top-k margin exceeds 1e-4
    (asserted: the sampled units keep margins of 5e-4 or more at both
    re-selections)."""
    assert margin[b, h] > 1e-4, (b, h, margin[b, h])
    assert len(pos_g[b, h]) == len(pos_o[b, h])
    assert np.array_equal(pos_g[b, h], pos_o[b, h]), (b, h, margin[b, h])
    assert np.all(np.diff(pos_g[b, h]) > 0)


def test_streaming_config5_sampled_units():
    cfg = synth.config(5)
    case = Case(cfg, oracle_units=UNITS)
    n_q, k = cfg.n_q, cfg.k
    ring = torch.zeros(cfg.B, cfg.Hq, n_q, 128, dtype=torch.float16, device="cuda")
    ws = hyq.workspace(hyq.hyq_decode_step_workspace(case.g))
    sws = hyq.workspace(hyq.hyq_select_vl_workspace(case.g, n_q))
    nu = torch.zeros(1, dtype=torch.int32, device="cuda")
    heads = case.heads_of(UNITS)
    bi = np.array([b for b, _ in heads]); hi = np.array([h for _, h in heads])
    qs_hist = []
    n_resel = 0
    for step in range(STEPS):
        kn, vn = synth.step_kv(cfg, step)
        qn = synth.q(cfg, step)
        qs_hist.append(qn)
        q = dev(qn)
        o = torch.empty_like(q)
        lse = torch.empty(cfg.B, cfg.Hq, dtype=torch.float32, device="cuda")
        hyq.hyq_decode_step(case.g, q, dev(kn), dev(vn), o, ws, q_ring=ring, lse=lse)
        case.o.append(kn, vn)
        if step in (0, 64, 100, STEPS - 1):
            torch.cuda.synchronize()
            oo, lo = oracle.decode(case.o, qn, units=UNITS)
            og, lg = host(o.float()).astype(np.float64), host(lse).astype(np.float64)
            compare_decode(og[bi, hi][None], lg[bi, hi][None], oo[bi, hi][None], lo[bi, hi][None])
        if (step + 1) % 64 == 0:
            T = cfg.T + step + 1
            # GPU: cache-mode selection from the ring, then the cache-mode apply
            pos = torch.full((cfg.B, cfg.Hkv, k), -1, dtype=torch.int32, device="cuda")
            cs = torch.zeros(cfg.B, cfg.Hkv, case.cap, dtype=torch.float32, device="cuda")
            hyq.hyq_select_vl(case.g, ring, k, pos, sws, out_colsum=cs, q_is_ring=True)
            prev_pos = host(case.g.vl_pos).copy()
            prev_cnt = host(case.g.vl_count).copy()
            nu.zero_()
            hyq.hyq_vl_apply(case.g, pos, n_unpromoted=nu)
            torch.cuda.synchronize()
            pos_g = host(pos)
            # oracle: the same 64 queries in position order
            q_sel = np.stack(qs_hist[-64:], axis=2)  # [B][Hq][64][128]
            pos_o, cs_o, margin = oracle.select_vl(case.o, q_sel, k, units=UNITS)
            for u in UNITS:
                b, h = divmod(u, cfg.Hkv)
                _selection_ok(pos_g, pos_o, cs_o, margin, b, h, T - cfg.W)
                got = host(cs)[b, h, :T - cfg.W].astype(np.float64)
                ref = cs_o[b, h, :T - cfg.W]
                assert np.allclose(got, ref, rtol=2e-4, atol=1e-6 * ref.max())
            # unpromoted = newly selected positions, over every unit
            expect = sum(len(np.setdiff1d(pos_g[b, h], prev_pos[b, h, :prev_cnt[b, h]]))
                         for b in range(cfg.B) for h in range(cfg.Hkv))
            assert int(nu[0]) == expect
            # the oracle applies the GPU's set; its rows must then match on the sampled units
            case.o.apply_vl(pos_g, units=UNITS)
            for u in UNITS:
                b, h = divmod(u, cfg.Hkv)
                n = int(host(case.g.vl_count)[b, h])
                assert n == int(case.o.vl_count[u])
                assert np.array_equal(host(case.g.vl_pos)[b, h, :n], case.o.vl_pos[u, :n])
                assert np.array_equal(host(case.g.vl_k)[b, h, :n].view(np.uint16), case.o.vl_k[u, :n])
            n_resel += 1
    assert n_resel == 2
    assert case.g.status() == 0
