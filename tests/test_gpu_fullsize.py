"""The four long-context workloads at their full sizes, CUDA path vs the
oracle on sampled units (the oracle takes seconds per unit at 32K-128K
positions): Llama-3.1-8B shape at 32K (batch 1), the batched 32K workload
(batch 16), the 128K workload with an attention sink at position 0 (batch
4) and the streaming workload's 16K prompt (batch 8, Qwen3-8B shape).

Per workload, in the launch configuration the benchmark uses (automatic
block count):
  * hyq_prefill: INT4 codes, scale/zero bits and window rows bit for bit;
  * hyq_select_vl (prefill mode): column sums to fp32 accuracy and the
    selected positions bit for bit, on units whose oracle top-k margin is
    asserted to exceed 1e-4 (the selection is by column totals of attention:
    wpnews.pro summary, hotpaper.ai summary);
  * hyq_vl_apply with the planted set: vertical-line rows, positions and
    bitmask bit for bit;
  * hyq_decode: outputs within 2e-3 max-abs / 1e-3 relative L2.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from fp16_kv_cache_b200 import hyq
from gpu_cases import Case, assert_cache_equal, check_selection, compare_decode, dev, select_gpu

pytestmark = pytest.mark.gpu

# Sampled units (b * 8 + kv head).  Every one of them has an oracle top-k
# margin above 1e-4 (checked inside check_selection).  The 128K set holds
# unit 0, whose position 0 is the planted attention sink.
UNITS = {
    2: list(range(8)),
    3: [17, 37, 64, 77, 127],
    4: [0, 5, 13, 20, 31],
    5: [0, 9, 37, 63],
}


@pytest.fixture(scope="module", params=[2, 3, 4, 5])
def full_case(request):
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    cid = request.param
    cfg = synth.config(cid)
    units = UNITS[cid]
    # the prompt alone first (no vertical lines): codes and window
    case = Case(cfg, vl=np.zeros((cfg.B, cfg.Hkv, 0), np.int32), oracle_units=units, vl_cap=cfg.k)
    yield cid, cfg, units, case
    del case
    torch.cuda.empty_cache()


def test_prefill_codes_bitexact(full_case):
    cid, cfg, units, case = full_case
    assert_cache_equal(case, units)
    assert case.g.status() == 0


def test_select_prefill_mode_bitexact(full_case):
    cid, cfg, units, case = full_case
    qs = np.stack([synth.qsel(cfg, b) for b in range(cfg.B)])
    pos_g, cs_g = select_gpu(case, dev(qs), cfg.k, k_full=case.Kd)
    pos_o, cs_o, margin = oracle.select_vl(case.o, qs, cfg.k, k_full=case.K, units=units)
    check_selection(pos_g, cs_g, pos_o, cs_o, margin, cfg.T, cfg.W, [divmod(u, cfg.Hkv) for u in units])
    if cfg.sink:
        assert pos_g[0, 0, 0] == 0, "the attention sink at position 0 is selected"
    assert case.g.status() == 0


def test_vl_apply_and_decode(full_case):
    cid, cfg, units, case = full_case
    planted = np.stack([np.stack([synth.planted_positions(cfg, b, h) for h in range(cfg.Hkv)])
                        for b in range(cfg.B)])
    hyq.hyq_vl_apply(case.g, dev(planted), case.Kd, case.Vd)
    case.o.apply_vl(planted, case.K, case.V, units=units)
    torch.cuda.synchronize()
    assert_cache_equal(case, units)
    q = synth.q(cfg)
    og, lg = case.decode_gpu(q)
    oo, lo = oracle.decode(case.o, q, units=units)
    compare_decode(og, lg, oo, lo, heads=case.heads_of(units))
    assert case.g.status() == 0
