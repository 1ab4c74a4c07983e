"""Ragged batches: the sequences of one launch have different lengths,
empty ones included.  Prefill, vertical lines and decode go through the
library; the result is compared with the oracle.  The block counts make the
launch take the unit-aligned split (each unit on whole blocks) or the
contiguous one, and neither may change the result."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import compare_decode, dev, host, round_cap
from fp16_kv_cache_b200 import hyq

pytestmark = pytest.mark.gpu


def _run(lengths, Hq, Hkv, k, n_ctas, seed):
    B = len(lengths)
    cfg = synth.custom(B, Hq, Hkv, max(lengths), 0, seed=seed)
    cap = round_cap(max(lengths))
    K, V, _ = synth.kv_full(cfg, cap)
    vl = None
    if k:
        rng = np.random.default_rng(seed)
        vl = np.stack([np.stack([np.sort(rng.choice(T - 128, k, replace=False)) for _ in range(Hkv)])
                       for T in lengths]).astype(np.int32)
    g = hyq.HybridCache(B, Hq, Hkv, cap, max(k, 1))
    g.seq_len.copy_(torch.tensor(lengths, dtype=torch.int32))
    Kd, Vd = dev(K), dev(V)
    hyq.hyq_prefill(g, Kd, Vd)
    if k:
        hyq.hyq_vl_apply(g, dev(vl), Kd, Vd)
    q = synth.q(cfg, seed)
    qd = dev(q)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_decode_workspace(g, n_ctas))
    hyq.hyq_decode(g, qd, o, ws, lse=lse, n_ctas=n_ctas)
    torch.cuda.synchronize()
    oc = oracle.OracleCache(B, Hq, Hkv, cap, max(k, 1))
    oc.load_prompt(K, V, lengths)
    if k:
        oc.apply_vl(vl, K, V)
    oo, lo = oracle.decode(oc, q)
    assert g.status() == 0
    return host(o.float()).astype(np.float64), host(lse).astype(np.float64), oo, lo


@pytest.mark.parametrize("n_ctas", [0, 7, 300])
def test_ragged_batch_with_empty_and_one_token_sequences(n_ctas):
    """Lengths 0, 700, 129, 4096, 1: the empty sequence's heads get o = 0 and
    lse = -inf, the others match the oracle (the 1-token units are too small
    for the aligned split, so every block count takes the contiguous one)."""
    lengths = [0, 700, 129, 4096, 1]
    og, lg, oo, lo = _run(lengths, 16, 2, 0, n_ctas, seed=77)
    live = [b for b, T in enumerate(lengths) if T > 0]
    compare_decode(og[live], lg[live], oo[live], lo[live])
    assert np.all(og[0] == 0) and np.all(np.isneginf(lg[0]))


@pytest.mark.parametrize("n_ctas", [0, 300, 7])
def test_ragged_batch_with_vertical_lines(n_ctas):
    """Lengths 3000, 700, 4096, 1500 with 16 vertical lines per unit: at 148
    and 300 blocks the split is aligned to units (7 to 63 blocks per unit),
    at 7 blocks it is contiguous."""
    og, lg, oo, lo = _run([3000, 700, 4096, 1500], 8, 2, 16, n_ctas, seed=78)
    compare_decode(og, lg, oo, lo)
