"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks one oracle function against a brute-force search, a closed
form, an invariant, or a library routine (numpy's binary16 conversion,
torch's fp64 scaled-dot-product attention / softmax / sort).  Chosen so that a
plausible slip -- a dropped term, a wrong sign, scale or index, a transposed
operand, a wrong rounding rule -- fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

D = 128


# --------------------------------------------------------------- binary16
def test_half_to_double_matches_numpy_for_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_float_to_half_matches_numpy_rounding():
    rng = np.random.default_rng(7)
    vals = [0.0, -0.0, 65504.0, 65519.996, 65520.0, -65520.0, 1e9, 2.0 ** -25,
            3 * 2.0 ** -25, 2.0 ** -24, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 1.0 + 2.0 ** -11,
            1.0 + 3 * 2.0 ** -11, 2049.0, 2051.0, float("inf"), -float("inf")]
    # every exact midpoint between two adjacent finite halves (ties to even)
    h = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mids = ((lo + hi) / 2).astype(np.float32)
    vals += list(mids[::7]) + list(-mids[::11])
    vals += list(rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.uniform(-9, 5, 20000))
    vals = np.array(vals, dtype=np.float32)
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------- quantizer
def _row(values):
    r = np.zeros(D, np.float16)
    r[:] = values
    return r


def test_quantizer_hand_vectors_round_half_even():
    # group 0: min 0, max 15 -> scale exactly 1, zero 0; halves round to even
    x = np.zeros(D, np.float16)
    x[0], x[1], x[2], x[3], x[4], x[5] = 0.0, 15.0, 2.5, 3.5, 14.5, 0.5
    code, s, z, rc = oracle.quantize_row(x)
    assert rc == 0
    assert s[0] == np.float16(1.0).view(np.uint16) and z[0] == 0
    assert list(code[:6]) == [0, 15, 2, 4, 14, 0]
    # the other groups are constant (all 0): scale 0, every code 0
    assert list(s[1:]) == [0, 0, 0] and not code[32:].any()


def test_quantizer_constant_negative_group_and_extremes():
    x = np.full(D, -3.0, np.float16)
    x[32:64] = np.linspace(-65504, 65504, 32).astype(np.float16)
    code, s, z, rc = oracle.quantize_row(x)
    assert rc == 0
    assert s[0] == 0 and z[0] == np.float16(-3.0).view(np.uint16) and not code[:32].any()
    # (65504 - (-65504)) / 15 = 8733.866... -> nearest fp16 is 8736
    assert s[1] == np.float16(8736.0).view(np.uint16)
    assert z[1] == np.float16(-65504.0).view(np.uint16)
    assert code[32] == 0 and code[63] == 15


def test_quantizer_stores_a_negative_zero_minimum_as_plus_zero():
    """Reading of the grid: a -0 minimum is stored as +0, so the bytes do not
    depend on the sign of a zero (group 0 here: -0 then values up to 1.5;
    group 1: all -0, a constant group)."""
    x = np.zeros(D, np.float16)
    x[0] = np.float16(-0.0)
    x[1:32] = np.linspace(0.0, 1.5, 31).astype(np.float16)
    x[32:64] = np.float16(-0.0)
    code, s, z, rc = oracle.quantize_row(x)
    assert rc == 0
    assert z[0] == 0x0000 and z[1] == 0x0000
    assert s[0] == np.float16(np.float32(1.5) / np.float32(15)).view(np.uint16) and s[1] == 0
    assert code[0] == 0 and code[31] == 15


def test_quantizer_divides_instead_of_multiplying_by_the_reciprocal():
    """Codes use an IEEE fp32 division.  Group 0 spans [0, 1.640625], so the
    scale is 1.640625 / 15 = 0.109375 exactly, and 0.7109375, 1.3671875,
    1.5859375 divide to exactly 6.5, 12.5, 14.5: ties to even give 6, 12, 14
    (multiplying by the fp32 reciprocal of the scale lands just above the
    ties and would give 7, 13, 15)."""
    x = np.zeros(D, np.float16)
    x[:5] = [0.0, 1.640625, 0.7109375, 1.3671875, 1.5859375]
    code, s, z, rc = oracle.quantize_row(x)
    assert rc == 0
    assert s[0] == np.float16(0.109375).view(np.uint16) and z[0] == 0
    assert list(code[:5]) == [0, 15, 6, 12, 14]


def test_quantizer_subnormal_scale_clamps_to_15():
    x = np.zeros(D, np.float16)
    x[1] = np.float16(2.0 ** -20)            # max; (2^-20)/15 -> one fp16 ulp 2^-24
    code, s, z, rc = oracle.quantize_row(x)
    assert s[0] == 1                          # smallest subnormal
    assert code[1] == 15 and code[0] == 0     # 16 ulps clamps to 15


def test_quantizer_rejects_non_finite():
    x = np.zeros(D, np.float16)
    x[77] = np.inf
    assert oracle.quantize_row(x)[3] != 0
    x[77] = np.nan
    assert oracle.quantize_row(x)[3] != 0


def _random_rows(n, seed):
    rng = np.random.default_rng(seed)
    a, b = n // 3, 2 * n // 3
    rows = rng.standard_normal((n, D)).astype(np.float32)
    rows[:a, rng.choice(D, 4, replace=False)] *= 8.0                     # outlier channels
    rows[a:b] *= (10.0 ** rng.uniform(-6, 4, (b - a, 1))).astype(np.float32)  # wide dynamic range
    rows[b:] = rng.integers(-40, 40, (n - b, D)) * 0.25                   # many exact .5 ties
    return rows.astype(np.float16)


def test_quantizer_codes_are_nearest_levels_by_brute_force():
    """Independent of the division formula: the code must be the grid level
    c in 0..15 nearest to fl32(x - zero) in units of the stored scale (exact
    fp64 distance), ties to the even c.  Elements whose fp32 quotient sits
    within a few ulps of a .5 boundary are checked separately."""
    rows = _random_rows(600, 11)
    codes_p, sz, bad = oracle.pack(rows)
    assert bad == 0
    codes = oracle.unpack_codes(codes_p)
    levels = np.arange(16, dtype=np.float64)
    n_boundary = 0
    for r in range(rows.shape[0]):
        x32 = rows[r].astype(np.float32)
        for g in range(4):
            xs = x32[32 * g: 32 * g + 32]
            s = sz[r, 2 * g: 2 * g + 1].view(np.float16).astype(np.float64)[0]
            z = sz[r, 2 * g + 1: 2 * g + 2].view(np.float16).astype(np.float64)[0]
            assert z == float(xs.min())
            exact = (float(xs.max()) - float(xs.min())) / 15.0
            # fp32 rounding, then fp16 rounding: within half an fp16 ulp (+fp32 slack)
            if exact > 0:
                ulp = 2.0 ** (math.floor(math.log2(exact)) - 10) if exact >= 2.0 ** -14 else 2.0 ** -24
                assert abs(s - exact) <= 0.5 * ulp * (1 + 2 ** -12) + exact * 2 ** -23
            for i in range(32):
                c = int(codes[r, 32 * g + i])
                if s == 0:
                    assert c == 0
                    continue
                num = float(np.float32(xs[i]) - np.float32(z))  # fl32(x - zero)
                dist = np.abs(num - levels * s)
                best = np.flatnonzero(dist == dist.min())
                want = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
                q = num / s
                frac = q - math.floor(q)
                if abs(frac - 0.5) < 4 * 2.0 ** -23 * max(1.0, abs(q)):
                    n_boundary += 1
                    assert c in (math.floor(q), math.floor(q) + 1) or c in (0, 15)
                else:
                    assert c == want, (r, g, i, c, want, q)
    assert codes.max() <= 15


def test_dequant_error_within_half_scale():
    rows = _random_rows(300, 12)
    cp, sz, _ = oracle.pack(rows)
    xh = oracle.dequant(cp, sz)
    x = rows.astype(np.float64)
    s = sz[:, 0::2].view(np.float16).astype(np.float64)          # [n][4]
    z = sz[:, 1::2].view(np.float16).astype(np.float64)
    s_c = np.repeat(s, 32, axis=1)
    rng_c = np.repeat(x.reshape(-1, 4, 32).max(2) - x.reshape(-1, 4, 32).min(2), 32, axis=1)
    bound = np.maximum(s_c / 2, rng_c - 15 * s_c) * (1 + 2 ** -9) + np.abs(x) * 2 ** -22
    assert np.all(np.abs(xh - x) <= bound + 1e-300)
    # the group minimum is reproduced exactly (code 0)
    assert np.all(xh.reshape(-1, 4, 32).min(2) == np.repeat(z, 1, axis=1))


def test_packed_layout_is_a_bijection_with_stated_pieces():
    seen = set()
    for c in range(D):
        b, hi = oracle.code_slot(c)
        seen.add((b, hi))
        g, w = divmod(c, 32)
        assert b // 8 == w // 4                      # piece p holds channels 4p..4p+3
        assert (b % 8) // 4 == g // 2 and b % 2 == g % 2
        assert hi == w % 2
    assert len(seen) == 128
    # round trip of arbitrary codes through the packed format
    rng = np.random.default_rng(3)
    rows = rng.standard_normal((5, D)).astype(np.float16)
    cp, sz, _ = oracle.pack(rows)
    codes = oracle.unpack_codes(cp)
    for r in range(5):
        for c in range(D):
            b, hi = oracle.code_slot(c)
            assert (cp[r, b] >> (4 * hi)) & 15 == codes[r, c]


# --------------------------------------------------------------- decode
def _build(cfg, vl=None, T=None):
    T = cfg.T if T is None else T
    K, V, planted = synth.kv_full(cfg)
    c = oracle.OracleCache(cfg.B, cfg.Hq, cfg.Hkv, cfg.capacity, max(cfg.k, 1))
    c.load_prompt(K, V, [T] * cfg.B)
    if vl is None:
        vl = planted
    if vl.shape[-1]:
        c.apply_vl(vl, K, V)
    return c, K, V, vl


def _materialize(c, K, V, b, h):
    """K/V rows of unit (b, h) as decode should see them, built from the
    separately pinned dequantizer and the raw fp16 inputs."""
    T = int(c.seq_len[b])
    u = b * c.Hkv + h
    kk = oracle.dequant(c.k_codes[u, :T], c.k_sz[u, :T])
    vv = oracle.dequant(c.v_codes[u, :T], c.v_sz[u, :T])
    for i in range(c.vl_count[u]):
        p = c.vl_pos[u, i]
        kk[p] = K[b, h, p].astype(np.float64)
        vv[p] = V[b, h, p].astype(np.float64)
    for p in range(max(0, T - c.W), T):
        kk[p] = K[b, h, p].astype(np.float64)
        vv[p] = V[b, h, p].astype(np.float64)
    return kk, vv


def _sdpa(q, kk, vv, G):
    """torch fp64 attention; q [Hq_unit][128], kk/vv [T][128]."""
    qt = torch.from_numpy(q.astype(np.float64))[None, :, None, :]
    kt = torch.from_numpy(kk)[None, None].expand(1, G, -1, -1)
    vt = torch.from_numpy(vv)[None, None].expand(1, G, -1, -1)
    o = F.scaled_dot_product_attention(qt, kt, vt)[0, :, 0]
    lse = torch.logsumexp((qt[0, :, 0] @ kt[0, 0].T) / math.sqrt(D), dim=-1)
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("T", [1, 50, 128, 129, 700])
def test_decode_matches_torch_attention_over_materialized_hybrid_cache(T):
    cfg = synth.custom(2, 8, 2, T, min(17, max(T - 128, 0)), seed=5)
    c, K, V, vl = _build(cfg)
    qv = synth.q(cfg)
    o, lse = oracle.decode(c, qv)
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            kk, vv = _materialize(c, K, V, b, h)
            ro, rl = _sdpa(qv[b, h * 4:(h + 1) * 4], kk, vv, 4)
            assert np.allclose(o[b, h * 4:(h + 1) * 4], ro, rtol=0, atol=1e-12)
            assert np.allclose(lse[b, h * 4:(h + 1) * 4], rl, rtol=0, atol=1e-11)


def test_decode_all_fp16_equals_exact_attention_and_fp16_oracle():
    cfg = synth.custom(1, 8, 2, 600, 600 - 128, seed=9)
    allpos = np.broadcast_to(np.arange(600 - 128, dtype=np.int32), (1, 2, 472)).copy()
    c, K, V, _ = _build(cfg, vl=allpos)
    qv = synth.q(cfg)
    o, lse = oracle.decode(c, qv)
    o2, lse2 = oracle.decode_fp16(qv, K, V, [600], 8)
    for h in range(2):
        ro, rl = _sdpa(qv[0, h * 4:(h + 1) * 4], K[0, h].astype(np.float64), V[0, h].astype(np.float64), 4)
        assert np.allclose(o[0, h * 4:(h + 1) * 4], ro, atol=1e-12, rtol=0)
        assert np.allclose(o2[0, h * 4:(h + 1) * 4], ro, atol=1e-12, rtol=0)
        assert np.allclose(lse2[0, h * 4:(h + 1) * 4], rl, atol=1e-11, rtol=0)


def test_decode_single_token_returns_its_value():
    cfg = synth.custom(1, 4, 1, 1, 0, seed=2)
    c, K, V, _ = _build(cfg)
    o, lse = oracle.decode(c, synth.q(cfg))
    assert np.array_equal(o[0], np.repeat(V[0, 0, :1].astype(np.float64), 4, 0))


def test_decode_zero_query_is_mean_of_value_multiset():
    cfg = synth.custom(1, 4, 1, 400, 20, seed=4)
    c, K, V, vl = _build(cfg)
    o, lse = oracle.decode(c, np.zeros((1, 4, D), np.float16))
    _, vv = _materialize(c, K, V, 0, 0)
    assert np.allclose(o[0], vv.mean(0)[None], atol=1e-13, rtol=0)
    assert np.allclose(lse[0], math.log(400), atol=1e-12)


def test_decode_one_dominant_key_returns_its_value():
    cfg = synth.custom(1, 4, 1, 300, 0, seed=6)
    K, V, _ = synth.kv_full(cfg)
    K = K * np.float16(0.01)
    qv = np.zeros((1, 4, D), np.float16)
    qv[0, :, 0] = 60.0
    K[0, 0, 290, :] = 0
    K[0, 0, 290, 0] = 60.0                     # logit 3600/sqrt(128) ~ 318 above the rest
    c = oracle.OracleCache(1, 4, 1, 300, 1)
    c.load_prompt(K, V, [300])
    o, _ = oracle.decode(c, qv)
    assert np.allclose(o[0], V[0, 0, 290].astype(np.float64)[None], atol=1e-12)


def test_decode_gqa_groups_read_their_own_kv_head():
    cfg = synth.custom(1, 8, 4, 200, 0, seed=8)          # G = 2
    c, K, V, _ = _build(cfg)
    qv = synth.q(cfg)
    o, _ = oracle.decode(c, qv)
    for h in range(8):
        kk, vv = _materialize(c, K, V, 0, h // 2)
        ro, _ = _sdpa(qv[0, h:h + 1], kk, vv, 1)
        assert np.allclose(o[0, h], ro[0], atol=1e-12)


# ------------------------------------------------ vertical-only ablation
@pytest.mark.parametrize("T,k", [(700, 17), (300, 0), (100, 0), (1, 0)])
def test_decode_vl_only_is_attention_over_vertical_lines_and_window(T, k):
    """The ablation's multiset, gathered here from the raw fp16 inputs: the
    selected positions plus the last W positions, nothing quantized."""
    cfg = synth.custom(2, 8, 2, T, k, seed=13)
    c, K, V, vl = _build(cfg)
    qv = synth.q(cfg, 4)
    o, lse = oracle.decode_vl_only(c, qv)
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            keep = sorted(set(vl[b, h, :k].tolist()) | set(range(max(0, T - 128), T)))
            ro, rl = _sdpa(qv[b, h * 4:(h + 1) * 4], K[b, h, keep].astype(np.float64),
                           V[b, h, keep].astype(np.float64), 4)
            assert np.allclose(o[b, h * 4:(h + 1) * 4], ro, rtol=0, atol=1e-12)
            assert np.allclose(lse[b, h * 4:(h + 1) * 4], rl, rtol=0, atol=1e-11)


def test_decode_vl_only_with_every_old_position_selected_equals_hybrid():
    cfg = synth.custom(1, 8, 2, 600, 600 - 128, seed=9)
    allpos = np.broadcast_to(np.arange(600 - 128, dtype=np.int32), (1, 2, 472)).copy()
    c, K, V, _ = _build(cfg, vl=allpos)
    qv = synth.q(cfg, 5)
    o, lse = oracle.decode_vl_only(c, qv)
    o2, lse2 = oracle.decode(c, qv)
    assert np.allclose(o, o2, rtol=0, atol=1e-12) and np.allclose(lse, lse2, rtol=0, atol=1e-11)


def test_decode_vl_only_drops_exactly_the_quantized_positions():
    """Moving one position from the quantized majority into the vertical
    lines changes the ablation's result and leaves the set of the others."""
    cfg = synth.custom(1, 4, 1, 400, 8, seed=21)
    c, K, V, vl = _build(cfg)
    qv = synth.q(cfg, 6)
    o1, _ = oracle.decode_vl_only(c, qv)
    extra = next(p for p in range(400 - 128) if p not in set(vl[0, 0].tolist()))
    vl2 = np.sort(np.append(vl[0, 0], extra)).astype(np.int32)[None, None]
    c2 = oracle.OracleCache(1, 4, 1, cfg.capacity, 9)
    c2.load_prompt(K, V, [400])
    c2.apply_vl(vl2, K, V)
    o2, _ = oracle.decode_vl_only(c2, qv)
    keep = sorted(set(vl2[0, 0].tolist()) | set(range(400 - 128, 400)))
    ro, _ = _sdpa(qv[0], K[0, 0, keep].astype(np.float64), V[0, 0, keep].astype(np.float64), 4)
    assert np.allclose(o2[0], ro, rtol=0, atol=1e-12)
    assert not np.allclose(o1, o2, rtol=0, atol=1e-9)


def test_ablation_keeping_the_quantized_tail_cuts_the_error():
    """The ablation the pages discuss (Table twelve: dropping the long-tail
    positions costs accuracy), reproduced on the synthetic workload: against
    exact FP16 attention, the hybrid cache's error is a small fraction of the
    vertical-only variant's, for random decode queries and for queries drawn
    like the selection queries."""
    cfg = synth.config(1)
    K, V, planted = synth.kv_full(cfg)
    c = oracle.OracleCache(cfg.B, cfg.Hq, cfg.Hkv, cfg.capacity, cfg.k)
    c.load_prompt(K, V, [cfg.T] * cfg.B)
    c.apply_vl(planted, K, V)
    for q in (synth.q(cfg, 100), synth.qsel(cfg, 0)[None, :, cfg.n_q - 1]):
        ref, _ = oracle.decode_fp16(q, K, V, [cfg.T], cfg.Hq)
        err = {}
        for name, fn in (("hybrid", oracle.decode), ("vl_only", oracle.decode_vl_only)):
            o, _ = fn(c, q)
            err[name] = np.linalg.norm(o - ref) / np.linalg.norm(ref)
        assert 5 * err["hybrid"] < err["vl_only"], err


# ------------------------------------------------------- prefill operator
def _causal_sdpa(Q, K, V, T, G):
    """torch fp64 causal attention for one unit: Q [G][T][128], K/V [T][128]."""
    qt = torch.from_numpy(Q[:, :T].astype(np.float64))[None]
    kt = torch.from_numpy(K[:T].astype(np.float64))[None, None].expand(1, G, -1, -1)
    vt = torch.from_numpy(V[:T].astype(np.float64))[None, None].expand(1, G, -1, -1)
    o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)[0]
    s_ = (qt[0] @ kt[0, 0].T) / math.sqrt(D)
    s_ = s_.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), -math.inf)
    return o.numpy(), torch.logsumexp(s_, dim=-1).numpy()


def _prefill_inputs(T, k, seed, grid_q=False):
    cfg = synth.custom(1, 4, 1, T, k, seed=seed)
    K, V, vl = synth.kv_full(cfg)
    rng = np.random.default_rng(seed)
    if grid_q:   # every group holds 0 and 15 * 0.25: quantizing q is lossless
        c = rng.integers(0, 16, (1, 4, K.shape[2], D))
        c[..., 0::32], c[..., 1::32] = 0, 15
        Q = (c * 0.25).astype(np.float16)
    else:
        Q = rng.standard_normal((1, 4, K.shape[2], D)).astype(np.float16)
    return cfg, Q, K, V, vl


def test_prefill_rows_inside_the_window_are_exact_causal_attention():
    T = 300
    cfg, Q, K, V, vl = _prefill_inputs(T, 8, seed=71)
    o, lse = oracle.prefill_attention(Q, K, V, [T], vl)
    ro, rl = _causal_sdpa(Q[0], K[0, 0], V[0, 0], T, 4)
    assert np.allclose(o[0, :, :128], ro[:, :128], rtol=0, atol=1e-12)
    assert np.allclose(lse[0, :, :128], rl[:, :128], rtol=0, atol=1e-11)
    assert np.abs(o[0, :, 200:T] - ro[:, 200:]).max() > 1e-6   # the quantized majority is in effect


def test_prefill_with_every_old_position_selected_is_exact_causal_attention():
    T = 260
    cfg, Q, K, V, _ = _prefill_inputs(T, 0, seed=72)
    allpos = np.arange(T - 128, dtype=np.int32)[None, None]
    o, lse = oracle.prefill_attention(Q, K, V, [T], allpos)
    ro, rl = _causal_sdpa(Q[0], K[0, 0], V[0, 0], T, 4)
    assert np.allclose(o[0, :, :T], ro, rtol=0, atol=1e-12)
    assert np.allclose(lse[0, :, :T], rl, rtol=0, atol=1e-11)


@pytest.mark.parametrize("i", [130, 260, 371, 499])
def test_prefill_row_with_grid_queries_equals_decode_of_the_prefix(i):
    """With q on the INT4 grid, row i is the decode of the cache holding the
    first i + 1 positions (same vertical lines, window = the last W of them)."""
    T = 500
    cfg, Q, K, V, vl = _prefill_inputs(T, 16, seed=73, grid_q=True)
    o, lse = oracle.prefill_attention(Q, K, V, [T], vl)
    Ti = i + 1
    c = oracle.OracleCache(1, 4, 1, cfg.capacity, 16)
    c.load_prompt(K, V, [Ti])
    pre = vl[0, 0][vl[0, 0] < Ti - 128]
    if len(pre):
        c.apply_vl(pre[None, None].astype(np.int32), K, V)
    od, ld = oracle.decode(c, Q[:, :, i])
    assert np.allclose(o[0, :, i], od[0], rtol=0, atol=1e-12)
    assert np.allclose(lse[0, :, i], ld[0], rtol=0, atol=1e-11)


def test_prefill_is_causal():
    T = 400
    cfg, Q, K, V, vl = _prefill_inputs(T, 8, seed=74)
    o1, _ = oracle.prefill_attention(Q, K, V, [T], vl)
    K2, V2 = K.copy(), V.copy()
    K2[:, :, 301:T] = -K2[:, :, 301:T]
    V2[:, :, 301:T] = V2[:, :, 301:T] * np.float16(2)
    o2, _ = oracle.prefill_attention(Q, K2, V2, [T], vl)
    assert np.array_equal(o1[:, :, :301], o2[:, :, :301])
    assert not np.allclose(o1[:, :, 301:T], o2[:, :, 301:T])


# --------------------------------------------------------------- selection
def _select_by_torch(q_rows, kk, T, n_cand, k, n_q, G):
    """Brute force: full fp64 causal softmax, column sums, stable sort."""
    qt = torch.from_numpy(q_rows.astype(np.float64))         # [G][n_q][128]
    kt = torch.from_numpy(kk)                                # [T][128]
    s = (qt @ kt.T) / math.sqrt(D)                           # [G][n_q][T]
    qpos = torch.arange(T - n_q, T)[:, None]
    mask = torch.arange(T)[None, :] <= qpos
    s = s.masked_fill(~mask[None], float("-inf"))
    p = torch.softmax(s, dim=-1)
    cs = p.sum(dim=(0, 1))[:n_cand]
    order = sorted(range(n_cand), key=lambda j: (-cs[j].item(), j))
    return np.sort(np.array(order[:k], np.int32)), cs.numpy()


@pytest.mark.parametrize("T,k,Hkv,G", [(64 + 128, 8, 1, 1), (256, 16, 2, 4), (200, 5, 1, 2), (400, 16, 2, 8)])
def test_select_matches_bruteforce_prefill_mode(T, k, Hkv, G):
    cfg = synth.custom(1, Hkv * G, Hkv, T, min(k, T - 128), seed=T + k)
    K, V, _ = synth.kv_full(cfg)
    c = oracle.OracleCache(1, Hkv * G, Hkv, T, k)
    c.load_prompt(K, V, [T])
    qs = synth.qsel(cfg, 0)[None]
    pos, cs, margin = oracle.select_vl(c, qs, k, k_full=K)
    for h in range(Hkv):
        want, wcs = _select_by_torch(qs[0, h * G:(h + 1) * G], K[0, h].astype(np.float64), T, T - 128, k, 64, G)
        assert np.array_equal(pos[0, h], want)
        assert np.allclose(cs[0, h, :T - 128], wcs, rtol=1e-12, atol=1e-15)
        assert not cs[0, h, T - 128:].any()


def test_select_cache_mode_scores_the_hybrid_view():
    cfg = synth.custom(1, 8, 2, 500, 12, seed=21)
    c, K, V, vl = _build(cfg)
    qs = synth.qsel(cfg, 0)[None]
    pos, cs, _ = oracle.select_vl(c, qs, 12)
    for h in range(2):
        kk, _ = _materialize(c, K, V, 0, h)
        want, wcs = _select_by_torch(qs[0, h * 4:(h + 1) * 4], kk, 500, 500 - 128, 12, 64, 4)
        assert np.array_equal(pos[0, h], want)
        assert np.allclose(cs[0, h, :372], wcs, rtol=1e-12, atol=1e-15)


def test_select_ties_go_to_the_lower_position():
    cfg = synth.custom(1, 4, 1, 300, 0, seed=31)
    K, V, _ = synth.kv_full(cfg)
    qs = synth.qsel(cfg, 0)[None]
    c = oracle.OracleCache(1, 4, 1, 300, 4)
    c.load_prompt(K, V, [300])
    m = qs[0].reshape(-1, D).astype(np.float64).mean(0)
    dominant = (8.0 * math.sqrt(D) * m / np.linalg.norm(m)).astype(np.float16)
    K2 = K.copy()
    for p in (150, 20, 90):                  # three identical, dominant key rows
        K2[0, 0, p] = dominant
    pos, cs, margin = oracle.select_vl(c, qs, 2, k_full=K2)
    assert cs[0, 0, 20] == cs[0, 0, 90] == cs[0, 0, 150]
    assert np.sort(cs[0, 0, :172])[-4] < cs[0, 0, 20]     # the copies are the top 3
    assert list(pos[0, 0]) == [20, 90]
    assert margin[0, 0] == 0.0
    pos3, _, _ = oracle.select_vl(c, qs, 3, k_full=K2)
    assert list(pos3[0, 0]) == [20, 90, 150]


def test_select_margin_definition():
    cfg = synth.custom(1, 4, 1, 400, 10, seed=41)
    K, V, _ = synth.kv_full(cfg)
    c = oracle.OracleCache(1, 4, 1, 400, 10)
    c.load_prompt(K, V, [400])
    qs = synth.qsel(cfg, 0)[None]
    pos, cs, margin = oracle.select_vl(c, qs, 10, k_full=K)
    v = np.sort(cs[0, 0, :272])[::-1]
    assert math.isclose(margin[0, 0], (v[9] - v[10]) / v[9], rel_tol=1e-12)
    # column sums of probabilities: total mass over all keys is rows exactly,
    # and the candidates carry at most that
    assert cs[0, 0].sum() <= 64 * 4 + 1e-9


# --------------------------------------------------------------- cache bookkeeping
def test_append_equals_loading_the_longer_prompt():
    """Streaming T0 -> T0 + n by append must give the same cache as loading
    the T0 + n prompt directly (every token packed on leaving the window)."""
    cfg = synth.custom(2, 8, 2, 300, 0, seed=51)
    K, V, _ = synth.kv_full(cfg)
    a = oracle.OracleCache(2, 8, 2, 320, 1)
    a.load_prompt(K, V, [140, 140])
    for t in range(140, 300):
        a.append(K[:, :, t], V[:, :, t])
    b_ = oracle.OracleCache(2, 8, 2, 320, 1)
    b_.load_prompt(K, V, [300, 300])
    assert np.array_equal(a.seq_len, b_.seq_len)
    for name in ("k_codes", "v_codes", "k_sz", "v_sz", "win_k", "win_v"):
        assert np.array_equal(getattr(a, name), getattr(b_, name)), name


def test_cache_mode_reselection_keeps_only_known_fp16_rows():
    cfg = synth.custom(1, 4, 1, 400, 6, seed=61)
    K, V, _ = synth.kv_full(cfg)
    c = oracle.OracleCache(1, 4, 1, 400, 8)
    c.load_prompt(K, V, [400])
    c.apply_vl(np.array([[[3, 10, 50, 60, 200, 250]]]), K, V)
    n = c.apply_vl(np.array([[[10, 11, 60, 201, 250, 260]]]))
    assert n == 3
    assert list(c.vl_pos[0, :c.vl_count[0]]) == [10, 60, 250]
    assert np.array_equal(c.vl_k[0, 1], K[0, 0, 60].view(np.uint16))


def test_staging_ring_holds_the_most_recently_quantized_rows():
    """With staging, the ring holds the FP16 rows of [T - W - 64, T - W):
    the same after streaming 140 -> 300 as after loading the 300 prompt, and
    equal to the raw input rows."""
    cfg = synth.custom(2, 8, 2, 300, 0, seed=52)
    K, V, _ = synth.kv_full(cfg)
    a = oracle.OracleCache(2, 8, 2, 320, 1, stage=64)
    a.load_prompt(K, V, [140, 140])
    for t in range(140, 300):
        a.append(K[:, :, t], V[:, :, t])
    b_ = oracle.OracleCache(2, 8, 2, 320, 1, stage=64)
    b_.load_prompt(K, V, [300, 300])
    for name in ("stage_k", "stage_v", "k_codes", "win_k"):
        assert np.array_equal(getattr(a, name), getattr(b_, name)), name
    for b in range(2):
        for h in range(2):
            for p in range(300 - 128 - 64, 300 - 128):
                assert np.array_equal(a.stage_k[b * 2 + h, p % 64], K[b, h, p].view(np.uint16))
                assert np.array_equal(a.stage_v[b * 2 + h, p % 64], V[b, h, p].view(np.uint16))
                assert a.staged(b, p)
            assert not a.staged(b, 300 - 128 - 65) and not a.staged(b, 300 - 128)


@pytest.mark.parametrize("stage,kept,unpromoted", [
    # staged range [208, 272): 260 is promoted; 230 is staged but older than
    # the kept 250, so it stays INT4 (promoted rows follow the kept rows)
    (64, [10, 60, 250, 260], 3),
    (0, [10, 60, 250], 4),              # without staging only known FP16 rows stay
])
def test_cache_mode_reselection_promotes_staged_positions(stage, kept, unpromoted):
    cfg = synth.custom(1, 4, 1, 400, 6, seed=62)
    K, V, _ = synth.kv_full(cfg)
    c = oracle.OracleCache(1, 4, 1, 400, 8, stage=stage)
    c.load_prompt(K, V, [400])
    c.apply_vl(np.array([[[3, 10, 50, 60, 200, 250]]]), K, V)
    n = c.apply_vl(np.array([[[10, 11, 60, 201, 230, 250, 260]]]))
    assert n == unpromoted
    assert list(c.vl_pos[0, :c.vl_count[0]]) == kept
    for i, p in enumerate(kept):
        assert np.array_equal(c.vl_k[0, i], K[0, 0, p].view(np.uint16))
        assert np.array_equal(c.vl_v[0, i], V[0, 0, p].view(np.uint16))
    qv = synth.q(cfg, 7)
    o, _ = oracle.decode(c, qv)
    kk, vv = _materialize(c, K, V, 0, 0)
    ro, _ = _sdpa(qv[0], kk, vv, 4)
    assert np.allclose(o[0], ro, rtol=0, atol=1e-12)


def test_staged_promotion_at_the_method_cadence_promotes_every_recent_pick():
    """Re-selecting every 64 appends: every newly selected position that left
    the window since the previous selection is promoted (none unpromoted)."""
    cfg = synth.custom(1, 4, 1, 600, 0, seed=63)
    K, V, _ = synth.kv_full(cfg)
    c = oracle.OracleCache(1, 4, 1, 640, 16, stage=64)
    c.load_prompt(K, V, [400])
    c.apply_vl(np.array([[[5, 40, 90, 150, 260]]], np.int32), K, V)   # all < 400 - 128 = 272
    for t in range(400, 464):
        c.append(K[:, :, t], V[:, :, t])
    # T = 464: the 64 positions [272, 336) left the window since the selection
    new = np.array([[[5, 90, 260, 280, 300, 335]]], np.int32)
    assert c.apply_vl(new) == 0
    assert list(c.vl_pos[0, :c.vl_count[0]]) == [5, 90, 260, 280, 300, 335]
    for i, p in enumerate([5, 90, 260, 280, 300, 335]):
        assert np.array_equal(c.vl_k[0, i], K[0, 0, p].view(np.uint16))
