"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the C oracle (a text substitution),
builds the copy with the oracle's own flags, and runs the pins expected to
notice it in a child process pointed at the mutant library (HYQ_ORACLE_LIB).
The pins must fail.  The unmodified source built the same way must pass them,
which also shows that the child really loads the library it is given.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor


import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hyq_oracle.c")
HDR = os.path.join(ROOT, "oracle", "hyq_oracle.h")

# (mistake, text in hyq_oracle.c, replacement, pins that must fail: a -k expression)
MUTANTS = [
    ("softmax scale 1/d instead of 1/sqrt(d)",
     "double scale = 1.0 / sqrt((double)HYQO_D);", "double scale = 1.0 / (double)HYQO_D;",
     "decode_matches_torch"),
    ("codes rounded half away from zero",
     "float ri = rintf(r);", "float ri = roundf(r);", "quantizer_hand_vectors"),
    ("scale = range / 16",
     "float s32 = diff / 15.0f;", "float s32 = diff / 16.0f;", "quantizer_hand_vectors"),
    ("zero point dropped in the dequantization",
     "out[c] = z + (double)code[c] * s;", "out[c] = (double)code[c] * s;", "dequant_error"),
    ("query head reads the wrong KV head",
     "(int64_t)u.kvh * G + hg;", "(int64_t)hg * c->n_kv_heads + u.kvh;", "gqa_groups"),
    ("window boundary off by one",
     "if (p >= u->T - W) {", "if (p > u->T - W) {", "decode_matches_torch"),
    ("selection without the causal mask",
     "int32_t last = T - n_q + i; /* causal: keys 0..last */", "int32_t last = T - 1;",
     "select_matches_bruteforce"),
    ("ties go to the higher position",
     "return (x->p < y->p) ? -1 : (x->p > y->p);", "return (x->p > y->p) ? -1 : (x->p < y->p);",
     "ties_go_to_the_lower"),
    ("vertical-only variant keeps the quantized positions",
     "return p >= u->T - u->c->window || u->slot_of[p] >= 0;", "return 1;", "vl_only"),
    ("a -0 minimum stored as -0",
     "if (zh == 0x8000u) zh = 0;", "/* no canonical zero */", "quantizer"),
    ("codes clamped at 16",
     "if (ri > 15.0f) ri = 15.0f;", "if (ri > 16.0f) ri = 16.0f;", "quantizer"),
    ("scale and zero swapped in the dequantization",
     "double s = hyqo_half_to_double(sz[2 * g]);", "double s = hyqo_half_to_double(sz[2 * g + 1]);",
     "dequant_error"),
    ("selection candidates include the window",
     "int32_t n_cand = T - c->window;", "int32_t n_cand = T;", "select_matches_bruteforce"),
    ("low and high nibbles swapped in the packed layout",
     "*high_nibble = w % 2;", "*high_nibble = 1 - w % 2;", "packed_layout"),
    ("decode log-sum-exp in base 2",
     "*lse = (n > 0) ? m + log(l) : -INFINITY;", "*lse = (n > 0) ? m + log2(l) : -INFINITY;",
     "decode_matches_torch"),
    ("selection sums logits instead of probabilities",
     "cs[p] += exp(s[p] - m) / l;", "cs[p] += s[p];", "select_matches_bruteforce"),
    ("codes decided with the unrounded fp32 scale",
     "float sf = half_to_float(sh);", "float sf = s32;", "quantizer"),
    ("codes by reciprocal multiply instead of division",
     "float r = num / sf;", "float r = num * (1.0f / sf);", "quantizer"),
    ("vertical-line rows read from the next slot",
     "u->slot_of[pos[i]] = i;", "u->slot_of[pos[i]] = (i + 1) % cnt;", "select_cache_mode"),
    ("FP16 comparator reads the wrong KV head",
     "int64_t h = (int64_t)b * Hq + (int64_t)kvh * G + hg;", "int64_t h = (int64_t)b * Hq + (int64_t)hg * Hkv + kvh;",
     "decode_all_fp16"),
    ("selection query i sees one key too few",
     "int32_t last = T - n_q + i; /* causal: keys 0..last */", "int32_t last = T - n_q + i - 1;",
     "select_matches_bruteforce"),
    ("selection margin relative to the k+1-th sum",
     "margin[unit] = (cand[k - 1].cs - cand[k].cs) / cand[k - 1].cs;",
     "margin[unit] = (cand[k - 1].cs - cand[k].cs) / cand[k].cs;", "margin"),
    ("prefill high-precision pairs use the quantized value",
     "acc[d] += e * (high ? hyqo_half_to_double(vu[(int64_t)j * HYQO_D + d]) : vq[(int64_t)j * HYQO_D + d]);",
     "acc[d] += e * vq[(int64_t)j * HYQO_D + d];", "prefill_rows_inside_the_window"),
    ("vertical-only window one position short",
     "return p >= u->T - u->c->window || u->slot_of[p] >= 0;", "return p > u->T - u->c->window || u->slot_of[p] >= 0;",
     "vl_only"),
    ("prefill sliding window one key too wide",
     "int high = is_vl[j] || j > i - W;", "int high = is_vl[j] || j >= i - W;", "prefill_row_with_grid"),
    ("prefill high-precision pairs use the quantized query",
     "sdot += high ? qf[d] * hyqo_half_to_double(", "sdot += high ? qq[d] * hyqo_half_to_double(",
     "prefill_rows_inside_the_window"),
]


def _run_pins(workdir, source, pins):
    d = workdir / "src"
    d.mkdir(parents=True)
    (d / "hyq_oracle.c").write_text(source)
    shutil.copy(HDR, d / "hyq_oracle.h")
    lib = oracle.compile_to(str(d / "hyq_oracle.c"), str(workdir / "liboracle_variant.so"))
    env = dict(os.environ, HYQ_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-k", pins],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-1500:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    """The unmodified source passes the union of the pins; every mutant makes
    its pins fail.  The cases run in parallel child processes."""
    src = open(SRC).read()
    jobs = [("unmodified source", src, " or ".join(sorted({m[3] for m in MUTANTS})), 0)]
    for what, old, new, pins in MUTANTS:
        assert old in src, f"mutation site not found: {old}"
        jobs.append((what, src.replace(old, new), pins, 1))

    def run(job):
        n, (what, source, pins, want) = job
        rc, out = _run_pins(tmp_path / f"case{n}", source, pins)
        return what, want, rc, out

    with ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
        results = list(ex.map(run, enumerate(jobs)))
    bad = [f"{what}: pytest exit {rc}, expected {want}\n{out}" for what, want, rc, out in results if rc != want]
    assert not bad, "\n\n".join(bad)


# (mistake, text in oracle/cache.py, replacement, pins that must fail)
BOOKKEEPING_MUTANTS = [
    ("the new row packed instead of the row leaving the window",
     "c, s, bad = pack(self.win_k[u, slot])", "c, s, bad = pack(k_new[b, h][None])", "append_equals"),
    ("the leaving position off by one",
     "p_out = T - self.W\n", "p_out = T - self.W + 1\n", "append_equals"),
    ("K and V swapped when vertical lines are gathered",
     "rows_k = [K_full[b, h, p] for p in new]", "rows_k = [V_full[b, h, p] for p in new]",
     "decode_matches_torch"),
    ("the window filled from one row late",
     "for p in range(n_old, T):", "for p in range(n_old + 1, T):", "decode_matches_torch"),
    ("staged positions promoted without the order rule",
     "elif self.staged(b, p) and p > last_kept:", "elif self.staged(b, p):", "promotes_staged"),
    ("the staging ring filled one row short",
     "for p in range(max(0, n_old - self.stage), n_old):", "for p in range(max(0, n_old - self.stage + 1), n_old):",
     "staging_ring"),
    ("re-selection keeps no earlier rows",
     "                        if p in old:\n", "                        if False:\n", "reselection"),
]


def _run_pins_with_package(workdir, cache_source, pins):
    """Copies of tests/, synth/ and oracle/ (cache.py replaced) under a
    scratch root; the copied conftest puts that root first on sys.path."""
    for name in ("tests", "synth", "oracle"):
        shutil.copytree(os.path.join(ROOT, name), workdir / name,
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (workdir / "oracle" / "cache.py").write_text(cache_source)
    shutil.copy(os.path.join(ROOT, "pytest.ini"), workdir / "pytest.ini")
    env = dict(os.environ, OMP_NUM_THREADS="2")
    env.pop("HYQ_ORACLE_LIB", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        str(workdir / "tests" / "test_oracle_pins.py"), "-k", pins],
                       cwd=str(workdir), env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, r.stdout[-1500:]


def test_every_planted_bookkeeping_mistake_fails_a_pin(tmp_path):
    """The same check for the host-side bookkeeping of the oracle cache."""
    src = open(os.path.join(ROOT, "oracle", "cache.py")).read()
    jobs = [("unmodified cache.py", src, " or ".join(sorted({m[3] for m in BOOKKEEPING_MUTANTS})), 0)]
    for what, old, new, pins in BOOKKEEPING_MUTANTS:
        assert src.count(old) == 1, f"mutation site not found once: {old!r}"
        jobs.append((what, src.replace(old, new), pins, 1))

    def run(job):
        n, (what, source, pins, want) = job
        d = tmp_path / f"pkg{n}"
        d.mkdir()
        rc, out = _run_pins_with_package(d, source, pins)
        return what, want, rc, out

    with ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
        results = list(ex.map(run, enumerate(jobs)))
    bad = [f"{what}: pytest exit {rc}, expected {want}\n{out}" for what, want, rc, out in results if rc != want]
    assert not bad, "\n\n".join(bad)
