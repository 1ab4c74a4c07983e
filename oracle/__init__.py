"""CPU oracle for the HyQuant hybrid-precision KV-cache decode path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.  The CUDA library and its
Python binding never import it, and it imports nothing from them.

The arithmetic lives in ``hyq_oracle.c`` (plain C, fp64, built by
:func:`build`); this module only marshals numpy arrays through ctypes, and
``cache.py`` holds the host-side bookkeeping of the hybrid cache (which
position lives in which segment) in plain numpy.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# A library built elsewhere from a modified copy of the source: the pin tests
# run against it to show that a planted mistake makes a pin fail.
_LIB_OVERRIDE = os.environ.get("HYQ_ORACLE_LIB")
_lib = None

D = 128
GROUP = 32
NG = 4
ROW_BYTES = 64


def compile_to(src: str, out: str) -> str:
    """Compile an oracle source file (its header beside it) with IEEE
    fp32/fp64 semantics: no FMA contraction, no fast-math."""
    cmd = [
        "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
        "-ffp-contract=off", "-fno-fast-math", "-frounding-math",
        "-o", out, src, "-lm",
    ]
    subprocess.check_call(cmd, cwd=os.path.dirname(os.path.abspath(src)))
    return out


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (or return the
    library named by HYQ_ORACLE_LIB, built by its maker)."""
    if _LIB_OVERRIDE:
        return _LIB_OVERRIDE
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "hyq_oracle.h"))
    ):
        compile_to(_SRC, _LIB)
    return _LIB


class _Cache(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("window", ctypes.c_int32),
        ("capacity", ctypes.c_int32), ("vl_capacity", ctypes.c_int32),
        ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
        ("k_sz", ctypes.c_void_p), ("v_sz", ctypes.c_void_p),
        ("win_k", ctypes.c_void_p), ("win_v", ctypes.c_void_p),
        ("vl_k", ctypes.c_void_p), ("vl_v", ctypes.c_void_p),
        ("vl_pos", ctypes.c_void_p), ("vl_count", ctypes.c_void_p),
        ("seq_len", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L.hyqo_half_to_double.restype = ctypes.c_double
        L.hyqo_half_to_double.argtypes = [ctypes.c_uint16]
        L.hyqo_float_to_half.restype = ctypes.c_uint16
        L.hyqo_float_to_half.argtypes = [ctypes.c_float]
        L.hyqo_quantize_row.restype = ctypes.c_int
        L.hyqo_quantize_row.argtypes = [P, P, P, P]
        L.hyqo_code_slot.restype = None
        L.hyqo_code_slot.argtypes = [ctypes.c_int, P, P]
        L.hyqo_pack.restype = ctypes.c_int64
        L.hyqo_pack.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, P]
        L.hyqo_unpack_codes.restype = None
        L.hyqo_unpack_codes.argtypes = [P, P]
        L.hyqo_dequant_row.restype = None
        L.hyqo_dequant_row.argtypes = [P, P, P]
        L.hyqo_decode.restype = ctypes.c_int
        L.hyqo_decode.argtypes = [ctypes.POINTER(_Cache), P, P, ctypes.c_int32, P, P]
        L.hyqo_decode_vl_only.restype = ctypes.c_int
        L.hyqo_decode_vl_only.argtypes = [ctypes.POINTER(_Cache), P, P, ctypes.c_int32, P, P]
        L.hyqo_decode_fp16.restype = ctypes.c_int
        L.hyqo_decode_fp16.argtypes = [P, P, P, P, ctypes.c_int32, ctypes.c_int32,
                                       ctypes.c_int32, ctypes.c_int32, P,
                                       ctypes.c_int32, P, P]
        L.hyqo_prefill_attention.restype = ctypes.c_int
        L.hyqo_prefill_attention.argtypes = [P, P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_int32, P, P, ctypes.c_int32, P, P]
        L.hyqo_select_vl.restype = ctypes.c_int
        L.hyqo_select_vl.argtypes = [ctypes.POINTER(_Cache), P, ctypes.c_int32, P,
                                     ctypes.c_int32, P, ctypes.c_int32, P, P, P]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c16(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


# ---------------------------------------------------------------- scalars
def half_to_double(bits: int) -> float:
    return lib().hyqo_half_to_double(int(bits) & 0xFFFF)


def float_to_half(x: float) -> int:
    return int(lib().hyqo_float_to_half(float(np.float32(x))))


# ---------------------------------------------------------------- quantizer
def quantize_row(x):
    """One fp16 row of 128 -> (codes[128] u8, scale bits[4], zero bits[4], rc)."""
    x = _c16(np.asarray(x).reshape(D))
    code = np.zeros(D, np.uint8)
    s = np.zeros(NG, np.uint16)
    z = np.zeros(NG, np.uint16)
    rc = lib().hyqo_quantize_row(_ptr(x), _ptr(code), _ptr(s), _ptr(z))
    return code, s, z, rc


def code_slot(c: int):
    b = ctypes.c_int()
    hi = ctypes.c_int()
    lib().hyqo_code_slot(int(c), ctypes.byref(b), ctypes.byref(hi))
    return b.value, hi.value


def pack(x):
    """Rows [n][128] fp16 -> (codes [n][64] u8, sz [n][8] u16, n_bad)."""
    x = _c16(np.asarray(x).reshape(-1, D))
    n = x.shape[0]
    codes = np.zeros((n, ROW_BYTES), np.uint8)
    sz = np.zeros((n, 8), np.uint16)
    bad = lib().hyqo_pack(_ptr(x), n, D, _ptr(codes), _ptr(sz)) if n else 0
    return codes, sz, int(bad)


def unpack_codes(packed):
    packed = np.ascontiguousarray(packed, np.uint8).reshape(-1, ROW_BYTES)
    out = np.zeros((packed.shape[0], D), np.uint8)
    for i in range(packed.shape[0]):
        lib().hyqo_unpack_codes(_ptr(packed[i]), _ptr(out[i]))
    return out


def dequant(packed, sz):
    packed = np.ascontiguousarray(packed, np.uint8).reshape(-1, ROW_BYTES)
    sz = np.ascontiguousarray(sz, np.uint16).reshape(-1, 8)
    out = np.zeros((packed.shape[0], D), np.float64)
    for i in range(packed.shape[0]):
        lib().hyqo_dequant_row(_ptr(packed[i]), _ptr(sz[i]), _ptr(out[i]))
    return out


# ---------------------------------------------------------------- cache ops
def _cache_struct(c):
    s = _Cache()
    s.batch, s.n_q_heads, s.n_kv_heads = c.B, c.Hq, c.Hkv
    s.window, s.capacity, s.vl_capacity = c.W, c.cap, c.vl_cap
    s.k_codes, s.v_codes = _ptr(c.k_codes), _ptr(c.v_codes)
    s.k_sz, s.v_sz = _ptr(c.k_sz), _ptr(c.v_sz)
    s.win_k, s.win_v = _ptr(c.win_k), _ptr(c.win_v)
    s.vl_k, s.vl_v = _ptr(c.vl_k), _ptr(c.vl_v)
    s.vl_pos, s.vl_count = _ptr(c.vl_pos), _ptr(c.vl_count)
    s.seq_len = _ptr(c.seq_len)
    return s


def _decode(fn, what, cache, q, units):
    q = _c16(q)
    o = np.full((cache.B, cache.Hq, D), np.nan)
    lse = np.full((cache.B, cache.Hq), np.nan)
    u = None if units is None else np.ascontiguousarray(units, np.int32)
    s = _cache_struct(cache)
    rc = fn(ctypes.byref(s), _ptr(q), _ptr(u), 0 if u is None else len(u), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle {what}: inconsistent cache (code {rc})")
    return o, lse


def decode(cache, q, units=None):
    """fp64 decode over the oracle's hybrid cache.  q: [B][Hq][128] fp16.
    Returns (o [B][Hq][128] f64, lse [B][Hq] f64); rows of units not listed
    are NaN."""
    return _decode(lib().hyqo_decode, "decode", cache, q, units)


def decode_vl_only(cache, q, units=None):
    """The vertical-only ablation (AI Radio episode "HyQuant: Hybrid-Precision
    Quantization for LLM Attention", "Improvements and Ablation Studies",
    Table twelve): attention over the cache's vertical-line rows and window
    alone, the quantized majority left out.  Same arguments and results as
    decode."""
    return _decode(lib().hyqo_decode_vl_only, "decode_vl_only", cache, q, units)


def prefill_attention(q, k, v, seq_len, vl=None, W=128):
    """Prefill hybrid-precision attention (explainer "Two Operational Modes /
    Prefill Stage"): causal attention in which a (query row i, key j) pair is
    computed from FP16 q, k, v when j is a vertical line or j > i - W, and
    from the INT4-dequantized q, k, v otherwise.  q [B][Hq][cap][128], k/v
    [B][Hkv][cap][128] fp16, vl [B][Hkv][n] ascending positions (or None).
    Returns (o [B][Hq][cap][128] f64, lse [B][Hq][cap] f64); rows >= T are
    NaN."""
    q, k, v = _c16(q), _c16(k), _c16(v)
    B, Hq, cap, _ = q.shape
    Hkv = k.shape[1]
    seq_len = np.ascontiguousarray(seq_len, np.int32)
    o = np.full((B, Hq, cap, D), np.nan)
    lse = np.full((B, Hq, cap), np.nan)
    pos = cnt = None
    stride = 0
    if vl is not None:
        pos = np.ascontiguousarray(vl, np.int32).reshape(B * Hkv, -1)
        stride = pos.shape[1]
        cnt = np.full(B * Hkv, stride, np.int32)
    rc = lib().hyqo_prefill_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_len), B, Hq, Hkv, cap, W,
                                      _ptr(pos), _ptr(cnt), stride, _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle prefill_attention: bad arguments (code {rc})")
    return o, lse


def decode_fp16(q, k, v, seq_len, Hq, units=None):
    """fp64 attention over an all-FP16 cache k, v [B][Hkv][cap][128]."""
    q, k, v = _c16(q), _c16(k), _c16(v)
    B, Hkv, cap, _ = k.shape
    seq_len = np.ascontiguousarray(seq_len, np.int32)
    o = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    u = None if units is None else np.ascontiguousarray(units, np.int32)
    rc = lib().hyqo_decode_fp16(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_len), B, Hq, Hkv,
                                cap, _ptr(u), 0 if u is None else len(u), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle decode_fp16: bad arguments (code {rc})")
    return o, lse


def select_vl(cache, q_sel, k, k_full=None, units=None):
    """Top-k vertical-line positions.  q_sel: [B][Hq][n_q][128] fp16;
    k_full: optional [B][Hkv][cap][128] fp16 (prefill mode).
    Returns (pos [B][Hkv][k] i32, colsum [B][Hkv][cap] f64, margin [B][Hkv])."""
    q_sel = _c16(q_sel)
    n_q = q_sel.shape[2]
    kf = None if k_full is None else _c16(k_full)
    pos = np.full((cache.B, cache.Hkv, k), -1, np.int32)
    cs = np.zeros((cache.B, cache.Hkv, cache.cap), np.float64)
    margin = np.full((cache.B, cache.Hkv), np.nan)
    u = None if units is None else np.ascontiguousarray(units, np.int32)
    s = _cache_struct(cache)
    rc = lib().hyqo_select_vl(ctypes.byref(s), _ptr(q_sel), n_q, _ptr(kf), k, _ptr(u),
                              0 if u is None else len(u), _ptr(pos), _ptr(cs), _ptr(margin))
    if rc != 0:
        raise ValueError(f"oracle select_vl: bad arguments (code {rc})")
    return pos, cs, margin


from .cache import OracleCache  # noqa: E402  (host bookkeeping, numpy only)
