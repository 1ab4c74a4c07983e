"""Thin Python binding of libhyq.so (the C ABI in include/hyq.h).

Argument marshalling only: torch tensors supply device memory and streams,
every computation runs in the library's CUDA kernels.  There is no CPU or
PyTorch fallback: if the shared library is missing or no CUDA device is
present, the calls raise.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import numpy as np

import torch

from . import build as _build

HEAD_DIM = 128
GROUP = 32
WINDOW = 128
ROW_BYTES = 64
BLOCK_TOKENS = 32
BLOCK_BYTES = 5136
BLK_KCODES, BLK_KSZ, BLK_VCODES, BLK_VSZ, BLK_MASK = 0, 2048, 2560, 4608, 5120

DEV_NONFINITE = 0x1
DEV_OOB = 0x2  # raised by the index checks of the debug build only
DEV_TIMEOUT = 0x4
DEV_BADLEN = 0x8

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "pointer not 16-byte aligned",
          4: "workspace missing or too small", 5: "CUDA launch error"}

_lib = None
_debug_lib = None
_active = None  # the library the wrappers below call (None: libhyq.so)


class HyqError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)} (hyq status {code})")
        self.code = code


class hyq_cache(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("group", ctypes.c_int32), ("window", ctypes.c_int32),
        ("capacity", ctypes.c_int32), ("vl_capacity", ctypes.c_int32),
        ("blocks", ctypes.c_void_p),
        ("win_k", ctypes.c_void_p), ("win_v", ctypes.c_void_p),
        ("vl_k", ctypes.c_void_p), ("vl_v", ctypes.c_void_p),
        ("vl_pos", ctypes.c_void_p), ("vl_count", ctypes.c_void_p),
        ("seq_len", ctypes.c_void_p),
        ("dev_status", ctypes.c_void_p),
        ("stage_k", ctypes.c_void_p), ("stage_v", ctypes.c_void_p),
        ("stage_rows", ctypes.c_int32),
        ("block_table", ctypes.c_void_p), ("n_pages", ctypes.c_int32),
    ]


# (name, restype, argtypes) of every exported entry point
_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_CP = ctypes.POINTER(hyq_cache)
EXPORTS = [
    ("hyq_pack", ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    ("hyq_prefill", ctypes.c_int, [_CP, _P, _P, _P]),
    ("hyq_append", ctypes.c_int, [_CP, _P, _P, _P, _P, _I32, _P]),
    ("hyq_select_vl_workspace", _SZ, [_CP, _I32]),
    ("hyq_select_vl", ctypes.c_int, [_CP, _P, _I32, _I32, _P, _I32, _P, _P, _P, _SZ, _P]),
    ("hyq_vl_apply", ctypes.c_int, [_CP, _P, _I32, _P, _P, _P, _P]),
    ("hyq_decode_workspace", _SZ, [_CP, _I32]),
    ("hyq_decode", ctypes.c_int, [_CP, _P, _P, _P, _I32, _P, _SZ, _P]),
    ("hyq_decode_vl_only", ctypes.c_int, [_CP, _P, _P, _P, _I32, _P, _SZ, _P]),
    ("hyq_decode_step_workspace", _SZ, [_CP, _I32]),
    ("hyq_decode_step", ctypes.c_int, [_CP, _P, _P, _P, _P, _I32, _P, _P, _I32, _P, _SZ, _P]),
    ("hyq_decode_noalloc", ctypes.c_int, [_CP, _P, _P, _P, _P]),
    ("hyq_decode_fp16_workspace", _SZ, [_I32, _I32, _I32, _I32]),
    ("hyq_decode_fp16", ctypes.c_int, [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _I32, _P, _SZ, _P, _P]),
    ("hyq_prefill_attention_workspace", _SZ, [_CP]),
    ("hyq_prefill_attention", ctypes.c_int, [_CP, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    ("hyq_copy", ctypes.c_int, [_P, _P, _SZ, _P]),
    ("hyq_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("hyq_decode_default_ctas", _I32, []),
    ("hyq_version", _I32, []),
]


def lib_path() -> str:
    return _build.LIB


def lib():
    """Load libhyq.so (built in-tree by ``python -m fp16_kv_cache_b200.build``)."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is not built: run `python -m fp16_kv_cache_b200.build`")
        L = ctypes.CDLL(path)
        for name, res, args in EXPORTS:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


# extra entry point of the debug build (include/hyq_debug.h)
DEBUG_EXPORTS = [("hyq_debug_set_wait", ctypes.c_int, [ctypes.c_uint64, ctypes.c_int32])]


def debug_lib():
    """Load libhyq_debug.so: the same entry points built with device-side
    index checks (HYQ_DEV_OOB) and a settable decode wait limit."""
    global _debug_lib
    if _debug_lib is None:
        path = _build.DEBUG_LIB
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is not built: run `python -m fp16_kv_cache_b200.build`")
        L = ctypes.CDLL(path)
        for name, res, args in EXPORTS + DEBUG_EXPORTS:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _debug_lib = L
    return _debug_lib


@contextlib.contextmanager
def using_debug_library():
    """Route the wrappers below to libhyq_debug.so inside the block."""
    global _active
    prev, _active = _active, debug_lib()
    try:
        yield _active
    finally:
        _active = prev


def _L():
    return _active if _active is not None else lib()


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhyq takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libhyq takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc, what):
    if rc != 0:
        raise HyqError(int(rc), what)


# ------------------------------------------------------------------ cache
class HybridCache:
    """Device buffers of one layer's hybrid cache plus its C descriptor."""

    def __init__(self, batch, n_q_heads, n_kv_heads, capacity, vl_capacity, device="cuda", stage_rows=0,
                 block_table=None, n_pages=0):
        """block_table (int32 [B][capacity/32]) and n_pages: the quantized
        majority lives in a pool of n_pages pages of n_kv_heads records, and
        sequence b's 32-position block j in page block_table[b][j]."""
        if capacity % 128:
            raise ValueError("capacity must be a multiple of 128")
        B, Hkv = batch, n_kv_heads
        dev = torch.device(device)
        z = lambda *s, dt: torch.zeros(*s, dtype=dt, device=dev)  # noqa: E731
        self.B, self.Hq, self.Hkv, self.cap, self.vl_cap = B, n_q_heads, Hkv, capacity, vl_capacity
        self.block_table = None
        if block_table is not None:
            self.block_table = torch.as_tensor(block_table, dtype=torch.int32).reshape(B, capacity // BLOCK_TOKENS)
            self.block_table = self.block_table.to(dev).contiguous()
            self.n_pages = int(n_pages)
            self.blocks = z(self.n_pages, Hkv, BLOCK_BYTES, dt=torch.uint8)
        else:
            self.n_pages = 0
            self.blocks = z(B, Hkv, capacity // BLOCK_TOKENS, BLOCK_BYTES, dt=torch.uint8)
        self.win_k = z(B, Hkv, WINDOW, HEAD_DIM, dt=torch.float16)
        self.win_v = z(B, Hkv, WINDOW, HEAD_DIM, dt=torch.float16)
        self.vl_k = z(B, Hkv, vl_capacity, HEAD_DIM, dt=torch.float16)
        self.vl_v = z(B, Hkv, vl_capacity, HEAD_DIM, dt=torch.float16)
        self.vl_pos = z(B, Hkv, vl_capacity, dt=torch.int32)
        self.vl_count = z(B, Hkv, dt=torch.int32)
        self.seq_len = z(B, dt=torch.int32)
        self.dev_status = z(4, dt=torch.int32)
        self.stage_rows = int(stage_rows)
        self.stage_k = z(B, Hkv, max(self.stage_rows, 1), HEAD_DIM, dt=torch.float16)
        self.stage_v = z(B, Hkv, max(self.stage_rows, 1), HEAD_DIM, dt=torch.float16)
        c = hyq_cache()
        c.batch, c.n_q_heads, c.n_kv_heads = B, n_q_heads, Hkv
        c.head_dim, c.group, c.window = HEAD_DIM, GROUP, WINDOW
        c.capacity, c.vl_capacity = capacity, vl_capacity
        for name in ("blocks", "win_k", "win_v", "vl_k", "vl_v", "vl_pos", "vl_count", "seq_len",
                     "dev_status"):
            setattr(c, name, getattr(self, name).data_ptr())
        if self.stage_rows:
            c.stage_k, c.stage_v, c.stage_rows = self.stage_k.data_ptr(), self.stage_v.data_ptr(), self.stage_rows
        if self.block_table is not None:
            c.block_table, c.n_pages = self.block_table.data_ptr(), self.n_pages
        self.desc = c

    def ref(self):
        return ctypes.byref(self.desc)

    def status(self) -> int:
        return int(self.dev_status[0].item()) & 0xFFFFFFFF

    def clear_status(self):
        self.dev_status.zero_()

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (
            self.blocks, self.win_k, self.win_v, self.vl_k, self.vl_v, self.vl_pos, self.vl_count,
            self.seq_len))

    def unpack_blocks(self):
        """Host views of the block records as per-position rows: (k_codes
        [B][Hkv][cap][64] u8, k_sz [B][Hkv][cap][8] u16, v_codes, v_sz,
        mask [B][Hkv][cap/32] u32).  A copy; for inspection and tests."""
        b = self.blocks.cpu().numpy()
        if self.block_table is not None:  # gather the sequences' logical blocks from the pool
            tab = self.block_table.cpu().numpy()
            ok = (tab >= 0) & (tab < self.n_pages)
            b = np.where(ok[:, None, :, None], b[np.where(ok, tab, 0)].transpose(0, 2, 1, 3), 0).astype(np.uint8)
        B, H, nb, _ = b.shape
        cap = nb * BLOCK_TOKENS
        def field(off, width):
            return b[..., off:off + BLOCK_TOKENS * width].reshape(B, H, cap, width)
        kc = field(BLK_KCODES, ROW_BYTES)
        ks = field(BLK_KSZ, 16).copy().view("<u2")
        vc = vcode_rows(b[..., BLK_VCODES:BLK_VCODES + BLOCK_TOKENS * ROW_BYTES]).reshape(B, H, cap, ROW_BYTES)
        vs = field(BLK_VSZ, 16).copy().view("<u2")
        mask = b[..., BLK_MASK:BLK_MASK + 4].copy().view("<u4").reshape(B, H, nb)
        return kc, ks, vc, vs, mask


def vcode_rows(area):
    """Packed V code rows [..., 32, 64] (the row format of hyq_pack) from the
    V code areas [..., 2048] of block records, where codes are stored in
    position pairs (include/hyq.h): 16-bit halves indexed [pair][piece][word
    h][low/high][member of the pair], the members of pair i in the order
    (2i, 2i + 1) when i % 4 < 2, else (2i + 1, 2i), and piece p of pair i in
    16-byte unit p xor 2 (i mod 4) of the pair."""
    area = np.ascontiguousarray(area, dtype=np.uint8)
    lead = area.shape[:-1]
    w = area.view("<u2").reshape(lead + (BLOCK_TOKENS // 2, 8, 2, 2, 2))
    pair = np.arange(BLOCK_TOKENS // 2)[:, None]
    w = w[..., pair, np.arange(8)[None, :] ^ ((pair & 3) << 1), :, :, :]
    n = len(lead)
    w = w.transpose(tuple(range(n)) + (n, n + 4, n + 1, n + 2, n + 3)).copy()
    swapped = ((np.arange(BLOCK_TOKENS // 2) >> 1) & 1).astype(bool)
    w[..., swapped, :, :, :, :] = w[..., swapped, ::-1, :, :, :]
    return w.reshape(lead + (BLOCK_TOKENS, ROW_BYTES // 2)).view(np.uint8)


# ------------------------------------------------------------------ entry points
def hyq_pack(x, codes, sz, dst_rows=None, dev_status=None, stream=None):
    """x: fp16 [n][stride] (row-contiguous); codes u8 [*][64]; sz fp16 [*][8]."""
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    n, stride = x.shape[0], x.stride(0)
    if not x.is_cuda:
        raise ValueError("libhyq takes device tensors")
    rc = _L().hyq_pack(ctypes.c_void_p(x.data_ptr()), n, stride, _ptr(dst_rows), _ptr(codes),
                        _ptr(sz), _ptr(dev_status), _stream(stream))
    _check(rc, "hyq_pack")


def hyq_prefill(cache: HybridCache, k_full, v_full, stream=None):
    _check(_L().hyq_prefill(cache.ref(), _ptr(k_full), _ptr(v_full), _stream(stream)), "hyq_prefill")


def hyq_append(cache: HybridCache, k_new, v_new, q_new=None, q_ring=None, stream=None):
    n_q = 0 if q_ring is None else q_ring.shape[2]
    _check(_L().hyq_append(cache.ref(), _ptr(k_new), _ptr(v_new), _ptr(q_new), _ptr(q_ring), n_q,
                            _stream(stream)), "hyq_append")


def hyq_select_vl_workspace(cache: HybridCache, n_q: int) -> int:
    return int(_L().hyq_select_vl_workspace(cache.ref(), n_q))


def hyq_select_vl(cache: HybridCache, q_sel, k, out_pos, ws, out_colsum=None, k_full=None,
                  q_is_ring=False, stream=None):
    n_q = q_sel.shape[2]
    _check(_L().hyq_select_vl(cache.ref(), _ptr(q_sel), n_q, int(bool(q_is_ring)), _ptr(k_full), k,
                               _ptr(out_pos), _ptr(out_colsum), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream(stream)), "hyq_select_vl")


def hyq_vl_apply(cache: HybridCache, pos, k_full=None, v_full=None, n_unpromoted=None, stream=None):
    k = pos.shape[-1]
    _check(_L().hyq_vl_apply(cache.ref(), _ptr(pos), k, _ptr(k_full), _ptr(v_full),
                              _ptr(n_unpromoted), _stream(stream)), "hyq_vl_apply")


def hyq_decode_workspace(cache: HybridCache, n_ctas: int = 0) -> int:
    return int(_L().hyq_decode_workspace(cache.ref(), n_ctas))


def hyq_decode(cache: HybridCache, q, o, ws, lse=None, n_ctas: int = 0, stream=None):
    _check(_L().hyq_decode(cache.ref(), _ptr(q), _ptr(o), _ptr(lse), n_ctas, _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "hyq_decode")


def hyq_decode_vl_only(cache: HybridCache, q, o, ws, lse=None, n_ctas: int = 0, stream=None):
    """The vertical-only ablation: attention over the vertical-line rows and
    the window alone (workspace of hyq_decode_workspace)."""
    _check(_L().hyq_decode_vl_only(cache.ref(), _ptr(q), _ptr(o), _ptr(lse), n_ctas, _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "hyq_decode_vl_only")


def hyq_decode_step_workspace(cache: HybridCache, n_ctas: int = 0) -> int:
    return int(_L().hyq_decode_step_workspace(cache.ref(), n_ctas))


def hyq_decode_step(cache: HybridCache, q, k_new, v_new, o, ws, q_ring=None, lse=None, n_ctas: int = 0,
                    stream=None):
    """hyq_append(cache, k_new, v_new, q, q_ring) and hyq_decode(cache, q) in
    one launch."""
    n_q = int(q_ring.shape[2]) if q_ring is not None else 0
    _check(_L().hyq_decode_step(cache.ref(), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_ring), n_q, _ptr(o),
                                 _ptr(lse), n_ctas, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hyq_decode_step")


class DecodeStepCall:
    """hyq_decode_step with its arguments marshalled once, for a loop that
    calls it again and again on the same buffers: the pointers, sizes and the
    stream are fixed when the object is made, and each call is one foreign
    call.  The cache's descriptor is passed by reference, so the library's
    own updates of the lengths on the device are seen; the buffers are kept
    alive by the object."""

    def __init__(self, cache: HybridCache, q, k_new, v_new, o, ws, q_ring=None, lse=None, n_ctas: int = 0,
                 stream=None):
        n_q = int(q_ring.shape[2]) if q_ring is not None else 0
        self._f = _L().hyq_decode_step
        self._args = (cache.ref(), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_ring), n_q, _ptr(o), _ptr(lse),
                      n_ctas, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
        self._keep = (cache, q, k_new, v_new, q_ring, o, lse, ws)

    def __call__(self):
        rc = self._f(*self._args)
        if rc != 0:
            raise HyqError(int(rc), "hyq_decode_step")


def hyq_decode_noalloc(cache: HybridCache, q, o, lse=None, stream=None):
    """hyq_decode with the library's built-in scratch array instead of a
    caller workspace (for callers that cannot allocate device memory).  Calls
    sharing a device must not overlap on the GPU."""
    _check(_L().hyq_decode_noalloc(cache.ref(), _ptr(q), _ptr(o), _ptr(lse), _stream(stream)),
           "hyq_decode_noalloc")


def hyq_decode_fp16_workspace(batch, n_q_heads, n_kv_heads, n_ctas: int = 0) -> int:
    return int(_L().hyq_decode_fp16_workspace(batch, n_q_heads, n_kv_heads, n_ctas))


def hyq_decode_fp16(q, k, v, seq_len, o, ws, lse=None, n_ctas: int = 0, dev_status=None, stream=None):
    B, Hkv, cap, _ = k.shape
    Hq = q.shape[1]
    _check(_L().hyq_decode_fp16(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_len), B, Hq, Hkv, cap, _ptr(o),
                                 _ptr(lse), n_ctas, _ptr(ws), ws.numel() * ws.element_size(),
                                 _ptr(dev_status), _stream(stream)), "hyq_decode_fp16")


def hyq_prefill_attention_workspace(cache: HybridCache) -> int:
    return int(_L().hyq_prefill_attention_workspace(cache.ref()))


def hyq_prefill_attention(cache: HybridCache, q, k_full, v_full, o, ws, lse=None, stream=None):
    """Prefill hybrid-precision attention of the prompt: q fp16 [B][Hq][cap][128],
    k_full/v_full fp16 [B][Hkv][cap][128], o fp32 [B][Hq][cap][128] (output),
    lse optional fp32 [B][Hq][cap]; the cache gives T and the vertical lines."""
    _check(_L().hyq_prefill_attention(cache.ref(), _ptr(q), _ptr(k_full), _ptr(v_full), _ptr(o), _ptr(lse),
                                      _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hyq_prefill_attention")


def hyq_decode_default_ctas() -> int:
    return int(_L().hyq_decode_default_ctas())


def hyq_version() -> int:
    return int(_L().hyq_version())


def hyq_copy(dst, src, stream=None):
    """Copy src into dst (same number of bytes; device tensors or pinned host
    tensors) with the library's copy kernel, ordered on the stream."""
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() != nbytes:
        raise ValueError("hyq_copy: dst and src differ in size")
    _check(_L().hyq_copy(_ptr_io(dst), _ptr_io(src), nbytes, _stream(stream)), "hyq_copy")


def _ptr_io(t):
    """A device tensor's or a pinned host tensor's address (hyq_copy)."""
    if t.is_cuda:
        return _ptr(t)
    if not t.is_pinned():
        raise ValueError("hyq_copy takes device tensors or pinned host tensors")
    if not t.is_contiguous():
        raise ValueError("libhyq takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def workspace(nbytes: int, device="cuda"):
    """A zero-filled byte workspace (16-byte aligned, as torch allocations are)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)
