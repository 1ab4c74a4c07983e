"""HyQuant hybrid INT4/FP16 KV-cache decode attention for NVIDIA B200.

The compute lives in ``libhyq.so`` (CUDA, sm_100a; C ABI in ``include/hyq.h``);
:mod:`fp16_kv_cache_b200.hyq` is its thin ctypes binding.  Importing this
package loads nothing; the library is opened on first use.
"""
__all__ = ["hyq", "build"]
