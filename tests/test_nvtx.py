"""Tracing: every compute entry point of the C ABI opens one host-side NVTX
range named after itself, closed when the call returns.  A small NVTX tool
(tests/nvtx_capture.c, injected through NVTX_INJECTION64_PATH) records the
pushes and pops while a child process calls each entry point with arguments
the library rejects on the host, so no GPU is needed."""
import os
import shutil
import subprocess
import sys
import textwrap

import pytest

from fp16_kv_cache_b200 import build as hbuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

RANGED = ["hyq_pack", "hyq_prefill", "hyq_append", "hyq_select_vl", "hyq_vl_apply", "hyq_decode",
          "hyq_decode_vl_only", "hyq_decode_step", "hyq_decode_fp16", "hyq_decode_noalloc",
          "hyq_prefill_attention", "hyq_copy"]

CHILD = textwrap.dedent("""
    import ctypes, sys
    sys.path.insert(0, sys.argv[2])
    from fp16_kv_cache_b200.hyq import EXPORTS
    L = ctypes.CDLL(sys.argv[1])
    sig = {n: (r, a) for n, r, a in EXPORTS}
    for name in sys.argv[3:]:
        res, args = sig[name]
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
        # null pointers and zero sizes: rejected by the host-side checks
        rc = f(*[None if a in (ctypes.c_void_p,) or hasattr(a, "contents") else 0 for a in args])
        print(name, rc)
""")


def _tool(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    out = str(tmp_path / "libnvtx_capture.so")
    subprocess.run([cc, "-shared", "-fPIC", "-O1", "-I", "/usr/local/cuda/include",
                    os.path.join(HERE, "nvtx_capture.c"), "-o", out], check=True)
    return out


def test_each_compute_entry_point_opens_a_named_range(tmp_path):
    lib = hbuild.build()
    tool = _tool(tmp_path)
    log = tmp_path / "nvtx.log"
    env = dict(os.environ, NVTX_INJECTION64_PATH=tool, HYQ_NVTX_LOG=str(log), CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", CHILD, lib, ROOT] + RANGED, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    rcs = dict(line.split() for line in r.stdout.split("\n") if line.strip())
    assert all(int(rcs[n]) != 0 for n in RANGED), rcs  # every call was rejected
    events = log.read_text().split("\n")[:-1]
    # one push per call in call order, each closed before the next opens
    assert events == [e for n in RANGED for e in (f"push {n}", "pop")], events


def test_no_tool_attached_records_nothing(tmp_path):
    lib = hbuild.build()
    log = tmp_path / "nvtx.log"
    env = {k: v for k, v in os.environ.items() if k != "NVTX_INJECTION64_PATH"}
    env.update(HYQ_NVTX_LOG=str(log), CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", CHILD, lib, ROOT, "hyq_decode"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert not log.exists()
