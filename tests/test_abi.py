"""Host-side checks of the C-ABI library: it loads without a GPU, exports
every function include/fdllm.h declares, and fails cleanly (status code plus
message, no crash) when called without a device or with bad arguments that
are rejected before any device work."""
import ctypes
import os
import re

import pytest

from block_kv_cache_b200 import fdllm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"FDL_API\s+[\w\s\*]+?\b(fdl_\w+)\s*\(", src)
    return names


def test_library_loads_and_exports_every_declared_symbol():
    L = fdllm.load()
    declared = _declared()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(L, name), name
    assert set(fdllm.EXPORTS) <= set(declared)
    assert L.fdl_abi_version() == fdllm.ABI_VERSION


def test_null_arguments_rejected_without_device():
    L = fdllm.load()
    assert L.fdl_create(None, 0) == fdllm.FDL_EINVAL
    assert b"NULL" in L.fdl_last_error()
    d = fdllm.AttnDesc(1, 4, 4, 64, 128, 64, 32, fdllm.FDL_F32, 0.0)
    assert L.fdl_dualcache_attention(None, ctypes.byref(d), None, None, None, None, None,
                                     None, 0, None) == fdllm.FDL_EINVAL
    assert L.fdl_attention_workspace_bytes(None, ctypes.byref(d)) == 0
    lm = fdllm.LMHeadDesc(32, 256, 1024, fdllm.FDL_F32)
    assert L.fdl_lmhead_workspace_bytes(None, ctypes.byref(lm)) == 0
    u = fdllm.UnmaskDesc(1, 128, 64, 32, 0.9)
    assert L.fdl_threshold_unmask(None, ctypes.byref(u), None, None, None, None, None, None,
                                  None) == fdllm.FDL_EINVAL
    assert L.fdl_model_create(None, None, None) == fdllm.FDL_EINVAL
    assert L.fdl_generate(None, None, None, 1, 32, 32, 32, 0.9, None, None, None, None, 0,
                          None) == fdllm.FDL_EINVAL
    assert L.fdl_generate_workspace_bytes(None, None, 1, 64, 32) == 0
    assert L.fdl_set_wait_timeout(None, 1000) == fdllm.FDL_EINVAL
    assert L.fdl_model_destroy(None) == fdllm.FDL_OK
    assert L.fdl_destroy(None) == fdllm.FDL_OK


def test_create_without_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = fdllm.load()
    h = ctypes.c_void_p()
    rc = L.fdl_create(ctypes.byref(h), 0)
    assert rc in (fdllm.FDL_ECUDA, fdllm.FDL_EINVAL)
    assert h.value is None
    assert len(L.fdl_last_error()) > 0


def test_binding_raises_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(fdllm, "_lib", None)
    monkeypatch.setattr(fdllm, "LIB_PATH", str(tmp_path / "libfdllm.so"))
    with pytest.raises(RuntimeError, match="not built"):
        fdllm.load()
