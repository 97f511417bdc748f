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


def _header():
    return open(os.path.join(ROOT, "include", "fdllm.h")).read()


def _typedef_body(src, kind, name):
    end = re.search(r"\}\s*" + name + r"\s*;", src).start()
    start = src.rindex("typedef " + kind + " {", 0, end)
    return re.sub(r"/\*.*?\*/", "", src[start:end].split("{", 1)[1], flags=re.S)


def _struct_fields(src, name):
    body = _typedef_body(src, "struct", name)
    return re.findall(r"([\w\s\*]+?)\s*\b(\w+);", body)


def _enum(src, name):
    body = _typedef_body(src, "enum", name)
    return {k: int(v) for k, v in re.findall(r"(\w+)\s*=\s*(\d+)", body)}


def test_binding_structs_match_the_header():
    """The ctypes mirrors of the descriptor structs have the header's fields in
    the header's order, with C types of the same size."""
    src = _header()
    sizes = {"int": 4, "float": 4, "int32_t": 4, "uint64_t": 8, "size_t": 8}
    for cname, py in (("fdl_generate_opts", fdllm.GenerateOpts),
                      ("fdl_attn_desc", fdllm.AttnDesc),
                      ("fdl_lmhead_desc", fdllm.LMHeadDesc),
                      ("fdl_unmask_desc", fdllm.UnmaskDesc),
                      ("fdl_qkv_desc", fdllm.QKVDesc),
                      ("fdl_model_desc", fdllm.ModelDesc),
                      ("fdl_layer_weights", fdllm.LayerWeights),
                      ("fdl_model_weights", fdllm.ModelWeights)):
        fields = _struct_fields(src, cname)
        assert [f for _, f in fields] == [f for f, _ in py._fields_], cname
        for (ctype, fname), (_, pytype) in zip(fields, py._fields_):
            ctype = ctype.replace("const", "").strip()
            want = 8 if "*" in ctype else sizes[ctype]
            assert ctypes.sizeof(pytype) == want, (cname, fname)


def test_binding_enums_match_the_header():
    src = _header()
    batching = _enum(src, "fdl_batching")
    assert batching == {"FDL_BATCH_LOCKSTEP": fdllm.BATCHING["lockstep"],
                        "FDL_BATCH_COMPACT": fdllm.BATCHING["compact"],
                        "FDL_BATCH_PER_SEQUENCE": fdllm.BATCHING["per_sequence"]}
    cache = _enum(src, "fdl_cache_mode")
    assert cache == {"FDL_CACHE_DUAL": fdllm.CACHE_MODES["dual"],
                     "FDL_CACHE_PREFIX": fdllm.CACHE_MODES["prefix"],
                     "FDL_CACHE_NONE": fdllm.CACHE_MODES["none"]}
