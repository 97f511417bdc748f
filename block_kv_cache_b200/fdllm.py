"""Python binding of libfdllm.so, the C-ABI library of the Fast-dLLM step.

Argument marshalling only: every computation runs in the library's CUDA
kernels. torch provides device memory (outputs and scratch are allocated as
torch tensors) and the current CUDA stream. If the shared object is missing,
every call raises: there is no fallback of any kind.

Layouts follow include/fdllm.h:
  q, out   [b, B, Hq, d]     k_cache, v_cache [b, Hkv, L, d]
  h        [M, D]            w [V, D]
  conf/tok [b, B]            x [b, L] int32, masked [b, L] uint8
"""
from __future__ import annotations

import ctypes
import os

import torch

# FDLLM_LIB may name another build of the library (the instrumented
# libfdllm_timeline.so of `python -m block_kv_cache_b200.build --timeline`).
LIB_PATH = os.environ.get("FDLLM_LIB") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                       "libfdllm.so")

FDL_OK, FDL_EINVAL, FDL_EUNSUPPORTED, FDL_ECUDA, FDL_ETIMEOUT, FDL_EWORKSPACE, FDL_EDEVICE = (
    0, -1, -2, -3, -4, -5, -6)
FDL_F32, FDL_BF16 = 0, 1

EXPORTS = ("fdl_abi_version", "fdl_create", "fdl_destroy", "fdl_last_error",
           "fdl_get_device_status", "fdl_set_wait_timeout", "fdl_attention_workspace_bytes",
           "fdl_dualcache_attention", "fdl_kv_store", "fdl_lmhead_workspace_bytes",
           "fdl_lmhead_confidence", "fdl_threshold_unmask",
           "fdl_lmhead_confidence_noalloc", "fdl_rope_table", "fdl_rmsnorm", "fdl_embed",
           "fdl_qkv_rope_store", "fdl_linear_residual", "fdl_linear_swiglu",
           "fdl_full_attention", "fdl_ffn", "fdl_qkv_attention", "fdl_model_create",
           "fdl_model_destroy", "fdl_generate_workspace_bytes", "fdl_generate")


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("seq_len", ctypes.c_int), ("block_start", ctypes.c_int),
                ("block_len", ctypes.c_int), ("dtype", ctypes.c_int),
                ("scale", ctypes.c_float)]


ABI_VERSION = 6


class LMHeadDesc(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("hidden", ctypes.c_int),
                ("vocab", ctypes.c_int), ("dtype", ctypes.c_int)]


class UnmaskDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seq_len", ctypes.c_int),
                ("block_start", ctypes.c_int), ("block_len", ctypes.c_int),
                ("tau", ctypes.c_float)]


class QKVDesc(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("batch", ctypes.c_int), ("seq_len", ctypes.c_int),
                ("rows_per_seq", ctypes.c_int), ("pos0", ctypes.c_int),
                ("max_pos", ctypes.c_int)]


class ModelDesc(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int), ("hidden", ctypes.c_int), ("n_layers", ctypes.c_int),
                ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int), ("mask_id", ctypes.c_int),
                ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("attn_norm", ctypes.c_void_p), ("w_qkv", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("wo", ctypes.c_void_p),
                ("ffn_norm", ctypes.c_void_p), ("w_gu", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p)]


class ModelWeights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p), ("layers", ctypes.POINTER(LayerWeights))]


FDL_CACHE_DUAL, FDL_CACHE_PREFIX, FDL_CACHE_NONE = 0, 1, 2
CACHE_MODES = {"dual": FDL_CACHE_DUAL, "prefix": FDL_CACHE_PREFIX, "none": FDL_CACHE_NONE}


class GenerateOpts(ctypes.Structure):
    _fields_ = [("cache", ctypes.c_int), ("device_loop", ctypes.c_int),
                ("bias_tok", ctypes.c_void_p), ("bias_val", ctypes.c_void_p),
                ("batching", ctypes.c_int)]


BATCHING = {"lockstep": 0, "compact": 1, "per_sequence": 2}


class FdlError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"fdllm error {code}: {msg}")
        self.code = code


_lib = None


def load() -> ctypes.CDLL:
    """Load libfdllm.so and declare its signatures (raises if not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m block_kv_cache_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.fdl_abi_version.restype = i
    if L.fdl_abi_version() != ABI_VERSION:
        raise RuntimeError(f"{LIB_PATH} has ABI {L.fdl_abi_version()}, this binding expects "
                           f"{ABI_VERSION}: rebuild with `python -m block_kv_cache_b200.build`")
    L.fdl_create.argtypes = [ctypes.POINTER(vp), i]
    L.fdl_destroy.argtypes = [vp]
    L.fdl_last_error.restype = ctypes.c_char_p
    L.fdl_get_device_status.argtypes = [vp, vp]
    L.fdl_set_wait_timeout.argtypes = [vp, ctypes.c_uint64]
    L.fdl_attention_workspace_bytes.argtypes = [vp, ctypes.POINTER(AttnDesc)]
    L.fdl_attention_workspace_bytes.restype = sz
    L.fdl_dualcache_attention.argtypes = [vp, ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp,
                                          vp, sz, vp]
    L.fdl_kv_store.argtypes = [vp, ctypes.POINTER(AttnDesc), vp, vp, i, i, vp, vp, vp]
    L.fdl_lmhead_workspace_bytes.argtypes = [vp, ctypes.POINTER(LMHeadDesc)]
    L.fdl_lmhead_workspace_bytes.restype = sz
    L.fdl_lmhead_confidence.argtypes = [vp, ctypes.POINTER(LMHeadDesc), vp, vp, vp, vp, vp,
                                        vp, vp, sz, vp]
    L.fdl_lmhead_confidence_noalloc.argtypes = [vp, ctypes.POINTER(LMHeadDesc), vp, vp, vp, vp,
                                                vp, vp, vp]
    L.fdl_threshold_unmask.argtypes = [vp, ctypes.POINTER(UnmaskDesc), vp, vp, vp, vp, vp,
                                       vp, vp]
    L.fdl_rope_table.argtypes = [ctypes.c_double, i, i, vp]
    L.fdl_rmsnorm.argtypes = [vp, i, i, vp, vp, vp, ctypes.c_float, vp, vp]
    L.fdl_embed.argtypes = [vp, i, i, vp, vp, vp, vp, vp]
    L.fdl_qkv_rope_store.argtypes = [vp, ctypes.POINTER(QKVDesc), vp, vp, vp, vp, vp, vp, vp, vp]
    L.fdl_linear_residual.argtypes = [vp, i, i, i, vp, vp, vp, vp]
    L.fdl_linear_swiglu.argtypes = [vp, i, i, i, vp, vp, vp, vp]
    L.fdl_full_attention.argtypes = [vp, ctypes.POINTER(AttnDesc), vp, vp, vp, vp, vp]
    fl = ctypes.c_float
    L.fdl_ffn.argtypes = [vp, i, i, i, vp, fl, vp, vp, vp, vp, vp, vp]
    L.fdl_qkv_attention.argtypes = [vp, ctypes.POINTER(QKVDesc), vp, vp, fl, vp, vp, vp, vp, vp,
                                    vp, vp, vp, vp]
    L.fdl_model_create.argtypes = [ctypes.POINTER(ModelDesc), ctypes.POINTER(ModelWeights),
                                   ctypes.POINTER(vp)]
    L.fdl_model_destroy.argtypes = [vp]
    L.fdl_generate_workspace_bytes.argtypes = [vp, vp, i, i, i]
    L.fdl_generate_workspace_bytes.restype = sz
    L.fdl_generate.argtypes = [vp, vp, vp, i, i, i, i, fl, ctypes.POINTER(GenerateOpts), vp,
                               ctypes.POINTER(i), vp, sz, vp]
    for name in EXPORTS:
        getattr(L, name).restype = getattr(L, name).restype or i
    _lib = L
    return L


def _check(rc: int):
    if rc != FDL_OK:
        raise FdlError(rc, load().fdl_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return FDL_F32
    if t.dtype == torch.bfloat16:
        return FDL_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t: torch.Tensor, name: str, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def rope_table(theta: float, max_pos: int, head_dim: int):
    """(cos, sin) table of rotate-half RoPE as a host float32 array [max_pos, head_dim/2, 2]
    (computed by the library in double precision)."""
    import numpy as np
    out = np.empty((max_pos, head_dim // 2, 2), np.float32)
    _check(load().fdl_rope_table(float(theta), int(max_pos), int(head_dim),
                                 ctypes.c_void_p(out.ctypes.data)))
    return out


class Model:
    """A model recorded in the library (fdl_model_create): the description and
    the device pointers of the weights, which the caller keeps alive.
    `layers` holds per layer the tensors attn_norm, w_qkv, bias (or None), wo,
    ffn_norm, w_gu, wd."""

    def __init__(self, *, vocab, hidden, n_q_heads, n_kv_heads, ffn, mask_id, embed,
                 final_norm, lm_head, layers, head_dim=128, rope_theta=10000.0, rms_eps=1e-5):
        L = load()
        self._keep = (embed, final_norm, lm_head, layers)
        self.desc = ModelDesc(vocab, hidden, len(layers), n_q_heads, n_kv_heads, head_dim, ffn,
                              mask_id, rope_theta, rms_eps)
        arr = (LayerWeights * len(layers))()
        for k, Lw in enumerate(layers):
            arr[k] = LayerWeights(Lw["attn_norm"].data_ptr(), Lw["w_qkv"].data_ptr(),
                                  Lw["bias"].data_ptr() if Lw.get("bias") is not None else None,
                                  Lw["wo"].data_ptr(), Lw["ffn_norm"].data_ptr(),
                                  Lw["w_gu"].data_ptr(), Lw["wd"].data_ptr())
        w = ModelWeights(embed.data_ptr(), final_norm.data_ptr(), lm_head.data_ptr(), arr)
        h = ctypes.c_void_p()
        _check(L.fdl_model_create(ctypes.byref(self.desc), ctypes.byref(w), ctypes.byref(h)))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            load().fdl_model_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Context:
    """One library context on one CUDA device. Holds a torch-allocated scratch
    buffer that grows to the largest workspace asked for."""

    def __init__(self, device: int | None = None):
        L = load()
        self.device = torch.cuda.current_device() if device is None else int(device)
        h = ctypes.c_void_p()
        _check(L.fdl_create(ctypes.byref(h), self.device))
        self._h = h
        self._ws = None

    def close(self):
        if getattr(self, "_h", None):
            load().fdl_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- scratch ---------------------------------------------------------
    def workspace(self, nbytes: int) -> torch.Tensor:
        nbytes = max(int(nbytes), 16)
        if self._ws is None or self._ws.numel() < nbytes:
            self._ws = torch.empty(nbytes, dtype=torch.uint8, device=f"cuda:{self.device}")
        return self._ws

    def set_wait_timeout(self, ns: int):
        """Limit (ns) of the kernels' progress waits on this context
        (fdl_set_wait_timeout)."""
        _check(load().fdl_set_wait_timeout(self._h, int(ns)))

    def device_status(self, stream=None) -> int:
        """Synchronise and raise FdlError if a kernel recorded a device error."""
        _check(load().fdl_get_device_status(self._h, _stream(stream)))
        return FDL_OK

    # -- (a) attention ----------------------------------------------------
    def attn_desc(self, q, k_cache, block_start, scale=0.0) -> AttnDesc:
        b, B, Hq, d = q.shape
        _, Hkv, L, _ = k_cache.shape
        return AttnDesc(b, Hq, Hkv, d, L, int(block_start), B, _dtype_code(q), float(scale))

    def attention_workspace_bytes(self, desc: AttnDesc) -> int:
        return int(load().fdl_attention_workspace_bytes(self._h, ctypes.byref(desc)))

    def dualcache_attention(self, q, k_cache, v_cache, block_start, *, out=None, lse=None,
                            want_lse=False, scale=0.0, ws=None, stream=None):
        for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
            _need(t, n, q.dtype, 4)
        d = self.attn_desc(q, k_cache, block_start, scale)
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty((d.batch, d.n_q_heads, d.block_len), dtype=torch.float32,
                              device=q.device)
        need = self.attention_workspace_bytes(d)
        if ws is None:
            ws = self.workspace(need)
        _check(load().fdl_dualcache_attention(self._h, ctypes.byref(d), _ptr(q), _ptr(k_cache),
                                              _ptr(v_cache), _ptr(out), _ptr(lse), _ptr(ws),
                                              ws.numel() * ws.element_size(), _stream(stream)))
        return (out, lse) if (want_lse or lse is not None) else out

    def kv_store(self, k_new, v_new, k_cache, v_cache, start, stream=None):
        _need(k_new, "k_new", k_cache.dtype, 4)
        _need(v_new, "v_new", k_cache.dtype, 4)
        _need(k_cache, "k_cache", None, 4)
        _need(v_cache, "v_cache", k_cache.dtype, 4)
        b, Hkv, L, d = k_cache.shape
        n = k_new.shape[1]
        desc = AttnDesc(b, Hkv, Hkv, d, L, 0, 1, _dtype_code(k_cache), 0.0)
        _check(load().fdl_kv_store(self._h, ctypes.byref(desc), _ptr(k_new), _ptr(v_new),
                                   int(start), int(n), _ptr(k_cache), _ptr(v_cache),
                                   _stream(stream)))

    # -- (b) LM head + confidence ----------------------------------------
    def lmhead_workspace_bytes(self, desc: LMHeadDesc) -> int:
        return int(load().fdl_lmhead_workspace_bytes(self._h, ctypes.byref(desc)))

    def lmhead_confidence(self, h, w, bias_tok=None, bias_val=None, *, conf=None, tok=None,
                          ws=None, stream=None):
        _need(h, "h", None, 2)
        _need(w, "w", h.dtype, 2)
        if bias_tok is not None:
            _need(bias_tok, "bias_tok", torch.int32, 1)
            _need(bias_val, "bias_val", torch.float32, 1)
        M, D = h.shape
        V = w.shape[0]
        d = LMHeadDesc(M, D, V, _dtype_code(h))
        if conf is None:
            conf = torch.empty(M, dtype=torch.float32, device=h.device)
        if tok is None:
            tok = torch.empty(M, dtype=torch.int32, device=h.device)
        if ws is None:
            ws = self.workspace(self.lmhead_workspace_bytes(d))
        _check(load().fdl_lmhead_confidence(self._h, ctypes.byref(d), _ptr(h), _ptr(w),
                                            _ptr(bias_tok), _ptr(bias_val), _ptr(conf),
                                            _ptr(tok), _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)))
        return conf, tok

    def lmhead_confidence_noalloc(self, h, w, bias_tok=None, bias_val=None, *, conf=None,
                                  tok=None, stream=None):
        """fdl_lmhead_confidence_noalloc: no workspace argument; the library's
        built-in 8 MiB scratch array is used (see include/fdllm.h)."""
        _need(h, "h", None, 2)
        _need(w, "w", h.dtype, 2)
        if bias_tok is not None:
            _need(bias_tok, "bias_tok", torch.int32, 1)
            _need(bias_val, "bias_val", torch.float32, 1)
        M, D = h.shape
        d = LMHeadDesc(M, D, w.shape[0], _dtype_code(h))
        if conf is None:
            conf = torch.empty(M, dtype=torch.float32, device=h.device)
        if tok is None:
            tok = torch.empty(M, dtype=torch.int32, device=h.device)
        _check(load().fdl_lmhead_confidence_noalloc(self._h, ctypes.byref(d), _ptr(h), _ptr(w),
                                                    _ptr(bias_tok), _ptr(bias_val), _ptr(conf),
                                                    _ptr(tok), _stream(stream)))
        return conf, tok

    # -- (b) threshold select + scatter -----------------------------------
    def threshold_unmask(self, conf, tok, x, masked, block_start, tau, *, remaining=None,
                         n_decoded=None, stream=None):
        _need(conf, "conf", torch.float32, 2)
        _need(tok, "tok", torch.int32, 2)
        _need(x, "x", torch.int32, 2)
        _need(masked, "masked", torch.uint8, 2)
        b, L = x.shape
        B = conf.shape[1]
        if remaining is None:
            remaining = torch.empty(b, dtype=torch.int32, device=x.device)
        d = UnmaskDesc(b, L, int(block_start), B, float(tau))
        _check(load().fdl_threshold_unmask(self._h, ctypes.byref(d), _ptr(conf), _ptr(tok),
                                           _ptr(x), _ptr(masked), _ptr(remaining),
                                           _ptr(n_decoded), _stream(stream)))
        return remaining

    # -- transformer scaffold ------------------------------------------------
    def rmsnorm(self, h, weight, eps, *, out=None, row_map=None, rows=None, stream=None):
        """bf16 RMSNorm of f32 rows of h (optionally gathered through row_map)."""
        _need(h, "h", torch.float32, 2)
        _need(weight, "weight", torch.float32, 1)
        n = rows if rows is not None else (row_map.numel() if row_map is not None else h.shape[0])
        if out is None:
            out = torch.empty((n, h.shape[1]), dtype=torch.bfloat16, device=h.device)
        _check(load().fdl_rmsnorm(self._h, int(n), h.shape[1], _ptr(h), _ptr(row_map),
                                  _ptr(weight), float(eps), _ptr(out), _stream(stream)))
        return out

    def embed(self, ids, table, *, out=None, row_map=None, stream=None):
        """f32 rows of the embedding table: table[ids[row_map[i]]] (or ids[i])."""
        _need(ids, "ids", torch.int32, None)
        _need(table, "table", torch.bfloat16, 2)
        n = row_map.numel() if row_map is not None else ids.numel()
        if out is None:
            out = torch.empty((n, table.shape[1]), dtype=torch.float32, device=ids.device)
        _check(load().fdl_embed(self._h, int(n), table.shape[1], _ptr(ids), _ptr(row_map),
                                _ptr(table), _ptr(out), _stream(stream)))
        return out

    def qkv_rope_store(self, x, w, rope, q_out, k_cache, v_cache, *, n_q_heads, rows_per_seq,
                       pos0, bias=None, stream=None):
        """[q|k|v] = x w^T (+bias), RoPE on q and k, q -> q_out, k/v -> caches."""
        _need(x, "x", torch.bfloat16, 2)
        _need(w, "w", torch.bfloat16, 2)
        b, hkv, L, d = k_cache.shape
        d_ = QKVDesc(x.shape[0], x.shape[1], int(n_q_heads), hkv, d, b, L, int(rows_per_seq),
                     int(pos0), rope.shape[0])
        _check(load().fdl_qkv_rope_store(self._h, ctypes.byref(d_), _ptr(x), _ptr(w),
                                         _ptr(bias), _ptr(rope), _ptr(q_out), _ptr(k_cache),
                                         _ptr(v_cache), _stream(stream)))
        return q_out

    def qkv_attention(self, x, w, rope, q_out, k_cache, v_cache, out, *, n_q_heads,
                      rows_per_seq, pos0, bias=None, h=None, norm_w=None, eps=1e-5,
                      stream=None):
        """[x = RMSNorm(h) * norm_w if norm_w is given], qkv_rope_store of the block
        rows, then DualCache attention of the block [pos0, pos0 + rows_per_seq) of
        every sequence over the caches -> out."""
        _need(x, "x", torch.bfloat16, 2)
        _need(w, "w", torch.bfloat16, 2)
        if norm_w is not None:
            _need(h, "h", torch.float32, 2)
        b, hkv, L, d = k_cache.shape
        d_ = QKVDesc(x.shape[0], x.shape[1], int(n_q_heads), hkv, d, b, L, int(rows_per_seq),
                     int(pos0), rope.shape[0])
        _check(load().fdl_qkv_attention(self._h, ctypes.byref(d_), _ptr(h), _ptr(norm_w),
                                        float(eps), _ptr(x), _ptr(w), _ptr(bias), _ptr(rope),
                                        _ptr(q_out), _ptr(k_cache), _ptr(v_cache), _ptr(out),
                                        _stream(stream)))
        return out

    def generate(self, model: Model, prompt, gen_len, *, block=32, tau=0.9, cache="dual",
                 bias_tok=None, bias_val=None, device_loop=False, batching="lockstep",
                 stream=None):
        """The whole decode in the library (fdl_generate). prompt [b, P] int32,
        a CUDA tensor or a host tensor (then copied to the device first, and
        the result copied back to a host tensor: the public call with host
        buffers). cache: "dual", "prefix" or "none"; bias_tok / bias_val [b,
        gen_len] (CUDA, int32 / float32): optional planted logit bias of the
        generated positions. device_loop: the decode as one CUDA graph with the
        steps sequenced on the device (kept in the context for the next call
        with the same arguments; the workspace is kept by this Context so that
        it does). batching (DualCache, host loop for the last two): "lockstep",
        "compact" (cached steps only on the sequences with masked positions
        left in the block) or "per_sequence" (each sequence moves to its next
        block on its own). Returns (x [b, P + gen_len] int32, steps)."""
        on_host = not prompt.is_cuda
        dev = torch.device("cuda", self.device)
        if on_host:
            prompt = prompt.to(dev, non_blocking=True)
        _need(prompt, "prompt", torch.int32, 2)
        b, P = prompt.shape
        if bias_tok is not None:
            _need(bias_tok, "bias_tok", torch.int32, 2)
            _need(bias_val, "bias_val", torch.float32, 2)
        L = load()
        n = L.fdl_generate_workspace_bytes(self._h, model._h, b, P + gen_len, int(block))
        if n == 0:
            raise ValueError("generate: bad shape")
        if getattr(self, "_gen_ws", None) is None or self._gen_ws.numel() < n:
            self._gen_ws = None
            self._gen_ws = torch.empty(n, dtype=torch.uint8, device=dev)
        ws = self._gen_ws
        x = torch.empty((b, P + gen_len), dtype=torch.int32, device=dev)
        steps = ctypes.c_int(0)
        opts = GenerateOpts(CACHE_MODES[cache], int(bool(device_loop)),
                            None if bias_tok is None else bias_tok.data_ptr(),
                            None if bias_val is None else bias_val.data_ptr(),
                            BATCHING[batching])
        _check(L.fdl_generate(self._h, model._h, _ptr(prompt), b, P, int(gen_len), int(block),
                              float(tau), ctypes.byref(opts), _ptr(x), ctypes.byref(steps),
                              _ptr(ws), ws.numel(), _stream(stream)))
        if on_host:
            x = x.cpu()
        return x, steps.value

    def linear_residual(self, x, w, h, *, stream=None):
        """h += x w^T (h f32)."""
        _need(x, "x", torch.bfloat16, 2)
        _need(w, "w", torch.bfloat16, 2)
        _need(h, "h", torch.float32, 2)
        _check(load().fdl_linear_residual(self._h, x.shape[0], w.shape[0], x.shape[1], _ptr(x),
                                          _ptr(w), _ptr(h), _stream(stream)))
        return h

    def linear_swiglu(self, x, w_gu, *, out=None, stream=None):
        """silu(x Wg^T) * (x Wu^T) with gate/up rows interleaved in w_gu."""
        _need(x, "x", torch.bfloat16, 2)
        _need(w_gu, "w_gu", torch.bfloat16, 2)
        F = w_gu.shape[0] // 2
        if out is None:
            out = torch.empty((x.shape[0], F), dtype=torch.bfloat16, device=x.device)
        _check(load().fdl_linear_swiglu(self._h, x.shape[0], F, x.shape[1], _ptr(x), _ptr(w_gu),
                                        _ptr(out), _stream(stream)))
        return out

    def ffn(self, x, w_gu, w_down, h, *, f=None, norm_w=None, eps=1e-5, stream=None):
        """[x = RMSNorm(h) * norm_w if norm_w is given], then
        h += (silu(x Wg^T) * (x Wu^T)) Wd^T; returns f, the SwiGLU output."""
        _need(x, "x", torch.bfloat16, 2)
        _need(w_gu, "w_gu", torch.bfloat16, 2)
        _need(w_down, "w_down", torch.bfloat16, 2)
        _need(h, "h", torch.float32, 2)
        rows, hidden = x.shape
        F = w_gu.shape[0] // 2
        if f is None:
            f = torch.empty((rows, F), dtype=torch.bfloat16, device=x.device)
        _check(load().fdl_ffn(self._h, rows, hidden, F, _ptr(norm_w), float(eps), _ptr(x),
                              _ptr(w_gu), _ptr(w_down), _ptr(f), _ptr(h), _stream(stream)))
        return f

    def full_attention(self, q, k_cache, v_cache, *, q_start=0, out=None, scale=0.0,
                       stream=None):
        """Bidirectional attention of the positions [q_start, L) over all L
        positions of the caches: q, out [b, L - q_start, Hq, d] (q_start = 0:
        every position, the refresh; q_start = s: the block and the suffix of a
        PrefixCache step)."""
        _need(q, "q", torch.bfloat16, 4)
        _need(k_cache, "k_cache", torch.bfloat16, 4)
        _need(v_cache, "v_cache", torch.bfloat16, 4)
        b, nq, Hq, d = q.shape
        hkv, L = k_cache.shape[1], k_cache.shape[2]
        if nq != L - int(q_start):
            raise ValueError(f"full_attention: q has {nq} rows per sequence, the caches "
                             f"{L} - q_start {q_start}")
        desc = AttnDesc(b, Hq, hkv, d, L, int(q_start), nq, FDL_BF16, float(scale))
        if out is None:
            out = torch.empty_like(q)
        _check(load().fdl_full_attention(self._h, ctypes.byref(desc), _ptr(q), _ptr(k_cache),
                                         _ptr(v_cache), _ptr(out), _stream(stream)))
        return out
