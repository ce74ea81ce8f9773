"""Python binding of the B200 decoder library (liblfwd.so, C ABI in include/llama_fwd.h).

Argument marshalling only: every step of the forward pass runs in the library's
CUDA kernels. The functions below carry the C names; ``Model`` bundles a model
handle with the tensors whose device pointers it holds. There is no fallback:
if the shared library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional

import torch

from .build import LIB as _LIB_PLAIN, LIB_CHECKED as _LIB_CHECKED

# LLM_LIB_VARIANT=checked selects the bounds-checking build (liblfwd_checked.so).
LIB_PATH = _LIB_CHECKED if os.environ.get("LLM_LIB_VARIANT") == "checked" else _LIB_PLAIN

LLM_OK = 0
LLM_ERR_BAD_CONFIG = -1
LLM_ERR_NULL_PTR = -2
LLM_ERR_SEQ_OVERFLOW = -3
LLM_ERR_BATCH = -4
LLM_ERR_CUDA = -5
LLM_ERR_DEVICE_TIMEOUT = -6
LLM_ERR_UNSUPPORTED = -7
LLM_ERR_BAD_ARG = -8
LLM_ERR_DEVICE_BOUNDS = -9
LLM_BUILD_BOUNDS_CHECK = 1
LLM_F32 = 0
LLM_BF16 = 1
LLM_FLAG_CUDA_GRAPH = 1
LLM_FLAG_DEBUG_TAPS = 2
LLM_FLAG_KERNEL_TIMING = 4
LLM_FLAG_PDL = 8
LLM_FLAG_FUSED_DECODE = 16
KERNEL_KINDS = ("embed", "qkv", "attn", "wo", "w13", "w2", "head", "out", "step")


class llm_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("dim", "n_layers", "n_heads", "n_kv_heads", "head_dim",
                                            "ffn_hidden", "vocab", "max_seq_len", "max_batch", "max_tokens")] + \
               [("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_float)] + \
               [(n, ctypes.c_int) for n in ("dtype", "tie_embeddings", "has_embed_and_head", "flags")]


_PP = ctypes.POINTER(ctypes.c_void_p)


class llm_weights(ctypes.Structure):
    _fields_ = [("tok_emb", ctypes.c_void_p), ("out", ctypes.c_void_p), ("final_norm", ctypes.c_void_p)] + \
               [(n, _PP) for n in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w3", "w2")]


class LlmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"llm error {code}: {msg}")
        self.code = code


_lib = None
_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

_SIGS = {
    "llm_model_init": (_i, [ctypes.POINTER(llm_config), ctypes.POINTER(llm_weights), _vp, ctypes.POINTER(_vp)]),
    "llm_prefill": (_i, [_vp, _vp, _i, _i, _vp, _vp]),
    "llm_prefill_hidden": (_i, [_vp, _vp, _i, _i, _vp]),
    "llm_decode_step": (_i, [_vp, _i, _vp, _vp, _vp]),
    "llm_decode_step_hidden": (_i, [_vp, _i, _vp, _vp]),
    "llm_kv_cache_reset": (_i, [_vp]),
    "llm_kv_cache_view": (_i, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_int64)]),
    "llm_kv_cache_set_lens": (_i, [_vp, ctypes.POINTER(ctypes.c_int32), _i]),
    "llm_kv_cache_get_lens": (_i, [_vp, ctypes.POINTER(ctypes.c_int32), _i]),
    "llm_debug_tap": (_i, [_vp, _i, _vp, _sz]),
    "llm_kernel_times": (_i, [_vp, _i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), _i]),
    "llm_debug_wait_probe": (_i, [_vp, _i, ctypes.c_double]),
    "llm_synchronize": (_i, [_vp]),
    "llm_build_flags": (_i, []),
    "llm_op_synchronize": (_i, [_vp]),
    "llm_model_free": (None, [_vp]),
    "llm_last_error": (ctypes.c_char_p, []),
    "llm_op_gemm_bf16": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "llm_op_gemv_workspace": (_sz, [_i, _i]),
    "llm_op_gemv_bf16": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "llm_op_attention_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "llm_op_attention_decode_workspace": (_sz, [_i, _i, _i, _i, _i]),
    "llm_op_attention_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "llm_op_attention_decode_static": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "llm_op_attention_decode_cluster": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
}


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load liblfwd.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"CUDA library not built: {p} is missing "
                          "(run python -m llama_decoder_forward_fwd_b200.build)")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGS.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def exported_symbols() -> List[str]:
    return list(_SIGS)


def check(rc: int):
    if rc != LLM_OK:
        raise LlmError(rc, load().llm_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        return None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------- C names
def llm_model_init(cfg: llm_config, w: llm_weights, stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    check(load().llm_model_init(ctypes.byref(cfg), ctypes.byref(w), _stream_ptr(stream), ctypes.byref(h)))
    return h


def llm_prefill(m, tokens: torch.Tensor, next_tok: torch.Tensor, logits: Optional[torch.Tensor] = None):
    B, T = tokens.shape
    check(load().llm_prefill(m, _ptr(tokens), B, T, _ptr(next_tok), _ptr(logits)))


def llm_prefill_hidden(m, h_in: torch.Tensor, h_out: torch.Tensor):
    B, T, _ = h_in.shape
    check(load().llm_prefill_hidden(m, _ptr(h_in), B, T, _ptr(h_out)))


def llm_decode_step(m, in_tok: torch.Tensor, next_tok: torch.Tensor, logits: Optional[torch.Tensor] = None):
    check(load().llm_decode_step(m, in_tok.shape[0], _ptr(in_tok), _ptr(next_tok), _ptr(logits)))


def llm_decode_step_hidden(m, h_in: torch.Tensor, h_out: torch.Tensor):
    check(load().llm_decode_step_hidden(m, h_in.shape[0], _ptr(h_in), _ptr(h_out)))


def llm_kv_cache_reset(m):
    check(load().llm_kv_cache_reset(m))


def llm_kv_cache_view(m):
    k, v = ctypes.c_void_p(), ctypes.c_void_p()
    st = (ctypes.c_int64 * 4)()
    check(load().llm_kv_cache_view(m, ctypes.byref(k), ctypes.byref(v), st))
    return k.value, v.value, list(st)


def llm_kv_cache_set_lens(m, lens: List[int]):
    arr = (ctypes.c_int32 * len(lens))(*lens)
    check(load().llm_kv_cache_set_lens(m, arr, len(lens)))


def llm_kv_cache_get_lens(m, B: int) -> List[int]:
    arr = (ctypes.c_int32 * B)()
    check(load().llm_kv_cache_get_lens(m, arr, B))
    return list(arr)


def llm_debug_tap(m, layer: int, dst: torch.Tensor):
    check(load().llm_debug_tap(m, layer, _ptr(dst), dst.numel()))


def llm_kernel_times(m, reset: bool = True):
    """{kind: (total ms, launches)} since the last reset (needs LLM_FLAG_KERNEL_TIMING)."""
    n = len(KERNEL_KINDS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    check(load().llm_kernel_times(m, n, ms, cnt, int(reset)))
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}


def llm_debug_wait_probe(m, which: int, limit_ms: float):
    """Queue a bounded device wait that cannot complete (0: mbarrier, 1: grid barrier)."""
    check(load().llm_debug_wait_probe(m, which, float(limit_ms)))


def llm_synchronize(m):
    check(load().llm_synchronize(m))


def llm_build_flags() -> int:
    return load().llm_build_flags()


def llm_op_synchronize(stream=None):
    check(load().llm_op_synchronize(_stream_ptr(stream)))


def llm_model_free(m):
    load().llm_model_free(m)


def llm_op_gemm_bf16(A, B, C, stream=None):
    M, K = A.shape
    N = B.shape[0]
    check(load().llm_op_gemm_bf16(_ptr(A), _ptr(B), _ptr(C), M, N, K, _stream_ptr(stream)))


def llm_op_gemv_workspace(N, K) -> int:
    return load().llm_op_gemv_workspace(N, K)


def llm_op_gemv_bf16(x, W, y, workspace, stream=None):
    M, K = x.shape
    N = W.shape[0]
    check(load().llm_op_gemv_bf16(_ptr(x), _ptr(W), _ptr(y), M, N, K, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream_ptr(stream)))


def _dt(t: torch.Tensor) -> int:
    return LLM_BF16 if t.dtype == torch.bfloat16 else LLM_F32


def llm_op_attention_prefill(q, kc, vc, pos0, out, stream=None):
    """q [B,T,H,d]; kc, vc [B,Hk,S_max,d]; pos0 int32 [B]; out [B,T,H*d]."""
    B, T, H, d = q.shape
    Hk, S = kc.shape[1], kc.shape[2]
    check(load().llm_op_attention_prefill(_ptr(q), _ptr(kc), _ptr(vc), _ptr(pos0), _ptr(out), B, T, H, Hk, d, S,
                                          _dt(q), _stream_ptr(stream)))


def llm_op_attention_decode_workspace(B, T, H, Hk, d) -> int:
    return load().llm_op_attention_decode_workspace(B, T, H, Hk, d)


def llm_op_attention_decode(q, kc, vc, pos0, out, workspace, stream=None):
    B, T, H, d = q.shape
    Hk, S = kc.shape[1], kc.shape[2]
    check(load().llm_op_attention_decode(_ptr(q), _ptr(kc), _ptr(vc), _ptr(pos0), _ptr(out), B, T, H, Hk, d, S,
                                         _dt(q), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                         _stream_ptr(stream)))


# ---------------------------------------------------------------- convenience
def make_config(shape, max_batch: int, max_tokens: int = 0, flags: int = 0) -> llm_config:
    """llm_config from a seeded_inputs.ModelShape-like object."""
    return llm_config(dim=shape.dim, n_layers=shape.n_layers, n_heads=shape.n_heads, n_kv_heads=shape.n_kv_heads,
                      head_dim=shape.head_dim, ffn_hidden=shape.ffn_hidden, vocab=shape.vocab,
                      max_seq_len=shape.max_seq_len, max_batch=max_batch, max_tokens=max_tokens,
                      norm_eps=shape.norm_eps, rope_theta=shape.rope_theta,
                      dtype=LLM_F32 if shape.dtype == "f32" else LLM_BF16,
                      tie_embeddings=int(shape.tie_embeddings), has_embed_and_head=int(shape.has_embed_and_head),
                      flags=flags)


class Model:
    """A model handle plus the device tensors it points into.

    ``glob`` and ``layers`` are the dicts made by ``seeded_inputs.make_weights``
    (tensors are moved to the GPU if needed and kept alive here).
    """

    def __init__(self, shape, glob: Dict[str, torch.Tensor], layers: List[Dict[str, torch.Tensor]],
                 max_batch: int, max_tokens: int = 0, flags: int = 0, stream=None, device="cuda"):
        self.shape = shape
        dev = torch.device(device)
        self.glob = {k: v.to(dev).contiguous() for k, v in glob.items()}
        self.layers = [{k: v.to(dev).contiguous() for k, v in lw.items()} for lw in layers]
        self.cfg = make_config(shape, max_batch, max_tokens, flags)
        L = shape.n_layers

        def arr(key):
            a = (ctypes.c_void_p * L)(*[lw[key].data_ptr() for lw in self.layers])
            return ctypes.cast(a, _PP), a

        self._keep = []
        fields = {}
        for key in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w3", "w2"):
            src = {"attn_norm": "attention_norm"}.get(key, key)
            p, a = arr(src)
            fields[key] = p
            self._keep.append(a)
        g = self.glob
        self.w = llm_weights(tok_emb=g["tok_embeddings"].data_ptr() if "tok_embeddings" in g else None,
                             out=g["output"].data_ptr() if "output" in g else None,
                             final_norm=g["norm"].data_ptr() if "norm" in g else None, **fields)
        torch.cuda.synchronize(dev)
        self.h = llm_model_init(self.cfg, self.w, stream)

    def kv_cache_tensors(self):
        """torch views [n_layers, max_batch, n_kv_heads, max_seq_len, head_dim] of the library's K and V caches."""
        k, v, st = llm_kv_cache_view(self.h)
        s, c = self.shape, self.cfg
        shp = (s.n_layers, c.max_batch, s.n_kv_heads, s.max_seq_len, s.head_dim)
        typestr = "<f4" if s.dtype == "f32" else "<i2"

        class _Dev:
            def __init__(self, ptr):
                self.__cuda_array_interface__ = {"shape": shp, "typestr": typestr, "data": (ptr, False),
                                                 "version": 3, "strides": None}

        out = []
        for ptr in (k, v):
            t = torch.as_tensor(_Dev(ptr), device="cuda")
            out.append(t if s.dtype == "f32" else t.view(torch.bfloat16))
        return out[0], out[1]

    def free(self):
        if self.h:
            llm_model_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def llm_op_attention_decode_cluster(q, kc, vc, pos0, out, stream=None):
    """Single-token decode attention on the tensor cores (bf16, head_dim 128, no workspace)."""
    B, T, H, d = q.shape
    Hk, S = kc.shape[1], kc.shape[2]
    check(load().llm_op_attention_decode_cluster(_ptr(q), _ptr(kc), _ptr(vc), _ptr(pos0), _ptr(out), B, H, Hk, S,
                                                 _stream_ptr(stream)))


def llm_op_attention_decode_static(q, kc, vc, pos0, out, stream=None):
    """As llm_op_attention_decode, on the library's fixed scratch (no workspace, no allocation)."""
    B, T, H, d = q.shape
    Hk, S = kc.shape[1], kc.shape[2]
    check(load().llm_op_attention_decode_static(_ptr(q), _ptr(kc), _ptr(vc), _ptr(pos0), _ptr(out), B, T, H, Hk, d,
                                                S, _dt(q), _stream_ptr(stream)))
