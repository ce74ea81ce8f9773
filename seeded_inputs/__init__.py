"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This module only draws random numbers and names workloads. It holds none of the
decoder's arithmetic: no normalisation, projection, rotation, attention or
activation. Both sides take their inputs from here, and neither imports the
other.

Every tensor has its own seed, derived from a workload seed and the tensor's
name, so one layer can be regenerated alone (the oracle walks a model layer by
layer to bound host memory). Weights are drawn N(0, 0.02) in fp32 and then
rounded to the model dtype (round-to-nearest-even for bf16); norm weights are 1.
Token ids are uniform in [0, vocab). Hidden-state inputs are N(0, 1) rounded to
bf16-representable values and kept as fp32.

Weight names follow the checkpoint keys the pages list ("Building llama3 from
scratch", the listing of the first keys of consolidated.00.pth): tok_embeddings,
layers.i.attention.{wq,wk,wv,wo}, layers.i.feed_forward.{w1,w2,w3},
layers.i.{attention_norm,ffn_norm}; the final norm is ``norm.weight`` and the
separate lm_head is ``output.weight``. Matrices are [out, in] row-major.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, Optional

import torch

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "tensor_seed", "layer_weight_names",
    "make_layer_weights", "make_global_weights", "make_weights", "make_tokens",
    "make_hidden", "make_kv_prefill",
]


@dataclasses.dataclass(frozen=True)
class ModelShape:
    dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn_hidden: int
    vocab: int
    max_seq_len: int
    norm_eps: float
    rope_theta: float
    dtype: str                 # "f32" or "bf16"
    tie_embeddings: bool
    has_embed_and_head: bool = True

    def replace(self, **kw) -> "ModelShape":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    batch: int
    prompt_len: int            # tokens (or hidden vectors) per sequence in prefill
    decode_steps: int
    input_kind: str            # "tokens" | "hidden" | "kv_prefilled"
    kv_len_range: Optional[tuple] = None   # for "kv_prefilled": (lo, hi) inclusive
    seed: int = 1234


_LLAMA3_8B = ModelShape(dim=4096, n_layers=32, n_heads=32, n_kv_heads=8, head_dim=128,
                        ffn_hidden=14336, vocab=128256, max_seq_len=8192 + 256,
                        norm_eps=1e-5, rope_theta=500000.0, dtype="bf16",
                        tie_embeddings=False)

WORKLOADS: Dict[str, Workload] = {
    # Tiny Llama-2-architecture decoder in fp32 (stories15M shape), tied lm_head.
    "tiny-llama2-f32-d288-b1-p8-g50": Workload(
        name="tiny-llama2-f32-d288-b1-p8-g50",
        shape=ModelShape(dim=288, n_layers=6, n_heads=6, n_kv_heads=6, head_dim=48,
                         ffn_hidden=768, vocab=32000, max_seq_len=256, norm_eps=1e-5,
                         rope_theta=10000.0, dtype="f32", tie_embeddings=True),
        batch=1, prompt_len=8, decode_steps=50, input_kind="tokens"),
    # One Llama-3-8B-shaped decoder layer fed N(0,1) hidden states.
    "llama3-8b-1layer-bf16-b1-h512-d64": Workload(
        name="llama3-8b-1layer-bf16-b1-h512-d64",
        shape=_LLAMA3_8B.replace(n_layers=1, has_embed_and_head=False, max_seq_len=1024),
        batch=1, prompt_len=512, decode_steps=64, input_kind="hidden"),
    # Full Llama-3-8B architecture: 2048-token prefill, 256 greedy decode steps.
    "llama3-8b-bf16-b1-p2048-g256": Workload(
        name="llama3-8b-bf16-b1-p2048-g256",
        shape=_LLAMA3_8B.replace(max_seq_len=2048 + 256),
        batch=1, prompt_len=2048, decode_steps=256, input_kind="tokens"),
    # Batched decode over KV caches pre-filled to ragged lengths in [4096, 8192].
    "llama3-8b-bf16-b16-kv4k8k-g128": Workload(
        name="llama3-8b-bf16-b16-kv4k8k-g128",
        shape=_LLAMA3_8B.replace(max_seq_len=8192 + 128),
        batch=16, prompt_len=0, decode_steps=128, input_kind="kv_prefilled",
        kv_len_range=(4096, 8192)),
    # Long-context single-sequence decode: the cache pre-filled to 8064 positions,
    # 128 greedy steps up to the 8192-position Llama-3 context.
    "llama3-8b-bf16-b1-kv8k-g128": Workload(
        name="llama3-8b-bf16-b1-kv8k-g128",
        shape=_LLAMA3_8B.replace(max_seq_len=8192),
        batch=1, prompt_len=0, decode_steps=128, input_kind="kv_prefilled",
        kv_len_range=(8064, 8064)),
    # Multi-query variant of the Llama-3-8B shape (one KV head for all 32 query
    # heads), otherwise the benchmark's configuration.
    "llama3-8b-mqa-bf16-b1-p2048-g256": Workload(
        name="llama3-8b-mqa-bf16-b1-p2048-g256",
        shape=_LLAMA3_8B.replace(n_kv_heads=1, max_seq_len=2048 + 256),
        batch=1, prompt_len=2048, decode_steps=256, input_kind="tokens"),
    # Llama-2-7B-shaped multi-head (no GQA) model, batch 8.
    "llama2-7b-mha-bf16-b8-p1024-g256": Workload(
        name="llama2-7b-mha-bf16-b8-p1024-g256",
        shape=ModelShape(dim=4096, n_layers=32, n_heads=32, n_kv_heads=32, head_dim=128,
                         ffn_hidden=11008, vocab=32000, max_seq_len=4096, norm_eps=1e-5,
                         rope_theta=10000.0, dtype="bf16", tie_embeddings=False),
        batch=8, prompt_len=1024, decode_steps=256, input_kind="tokens"),
}


def tensor_seed(seed: int, name: str) -> int:
    """A stable 63-bit seed for one named tensor of one workload seed."""
    h = hashlib.sha256(f"{seed}/{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _generator(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(tensor_seed(seed, name))
    return g


def _normal(shape, std, dtype, seed, name, device) -> torch.Tensor:
    g = _generator(seed, name, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def layer_weight_names(i: int):
    p = f"layers.{i}."
    return {
        "wq": p + "attention.wq.weight", "wk": p + "attention.wk.weight",
        "wv": p + "attention.wv.weight", "wo": p + "attention.wo.weight",
        "w1": p + "feed_forward.w1.weight", "w2": p + "feed_forward.w2.weight",
        "w3": p + "feed_forward.w3.weight",
        "attention_norm": p + "attention_norm.weight", "ffn_norm": p + "ffn_norm.weight",
    }


def make_layer_weights(shape: ModelShape, seed: int, layer: int, device="cpu") -> Dict[str, torch.Tensor]:
    """Weights of one decoder layer, keyed by short name (wq, wk, ..., ffn_norm)."""
    D, H, Hk, d, F = shape.dim, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.ffn_hidden
    dt = shape.torch_dtype
    names = layer_weight_names(layer)
    dims = {"wq": (H * d, D), "wk": (Hk * d, D), "wv": (Hk * d, D), "wo": (D, H * d),
            "w1": (F, D), "w3": (F, D), "w2": (D, F)}
    out = {k: _normal(dims[k], 0.02, dt, seed, names[k], device) for k in dims}
    out["attention_norm"] = torch.ones(D, dtype=dt, device=device)
    out["ffn_norm"] = torch.ones(D, dtype=dt, device=device)
    return out


def make_global_weights(shape: ModelShape, seed: int, device="cpu") -> Dict[str, torch.Tensor]:
    """Embedding, final norm and (untied) lm_head; empty dict for layer-only shapes."""
    if not shape.has_embed_and_head:
        return {}
    dt = shape.torch_dtype
    out = {"tok_embeddings": _normal((shape.vocab, shape.dim), 0.02, dt, seed,
                                     "tok_embeddings.weight", device),
           "norm": torch.ones(shape.dim, dtype=dt, device=device)}
    if not shape.tie_embeddings:
        out["output"] = _normal((shape.vocab, shape.dim), 0.02, dt, seed, "output.weight", device)
    return out


def make_weights(shape: ModelShape, seed: int, device="cpu"):
    """(global weights dict, list of per-layer dicts)."""
    return (make_global_weights(shape, seed, device),
            [make_layer_weights(shape, seed, i, device) for i in range(shape.n_layers)])


def make_tokens(seed: int, batch: int, length: int, vocab: int, tag: str = "prompt") -> torch.Tensor:
    """int32 [batch, length] uniform in [0, vocab) (CPU)."""
    g = _generator(seed, f"tokens/{tag}", "cpu")
    return torch.randint(0, vocab, (batch, length), generator=g, dtype=torch.int64).to(torch.int32)


def make_hidden(seed: int, batch: int, length: int, dim: int, tag: str = "prompt") -> torch.Tensor:
    """fp32 [batch, length, dim] of N(0,1) draws rounded to bf16-representable values (CPU)."""
    return _normal((batch, length, dim), 1.0, torch.bfloat16, seed,
                   f"hidden/{tag}", "cpu").to(torch.float32)


def make_kv_prefill(shape: ModelShape, seed: int, batch: int, lo: int, hi: int,
                    layers=None, device="cpu"):
    """Ragged pre-filled KV caches: lengths ~ U[lo, hi] per sequence and N(0,1) cache values.

    Returns (lens int32 [batch], {layer: (K, V)}) with K, V of shape
    [batch, n_kv_heads, hi, head_dim] in the model dtype; entries at positions
    >= lens[b] are drawn too but never read.
    """
    g = _generator(seed, "kv/lens", "cpu")
    lens = torch.randint(lo, hi + 1, (batch,), generator=g, dtype=torch.int64).to(torch.int32)
    layers = range(shape.n_layers) if layers is None else layers
    caches = {}
    for l in layers:
        shp = (batch, shape.n_kv_heads, hi, shape.head_dim)
        caches[l] = (_normal(shp, 1.0, shape.torch_dtype, seed, f"kv/{l}/k", device),
                     _normal(shp, 1.0, shape.torch_dtype, seed, f"kv/{l}/v", device))
    return lens, caches
