"""Meta's checkpoint layout -> the C ABI's config and weights.

"Building llama3 from scratch" reads a model as two files: ``params.json``
(dim, n_layers, n_heads, n_kv_heads, vocab_size, multiple_of,
ffn_dim_multiplier, norm_eps, rope_theta) and ``consolidated.00.pth``, a
torch state dict whose keys name every tensor: ``tok_embeddings.weight``, then
per layer ``layers.{i}.attention.{wq,wk,wv,wo}.weight``,
``layers.{i}.feed_forward.{w1,w3,w2}.weight``,
``layers.{i}.attention_norm.weight`` and ``layers.{i}.ffn_norm.weight``, plus
``norm.weight`` and ``output.weight``; every matrix is [out, in].

This module maps such a pair onto the library's model: the config fields come
from params.json, except the sizes params.json only implies (the FFN hidden
size, from the rows of w1; the vocabulary when given as -1, from the
embedding), and the weights dicts the binding's ``Model`` takes. Fields
params.json may leave out default to multi-head attention (n_kv_heads =
n_heads) and a RoPE base of 10000, as for the Llama-2 shapes. A model without ``output.weight`` reuses the
embedding as its lm_head (tied). Every tensor's shape is checked against the
config before anything reaches the GPU; problems raise ValueError naming the
key. Nothing here computes the model: the weights are only converted to the
model dtype and made contiguous.
"""
from __future__ import annotations

import dataclasses
import json
from typing import Dict, List, Mapping, Optional, Tuple

import torch

LAYER_KEYS = {
    "wq": "layers.{i}.attention.wq.weight",
    "wk": "layers.{i}.attention.wk.weight",
    "wv": "layers.{i}.attention.wv.weight",
    "wo": "layers.{i}.attention.wo.weight",
    "w1": "layers.{i}.feed_forward.w1.weight",
    "w3": "layers.{i}.feed_forward.w3.weight",
    "w2": "layers.{i}.feed_forward.w2.weight",
    "attention_norm": "layers.{i}.attention_norm.weight",
    "ffn_norm": "layers.{i}.ffn_norm.weight",
}
GLOBAL_KEYS = {"tok_embeddings": "tok_embeddings.weight", "norm": "norm.weight", "output": "output.weight"}


@dataclasses.dataclass(frozen=True)
class CheckpointConfig:
    """The model config in the attribute names the binding's make_config reads."""
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
    dtype: str                 # "bf16" or "f32"
    tie_embeddings: bool
    has_embed_and_head: bool = True


def key_order(n_layers: int) -> List[str]:
    """Every key of a checkpoint with n_layers layers: the embedding, then each
    layer's keys in the order the checkpoint lists them, then the final norm and
    the lm_head (their place in the file does not matter to the loader)."""
    keys = [GLOBAL_KEYS["tok_embeddings"]]
    for i in range(n_layers):
        keys += [LAYER_KEYS[k].format(i=i) for k in ("wq", "wk", "wv", "wo", "w1", "w3", "w2",
                                                      "attention_norm", "ffn_norm")]
    return keys + [GLOBAL_KEYS["norm"], GLOBAL_KEYS["output"]]


def read_params(path: str) -> dict:
    with open(path) as f:
        return json.load(f)


def read_state_dict(path: str) -> Dict[str, torch.Tensor]:
    """The consolidated checkpoint as a CPU state dict (tensors only, no code)."""
    return torch.load(path, map_location="cpu", weights_only=True)


def _need(sd: Mapping[str, torch.Tensor], key: str) -> torch.Tensor:
    if key not in sd:
        raise ValueError(f"checkpoint has no {key}")
    return sd[key]


def config_from_checkpoint(params: Mapping, sd: Mapping[str, torch.Tensor], max_seq_len: int,
                           dtype: Optional[str] = None) -> CheckpointConfig:
    """The model config of a params.json dict and its state dict.

    max_seq_len (the KV-cache capacity per sequence) is not in params.json and
    must be given; dtype defaults to the checkpoint's ("bf16" for bf16 tensors,
    else "f32").
    """
    for k in ("dim", "n_layers", "n_heads"):
        if k not in params:
            raise ValueError(f"params.json has no {k}")
    dim, n_layers, n_heads = int(params["dim"]), int(params["n_layers"]), int(params["n_heads"])
    n_kv_heads = int(params.get("n_kv_heads") or n_heads)
    if dim % n_heads or n_heads % n_kv_heads:
        raise ValueError(f"dim {dim}, n_heads {n_heads}, n_kv_heads {n_kv_heads} do not divide")
    emb = _need(sd, GLOBAL_KEYS["tok_embeddings"])
    vocab = int(params.get("vocab_size", -1))
    if vocab <= 0:
        vocab = emb.shape[0]
    w1 = _need(sd, LAYER_KEYS["w1"].format(i=0))
    if dtype is None:
        dtype = "bf16" if emb.dtype == torch.bfloat16 else "f32"
    if dtype not in ("bf16", "f32"):
        raise ValueError(f"dtype must be bf16 or f32, not {dtype}")
    return CheckpointConfig(dim=dim, n_layers=n_layers, n_heads=n_heads, n_kv_heads=n_kv_heads,
                            head_dim=dim // n_heads, ffn_hidden=int(w1.shape[0]), vocab=vocab,
                            max_seq_len=int(max_seq_len), norm_eps=float(params.get("norm_eps", 1e-5)),
                            rope_theta=float(params.get("rope_theta", 10000.0)), dtype=dtype,
                            tie_embeddings=GLOBAL_KEYS["output"] not in sd)


def expected_shapes(cfg: CheckpointConfig) -> Dict[str, Tuple[int, ...]]:
    """[out, in] shape of every key of a checkpoint with this config."""
    D, F, V = cfg.dim, cfg.ffn_hidden, cfg.vocab
    Hd, Hkd = cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim
    per = {"wq": (Hd, D), "wk": (Hkd, D), "wv": (Hkd, D), "wo": (D, Hd), "w1": (F, D), "w3": (F, D),
           "w2": (D, F), "attention_norm": (D,), "ffn_norm": (D,)}
    out = {GLOBAL_KEYS["tok_embeddings"]: (V, D), GLOBAL_KEYS["norm"]: (D,)}
    if not cfg.tie_embeddings:
        out[GLOBAL_KEYS["output"]] = (V, D)
    for i in range(cfg.n_layers):
        for k, shp in per.items():
            out[LAYER_KEYS[k].format(i=i)] = shp
    return out


def split_state_dict(sd: Mapping[str, torch.Tensor], cfg: CheckpointConfig, device="cpu"):
    """(glob, layers) dicts for the binding's Model, every tensor shape-checked,
    converted to the model dtype and contiguous on `device`."""
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32

    def take(key, shape):
        t = _need(sd, key)
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{key} has shape {tuple(t.shape)}, expected {tuple(shape)}")
        return t.to(device=device, dtype=dt).contiguous()

    shapes = expected_shapes(cfg)
    glob = {name: take(key, shapes[key]) for name, key in GLOBAL_KEYS.items() if key in shapes}
    layers = [{k: take(tmpl.format(i=i), shapes[tmpl.format(i=i)]) for k, tmpl in LAYER_KEYS.items()}
              for i in range(cfg.n_layers)]
    return glob, layers


def load_model(params, state_dict, max_seq_len: int, max_batch: int, max_tokens: int = 0, flags: int = 0,
               dtype: Optional[str] = None, stream=None, device="cuda"):
    """A ready model (the binding's Model) from params.json and consolidated.*.pth
    (paths, or an already-read dict and state dict)."""
    from . import Model
    if isinstance(params, str):
        params = read_params(params)
    if isinstance(state_dict, str):
        state_dict = read_state_dict(state_dict)
    cfg = config_from_checkpoint(params, state_dict, max_seq_len, dtype)
    glob, layers = split_state_dict(state_dict, cfg, device=device)
    return Model(cfg, glob, layers, max_batch=max_batch, max_tokens=max_tokens, flags=flags, stream=stream,
                 device=device)
