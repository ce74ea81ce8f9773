"""Plain, slow, fp64 CPU oracle of the Llama-2/3 decoder forward pass.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code with the CUDA path; both take their
inputs from ``seeded_inputs``.

Everything is computed in float64 with no intermediate rounding. bf16 or fp32
weights are widened exactly to float64 when a layer is used. A library matmul
(numpy) serves as the only primitive; there is no blocking, fusion or
reordering beyond what each step's definition states.

Sources (page title, then section), all restated in this module's own words:

* "Building llama3 from scratch": the params.json listing (dim, n_layers,
  n_heads, n_kv_heads, vocab_size, norm_eps, rope_theta), the checkpoint key
  listing, the embedding step (``torch.nn.Embedding``), the RMSNorm code block
  (x * rsqrt(mean(x^2) + eps) * w), the weight-shape printout (wq [4096,4096],
  wk/wv [1024,4096], wo [4096,4096]) and the per-head view of wq
  (``view(n_heads, head_dim, dim)``, q per token = x @ wq_head^T). Its prose says
  RMSNorm normalises the input of every transformer sub-layer (pre-norm).
* "Model Llama 3 yang Diimplementasikan dengan NumPy Murni" (llama3.np):
  "RoPE #1" (cos/sin precomputed from np.outer of positions and frequencies),
  "RoPE #2" (applied to Q and K only; input split into pairs, multiplied by cos
  and sin, summed/subtracted and reshaped back), "KV cache" (K and V cached; Q
  only for the newest token), "GQA", "Scaled Dot-Product Attention",
  "Feed Forward" (three bias-free linears: swish of one, times another, scaled
  back down by the third), "Linear" (only the last position's logits) and
  "Generasi" (prefill phase on the whole prompt, decode phase on the last id).
* "Resumen de una implementación desde cero del modelo LLaMA-3":
  "Implementación de la atención" (scores by dot product, mask of future
  tokens, softmax, weighted sum of values), "Atención multi-head" (concatenate
  heads, output matrix), "Red feed-forward" (SwiGLU; residual sum),
  "Repetición de todas las capas", "Predicción de tokens" (final RMSNorm, logits
  by the output matrix, the highest logit is the next token).
* "LLaMA2" (downcodes): RoPE as a rotation whose q.k product depends only on the
  position offset; GQA/MQA share K/V heads among query heads; the KV cache.

``OracleModel(..., rounding=points)`` is the same computation with the
activations rounded to bf16 (nearest, ties to even) at the named points where a
bf16 implementation can store them (``BF16_POINTS``): "x", each projection input
h * norm weight (the norm's 1/rms scale applied after the product); "q", "k" and
"v" after RoPE (k and v are the KV cache); "o", the attention output; "g", the
SwiGLU output. ``bf16_activations=True`` rounds at all of them. ``BF16_FORCED``
names the points no bf16 tensor-core implementation with a bf16 KV cache can
avoid: the inputs of the four projections (x, o, g: the bf16 operands of the
matrix products) and the cache (k, v). These modes exist to state what a storage
policy alone does to the result at depth; every other value stays exact.

Readings where the pages are silent or garbled (each is also listed in the
design notes): RoPE rotates interleaved adjacent pairs (2i, 2i+1) with angle
p * theta^(-2i/d); the score scale is 1/sqrt(head_dim); masked scores are -inf
before the max-subtracted softmax; query head h reads KV head floor(h / G); w1
is the gated (SiLU) branch, w3 the linear branch, w2 the down projection; argmax
ties go to the lowest index; every sequence's first token is at position 0.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional

import numpy as np
import torch

__all__ = [
    "BF16_POINTS", "BF16_FORCED", "f64", "round_bf16", "rmsnorm", "rope_tables", "rope", "softmax", "silu",
    "attention", "swiglu_ffn", "argmax_first", "OracleModel",
]


BF16_POINTS = frozenset({"x", "q", "k", "v", "o", "g"})
BF16_FORCED = frozenset({"x", "k", "v", "o", "g"})


def f64(t) -> np.ndarray:
    """Exact widening of a torch (bf16/fp32) tensor or numpy array to float64."""
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def round_bf16(x) -> np.ndarray:
    """Round to the nearest value with an 8-bit significand (bf16), ties to even.

    With x = m * 2^e and 0.5 <= |m| < 1, the nearest such value is
    rint(m * 2^8) * 2^(e - 8), where rint rounds halves to even. (bf16 keeps 8
    significant bits, 7 of them stored; subnormals and overflow do not arise for
    the activations this is used on.)
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def rmsnorm(x: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * w.

    "Building llama3 from scratch", RMSNorm code block: the mean of the squares
    along the last dimension, eps added inside the reciprocal square root, then
    the elementwise norm weight.
    """
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


def rope_tables(n_pos: int, head_dim: int, theta: float):
    """cos, sin of shape [n_pos, head_dim/2]: angle(p, i) = p * theta^(-2i/head_dim).

    llama3.np page, "RoPE #1": the table is the outer product of the positions
    and the per-pair frequencies, then cos and sin of it.
    """
    i = np.arange(head_dim // 2, dtype=np.float64)
    freqs = theta ** (-2.0 * i / head_dim)
    ang = np.outer(np.arange(n_pos, dtype=np.float64), freqs)
    return np.cos(ang), np.sin(ang)


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate pairs (x[2i], x[2i+1]) of the last axis by angle pos * theta^(-2i/d).

    x: [..., n_tok, n_heads, d]; pos: [n_tok] absolute positions.
    llama3.np page, "RoPE #2": the input is split into pairs, multiplied by cos
    and sin, summed and subtracted, and reshaped back. Reading: interleaved
    adjacent pairs.
    """
    d = x.shape[-1]
    cos_t, sin_t = rope_tables(int(np.max(pos)) + 1 if len(pos) else 1, d, theta)
    c = cos_t[pos][:, None, :]          # [n_tok, 1, d/2]
    s = sin_t[pos][:, None, :]
    xp = x.reshape(*x.shape[:-1], d // 2, 2)
    x0, x1 = xp[..., 0], xp[..., 1]
    out = np.empty_like(xp)
    out[..., 0] = x0 * c - x1 * s
    out[..., 1] = x0 * s + x1 * c
    return out.reshape(x.shape)


def softmax(s: np.ndarray) -> np.ndarray:
    """Row softmax over the last axis, max-subtracted; -inf entries get weight 0."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def silu(z: np.ndarray) -> np.ndarray:
    """Swish / SiLU: z * sigmoid(z)."""
    return z / (1.0 + np.exp(-z))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_pos: np.ndarray,
              k_pos: np.ndarray) -> np.ndarray:
    """Causal grouped-query attention for one sequence.

    q: [Tq, H, d]; k, v: [Tk, Hk, d]; q_pos: [Tq]; k_pos: [Tk] absolute positions.
    Returns [Tq, H*d] with heads concatenated in head order.

    Scores are q.k / sqrt(d) ("Scaled Dot-Product Attention"); a key at a
    position after the query's is masked to -inf before the softmax
    ("Implementación de la atención": scores of future tokens are masked); the
    output is the softmax-weighted sum of values, then the
    heads are concatenated ("Atención multi-head"). Query head h uses KV head
    floor(h / (H / Hk)) (GQA, "GQA(Grouped-Query Attention)").
    """
    Tq, H, d = q.shape
    Hk = k.shape[1]
    G = H // Hk
    out = np.empty((Tq, H, d))
    future = k_pos[None, :] > q_pos[:, None]            # [Tq, Tk]
    for h in range(H):
        g = h // G
        s = (q[:, h, :] @ k[:, g, :].T) / math.sqrt(d)
        s = np.where(future, -np.inf, s)
        out[:, h, :] = softmax(s) @ v[:, g, :]
    return out.reshape(Tq, H * d)


def swiglu_ffn(x: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """w2( silu(x w1^T) * (x w3^T) ): the bias-free three-linear feed-forward."""
    return (silu(x @ w1.T) * (x @ w3.T)) @ w2.T


def argmax_first(logits: np.ndarray) -> np.ndarray:
    """Index of the highest logit along the last axis; ties go to the lowest index."""
    return np.argmax(logits, axis=-1)


def top2_margin(logits: np.ndarray) -> np.ndarray:
    """Highest minus second-highest logit along the last axis."""
    part = np.partition(logits, -2, axis=-1)
    return part[..., -1] - part[..., -2]


class OracleModel:
    """The whole decoder in fp64, with its own KV cache.

    ``layers`` is a list of per-layer weight dicts (torch or numpy; keys wq, wk,
    wv, wo, w1, w3, w2, attention_norm, ffn_norm) or a callable layer -> dict
    (so a large model can be regenerated layer by layer). ``glob`` holds
    tok_embeddings, norm and output (absent when tied or for layer-only shapes).

    The cache holds post-RoPE keys and values per layer:
    K[l][b] has shape [n_pos, Hk, d].
    """

    def __init__(self, shape, glob: Dict, layers, batch: int, keep_f64_layers: bool = True,
                 bf16_activations: bool = False, rounding=None):
        self.s = shape
        if rounding is None:
            rounding = BF16_POINTS if bf16_activations else frozenset()
        assert set(rounding) <= BF16_POINTS, f"unknown rounding points {set(rounding) - BF16_POINTS}"
        self.rounding = frozenset(rounding)
        self.glob = glob
        self._layers = layers
        self._cache64: Dict[int, Dict[str, np.ndarray]] = {}
        self.keep = keep_f64_layers
        self.B = batch
        L = shape.n_layers
        self.K = [[np.zeros((0, shape.n_kv_heads, shape.head_dim)) for _ in range(batch)] for _ in range(L)]
        self.V = [[np.zeros((0, shape.n_kv_heads, shape.head_dim)) for _ in range(batch)] for _ in range(L)]
        self.lens = np.zeros(batch, dtype=np.int64)
        self._emb = None
        self._out = None

    # ---- weights -------------------------------------------------------
    def layer(self, l: int) -> Dict[str, np.ndarray]:
        if l in self._cache64:
            return self._cache64[l]
        src = self._layers(l) if callable(self._layers) else self._layers[l]
        w = {k: f64(v) for k, v in src.items()}
        if self.keep:
            self._cache64[l] = w
        return w

    def embedding(self) -> np.ndarray:
        if self._emb is None:
            self._emb = f64(self.glob["tok_embeddings"])
        return self._emb

    def lm_head(self) -> np.ndarray:
        if self._out is None:
            self._out = self.embedding() if self.s.tie_embeddings else f64(self.glob["output"])
        return self._out

    # ---- cache ---------------------------------------------------------
    def set_cache(self, l: int, b: int, k: np.ndarray, v: np.ndarray):
        """Install a pre-filled cache (post-RoPE keys, values) of shape [n, Hk, d]."""
        self.K[l][b] = np.array(k, dtype=np.float64)
        self.V[l][b] = np.array(v, dtype=np.float64)
        self.lens[b] = k.shape[0]

    # ---- one decoder layer ---------------------------------------------
    def layer_forward(self, l: int, h: np.ndarray, pos0: np.ndarray) -> np.ndarray:
        """h: [B, T, D] residual stream -> [B, T, D]; appends T positions to the cache.

        Pre-norm residual layer ("Building llama3 from scratch": RMSNorm on the
        input of each sub-layer; "Resumen ...": attention, then feed-forward,
        each added back): h + Attn(RMSNorm(h)), then + FFN(RMSNorm(.)).
        """
        s = self.s
        w = self.layer(l)
        B, T, D = h.shape
        H, Hk, d = s.n_heads, s.n_kv_heads, s.head_dim
        r = self._round
        x = self._norm_in(h, w["attention_norm"])
        out = np.empty((B, T, H * d))
        for b in range(B):
            pos = pos0[b] + np.arange(T)
            q = (x[b] @ w["wq"].T).reshape(T, H, d)
            k = (x[b] @ w["wk"].T).reshape(T, Hk, d)
            v = r((x[b] @ w["wv"].T).reshape(T, Hk, d), "v")
            q = r(rope(q, pos, s.rope_theta), "q")
            k = r(rope(k, pos, s.rope_theta), "k")
            assert self.K[l][b].shape[0] == pos0[b], "cache length and position disagree"
            self.K[l][b] = np.concatenate([self.K[l][b], k], axis=0)
            self.V[l][b] = np.concatenate([self.V[l][b], v], axis=0)
            kpos = np.arange(self.K[l][b].shape[0])
            out[b] = r(attention(q, self.K[l][b], self.V[l][b], pos, kpos), "o")
        h = h + out @ w["wo"].T
        x = self._norm_in(h, w["ffn_norm"])
        return h + r(silu(x @ w["w1"].T) * (x @ w["w3"].T), "g") @ w["w2"].T

    def _round(self, a: np.ndarray, point: str) -> np.ndarray:
        return round_bf16(a) if point in self.rounding else a

    def _norm_in(self, h: np.ndarray, wn: np.ndarray) -> np.ndarray:
        """RMSNorm(h) * wn; when "x" is rounded, h * wn is stored in bf16 and the
        1/rms scale is applied to it afterwards (the same value in exact arithmetic)."""
        if "x" not in self.rounding:
            return rmsnorm(h, wn, self.s.norm_eps)
        rinv = 1.0 / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + self.s.norm_eps)
        return round_bf16(h * wn) * rinv

    # ---- whole passes --------------------------------------------------
    def _run_layers(self, h: np.ndarray, taps: Optional[List[np.ndarray]]):
        pos0 = self.lens.copy()
        for l in range(self.s.n_layers):
            h = self.layer_forward(l, h, pos0)
            if taps is not None:
                taps.append(h.copy())
            if not self.keep:
                self._cache64.pop(l, None)
        self.lens = pos0 + h.shape[1]
        return h

    def logits_last(self, h: np.ndarray) -> np.ndarray:
        """Final RMSNorm of the last position, then logits = x @ output^T ("Linear")."""
        x = self._norm_in(h[:, -1, :], f64(self.glob["norm"]))
        return x @ self.lm_head().T

    def prefill(self, tokens, taps: Optional[List[np.ndarray]] = None):
        """Prefill phase: tokens [B, T] -> (next token ids [B], last-position logits [B, V])."""
        tok = np.asarray(tokens, dtype=np.int64)
        h = self.embedding()[tok]                 # embedding lookup, [B, T, D]
        h = self._run_layers(h, taps)
        logits = self.logits_last(h)
        return argmax_first(logits), logits

    def decode(self, tok, taps: Optional[List[np.ndarray]] = None):
        """Decode phase: one new token per sequence, [B] -> (next ids [B], logits [B, V])."""
        return self.prefill(np.asarray(tok, dtype=np.int64).reshape(-1, 1), taps)

    def forward_hidden(self, h_in, taps: Optional[List[np.ndarray]] = None) -> np.ndarray:
        """Layer stack on given hidden states [B, T, D] (no embedding, norm or lm_head)."""
        return self._run_layers(f64(h_in), taps)

    def generate(self, prompt, steps: int):
        """Greedy generation: prefill, then ``steps`` decode steps feeding back the argmax.

        Returns (list of emitted ids per step [steps+1][B], list of logits).
        """
        nxt, lg = self.prefill(prompt)
        toks, logits = [nxt], [lg]
        for _ in range(steps):
            nxt, lg = self.decode(nxt)
            toks.append(nxt)
            logits.append(lg)
        return toks, logits
