"""Helpers shared by the model-level GPU parity tests (not a test module)."""
import numpy as np
import torch

import llama_decoder_forward_fwd_b200 as L
import oracle as O
import seeded_inputs as S

# Acceptance bars: fp32 model -> identical greedy tokens, logits within 1e-4
# relative; bf16 models -> per-layer hidden states within 2e-2 relative L2 and
# the same argmax wherever the oracle's top-2 logit margin exceeds 0.05.
F32_LOGIT_REL = 1e-4
BF16_REL_L2 = 2e-2
ARGMAX_MARGIN = 0.05


def rel_l2(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def build_pair(shape, seed, batch, max_tokens=0, flags=0, taps=True):
    """GPU model and oracle on the same weights; with taps the GPU model keeps every
    layer's output (llm_debug_tap)."""
    glob, layers = S.make_weights(shape, seed)
    model = L.Model(shape, glob, layers, max_batch=batch, max_tokens=max_tokens,
                    flags=flags | (L.LLM_FLAG_DEBUG_TAPS if taps else 0))
    orc = O.OracleModel(shape, glob, layers, batch)
    return model, orc


def gpu_taps(model, n_tokens):
    D = model.shape.dim
    out = []
    buf = torch.empty(n_tokens * D, dtype=torch.float32, device="cuda")
    for l in range(model.shape.n_layers):
        L.llm_debug_tap(model.h, l, buf)
        L.llm_synchronize(model.h)
        out.append(buf.cpu().numpy().reshape(n_tokens, D).copy())
    return out


def check_taps(g_taps, o_taps, tol=BF16_REL_L2, what=""):
    worst = 0.0
    for l, (g, o) in enumerate(zip(g_taps, o_taps)):
        o = o.reshape(g.shape)
        r = rel_l2(g, o)
        worst = max(worst, r)
        assert r <= tol, f"{what} layer {l}: rel L2 {r:.3e} > {tol}"
    return worst


def check_argmax(gpu_next, orc_logits):
    """Same argmax where the oracle's top-2 margin exceeds the bar; returns #checked."""
    margin = O.top2_margin(orc_logits)
    ref = O.argmax_first(orc_logits)
    n = 0
    for b in range(len(ref)):
        if margin[b] > ARGMAX_MARGIN:
            assert int(gpu_next[b]) == int(ref[b]), f"seq {b}: gpu {int(gpu_next[b])} oracle {int(ref[b])} margin {margin[b]:.3f}"
            n += 1
    return n


def install_prefilled_cache(model, orc, lens, caches):
    """Copy ragged N(0,1) caches into the GPU model's cache and into the oracle's."""
    kc, vc = model.kv_cache_tensors()
    B = len(lens)
    for l, (K, V) in caches.items():
        kc[l, :B, :, :K.shape[2], :] = K.to("cuda")
        vc[l, :B, :, :V.shape[2], :] = V.to("cuda")
        for b in range(B):
            n = int(lens[b])
            orc.set_cache(l, b, O.f64(K[b, :, :n, :]).transpose(1, 0, 2), O.f64(V[b, :, :n, :]).transpose(1, 0, 2))
    torch.cuda.synchronize()
    L.llm_kv_cache_set_lens(model.h, [int(x) for x in lens])
