"""Small fixed workloads for profiling single kernels with ncu on one GPU.

    python -m llama_decoder_forward_fwd_b200.profile_case decode-layer
        one Llama-3-8B-shaped layer (436 MB of bf16 weights, larger than L2):
        a 64-token prefill on hidden states, then 4 decode steps against a
        2048-position cache
        (kernels per decode step: QKV GEMV, split-KV attention, wo GEMV,
        w1/w3 GEMV, w2 GEMV, hidden-state output)
    python -m llama_decoder_forward_fwd_b200.profile_case prefill-layer
        the same layer: a 2048-token prefill (tcgen05 GEMMs, flash attention)
    python -m llama_decoder_forward_fwd_b200.profile_case decode-head
        the lm_head + argmax of the Llama-3-8B shape on one token (1.05 GB)

A trailing --fused runs the decode steps as the fused single-launch kernel.

Weights are seeded random (the bench's distributions); nothing is checked here.
"""
import sys

import torch

import llama_decoder_forward_fwd_b200 as L


FLAGS = L.LLM_FLAG_FUSED_DECODE if "--fused" in sys.argv[2:] else 0


def _layer_model(prefill_tokens, S_max=4096, has_head=False, vocab=128256):
    import seeded_inputs as S
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(
        n_layers=1, has_embed_and_head=has_head, max_seq_len=S_max, vocab=vocab)
    glob, layers = S.make_weights(shape, 1234, device="cuda")
    return shape, L.Model(shape, glob, layers, max_batch=1, max_tokens=max(prefill_tokens, 1), flags=FLAGS)


def decode_layer():
    shape, m = _layer_model(64)
    h = torch.randn(1, 64, shape.dim, device="cuda")
    out = torch.empty_like(h)
    L.llm_prefill_hidden(m.h, h, out)
    # continue as if 2048 positions were cached (N(0,1) keys and values)
    kc, vc = m.kv_cache_tensors()
    kc[0, 0, :, :2048].normal_()
    vc[0, 0, :, :2048].normal_()
    torch.cuda.synchronize()
    L.llm_kv_cache_set_lens(m.h, [2048])
    x = torch.randn(1, shape.dim, device="cuda")
    o1 = torch.empty_like(x)
    for _ in range(4):
        L.llm_decode_step_hidden(m.h, x, o1)
    L.llm_synchronize(m.h)


def prefill_layer():
    shape, m = _layer_model(2048)
    h = torch.randn(1, 2048, shape.dim, device="cuda")
    out = torch.empty_like(h)
    L.llm_prefill_hidden(m.h, h, out)
    L.llm_synchronize(m.h)


def decode_head():
    shape, m = _layer_model(1, has_head=True)
    tok = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    L.llm_prefill(m.h, tok, nxt)
    L.llm_synchronize(m.h)


if __name__ == "__main__":
    {"decode-layer": decode_layer, "prefill-layer": prefill_layer, "decode-head": decode_head}[sys.argv[1]]()
    print("done")
