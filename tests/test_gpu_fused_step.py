"""The fused decode-step kernel (the whole bf16 model in one launch) against the
fp64 oracle and against the layer-by-layer decode path (GPU).

Models built with LLM_FLAG_FUSED_DECODE (and without per-layer taps) run each
bf16 decode step as the fused kernel, so these tests check what it hands back: the logits (relative L2 against the oracle's,
the bf16 bar), the greedy tokens (same argmax wherever the oracle's top-2 margin
exceeds the bar), the hidden states of a bare layer stack, and the cache lengths.
"""
import numpy as np
import pytest
import torch

import llama_decoder_forward_fwd_b200 as L
import seeded_inputs as S
from model_util import BF16_REL_L2, build_pair, check_argmax, install_prefilled_cache, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
FUSED = L.LLM_FLAG_FUSED_DECODE


def _tokens_case(shape, seed, B, T, steps, flags=0):
    model, orc = build_pair(shape, seed, batch=B, max_tokens=B * T, flags=flags | FUSED, taps=False)
    prompt = S.make_tokens(seed, B, T, shape.vocab)
    nxt = torch.empty(B, dtype=torch.int32, device=DEV)
    logits = torch.empty(B, shape.vocab, device=DEV)
    L.llm_prefill(model.h, prompt.to(DEV), nxt, logits)
    o_next, o_logits = orc.prefill(prompt.numpy())
    checked = check_argmax(nxt.cpu().numpy(), o_logits)
    worst = 0.0
    for step in range(steps):
        tok = torch.as_tensor(o_next, dtype=torch.int32).to(DEV)   # oracle's token into both sides
        L.llm_decode_step(model.h, tok, nxt, logits)
        L.llm_synchronize(model.h)
        o_next, o_logits = orc.decode(o_next)
        r = rel_l2(logits.cpu().numpy(), o_logits)
        assert r <= BF16_REL_L2, f"decode {step}: logits rel L2 {r:.3e}"
        worst = max(worst, r)
        checked += check_argmax(nxt.cpu().numpy(), o_logits)
    assert L.llm_kv_cache_get_lens(model.h, B) == [T + steps] * B
    assert checked >= (steps + 1) * B // 2, "too few argmax checks above the margin bar"
    print(f"worst logits rel L2 {worst:.3e}; argmax checked {checked}")
    model.free()


@pytest.mark.parametrize("flags", [0, L.LLM_FLAG_CUDA_GRAPH])
def test_fused_llama3_shape_two_layers(lib, flags):
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=512)
    _tokens_case(shape, seed=77, B=2, T=200, steps=6, flags=flags)


def test_fused_llama2_mha_shape(lib):
    """One query head per KV head (the smallest attention group)."""
    shape = S.WORKLOADS["llama2-7b-mha-bf16-b8-p1024-g256"].shape.replace(n_layers=2, max_seq_len=256)
    _tokens_case(shape, seed=79, B=3, T=77, steps=4, flags=L.LLM_FLAG_CUDA_GRAPH)


def test_fused_batch16_over_prefilled_ragged_caches(lib):
    """Llama-3-8B shape, batch 16 (the 16-column MMA variant), ragged N(0,1) caches."""
    w = S.WORKLOADS["llama3-8b-bf16-b16-kv4k8k-g128"]
    lo, hi = 40, 300
    shape = w.shape.replace(n_layers=2, max_seq_len=hi + 16)
    B = w.batch
    model, orc = build_pair(shape, w.seed, batch=B, max_tokens=B, flags=FUSED, taps=False)
    lens, caches = S.make_kv_prefill(shape, w.seed, B, lo, hi)
    install_prefilled_cache(model, orc, lens.numpy(), caches)
    tok = S.make_tokens(w.seed, B, 1, shape.vocab, tag="decode0")[:, 0].numpy()
    nxt = torch.empty(B, dtype=torch.int32, device=DEV)
    logits = torch.empty(B, shape.vocab, device=DEV)
    checked = 0
    for step in range(4):
        L.llm_decode_step(model.h, torch.as_tensor(tok, dtype=torch.int32).to(DEV), nxt, logits)
        L.llm_synchronize(model.h)
        tok, o_logits = orc.decode(tok)
        assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
        checked += check_argmax(nxt.cpu().numpy(), o_logits)
    assert L.llm_kv_cache_get_lens(model.h, B) == [int(x) + 4 for x in lens]
    assert checked >= 4 * B // 2
    model.free()


def test_fused_layer_stack_hidden_decode(lib):
    """One Llama-3-8B-shaped layer without embedding/head: 512 prompt hidden states
    through the prefill path, then 64 fused decode steps on hidden states."""
    w = S.WORKLOADS["llama3-8b-1layer-bf16-b1-h512-d64"]
    s = w.shape
    model, orc = build_pair(s, w.seed, batch=1, max_tokens=w.prompt_len, flags=FUSED, taps=False)
    h_all = S.make_hidden(w.seed, 1, w.prompt_len + w.decode_steps, s.dim)
    out = torch.empty(1, w.prompt_len, s.dim, device=DEV)
    L.llm_prefill_hidden(model.h, h_all[:, :w.prompt_len].contiguous().to(DEV), out)
    orc.forward_hidden(h_all[:, :w.prompt_len].contiguous())
    o1 = torch.empty(1, s.dim, device=DEV)
    worst = 0.0
    for step in range(w.decode_steps):
        x = h_all[:, w.prompt_len + step].contiguous()
        L.llm_decode_step_hidden(model.h, x.to(DEV), o1)
        L.llm_synchronize(model.h)
        ref = orc.forward_hidden(x.reshape(1, 1, s.dim))
        r = rel_l2(o1.cpu().numpy(), ref.reshape(1, s.dim))
        assert r <= BF16_REL_L2, f"decode step {step}: {r}"
        worst = max(worst, r)
    assert L.llm_kv_cache_get_lens(model.h, 1) == [w.prompt_len + w.decode_steps]
    print(f"worst rel L2 {worst:.3e}")
    model.free()


@pytest.mark.parametrize("B", [1, 5, 12])
def test_fused_agrees_with_layerwise_decode(lib, B):
    """Same weights and tokens through both decode paths. The paths differ in
    rounding only: the projections split their k sums differently, and the fused
    attention rounds the softmax probabilities to bf16 for its tensor-core P V
    (as the prefill attention does) where the layer-by-layer split-KV kernel keeps
    them in fp32. Each path is within ~1e-2 of the fp64 oracle (the bf16 bar is
    2e-2), so the two agree to the sum of their errors: 1.5e-2 relative L2."""
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=3, max_seq_len=160)
    glob, layers = S.make_weights(shape, 31)
    prompt = S.make_tokens(31, B, 33, shape.vocab).to(DEV)
    feed = S.make_tokens(32, B, 6, shape.vocab).to(DEV)
    out = []
    for flags in (L.LLM_FLAG_CUDA_GRAPH | L.LLM_FLAG_FUSED_DECODE, L.LLM_FLAG_CUDA_GRAPH):
        m = L.Model(shape, glob, layers, max_batch=B, max_tokens=B * 33, flags=flags)
        nxt = torch.empty(B, dtype=torch.int32, device=DEV)
        lg = torch.empty(B, shape.vocab, device=DEV)
        L.llm_prefill(m.h, prompt, nxt, lg)
        seq = []
        for i in range(6):
            L.llm_decode_step(m.h, feed[:, i].contiguous(), nxt, lg)
            L.llm_synchronize(m.h)
            seq.append((nxt.cpu().clone(), lg.cpu().numpy().copy()))
        out.append(seq)
        m.free()
    for i, ((ta, la), (tb, lb)) in enumerate(zip(*out)):
        assert rel_l2(la, lb) <= 1.5e-2, f"step {i}: {rel_l2(la, lb):.3e}"
        srt = np.sort(lb, axis=1)
        clear = srt[:, -1] - srt[:, -2] > 0.05
        assert torch.equal(ta[clear], tb[clear])


def test_fused_step_is_deterministic(lib):
    """Two models on the same GPU replay bit-identical steps."""
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=96)
    glob, layers = S.make_weights(shape, 8)
    prompt = S.make_tokens(8, 3, 20, shape.vocab).to(DEV)
    res = []
    for flags in (FUSED, FUSED | L.LLM_FLAG_CUDA_GRAPH):
        m = L.Model(shape, glob, layers, max_batch=3, max_tokens=60, flags=flags)
        nxt = torch.empty(3, dtype=torch.int32, device=DEV)
        lg = torch.empty(3, shape.vocab, device=DEV)
        L.llm_prefill(m.h, prompt, nxt, lg)
        seq = []
        for _ in range(4):
            L.llm_decode_step(m.h, nxt.clone(), nxt, lg)
            L.llm_synchronize(m.h)
            seq.append((nxt.cpu().clone(), lg.cpu().clone()))
        res.append(seq)
        m.free()
    for (a, la), (b, lb) in zip(*res):
        assert torch.equal(a, b) and torch.equal(la, lb)


def test_fused_small_model_fewer_units_than_sms(lib):
    """A 512-wide model with a 1000-token vocabulary: every projection has fewer
    weight units than the GPU has SMs, and the last lm_head tile is ragged."""
    shape = S.ModelShape(dim=512, n_layers=2, n_heads=4, n_kv_heads=2, head_dim=128, ffn_hidden=1024,
                         vocab=1000, max_seq_len=160, norm_eps=1e-5, rope_theta=500000.0, dtype="bf16",
                         tie_embeddings=False)
    _tokens_case(shape, seed=2024, B=2, T=130, steps=5, flags=L.LLM_FLAG_CUDA_GRAPH)


def test_fused_flag_runs_one_launch_per_step(lib):
    """With LLM_FLAG_FUSED_DECODE each decode step is one fused launch (kernel
    timing records it as "step"); without it, one launch per projection."""
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=64)
    glob, layers = S.make_weights(shape, 3)
    prompt = S.make_tokens(3, 1, 8, shape.vocab).to(DEV)
    for flags, fused in ((FUSED, True), (0, False)):
        m = L.Model(shape, glob, layers, max_batch=1, max_tokens=8, flags=flags | L.LLM_FLAG_KERNEL_TIMING)
        nxt = torch.empty(1, dtype=torch.int32, device=DEV)
        L.llm_prefill(m.h, prompt, nxt)
        L.llm_kernel_times(m.h, reset=True)
        for _ in range(3):
            L.llm_decode_step(m.h, nxt.clone(), nxt)
        kt = L.llm_kernel_times(m.h, reset=True)
        if fused:
            assert kt["step"][1] == 3 and kt["w13"][1] == 0
        else:
            assert kt["step"][1] == 0 and kt["w13"][1] == 3 * shape.n_layers
        m.free()
