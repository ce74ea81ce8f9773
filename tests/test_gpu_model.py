"""Whole-model parity: the CUDA path through the C ABI against the fp64 oracle (GPU).

Every workload shape is covered (the tiny fp32 model, one Llama-3-8B layer on
hidden states, the Llama-3-8B shape at batch 1 and batch 16 over ragged caches,
long-context decode at 8064+ positions, the Llama-2-7B MHA shape), plus
multi-query variants; the Llama-3-8B and Llama-2-7B shapes run with 2 layers
here (the layer is identical at any depth; full-depth runs are in
test_gpu_fullsize.py). Decode steps feed both sides the oracle's own greedy
token, so no value computed on the GPU is ever an oracle input.
"""
import numpy as np
import pytest
import torch

import llama_decoder_forward_fwd_b200 as L
import seeded_inputs as S
from model_util import (BF16_REL_L2, F32_LOGIT_REL, build_pair, check_argmax, check_taps,
                        gpu_taps, install_prefilled_cache, rel_l2)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("flags", [0, L.LLM_FLAG_CUDA_GRAPH])
def test_tiny_f32_greedy_stream_and_logits(lib, flags):
    """fp32 tiny model: the same 50-token greedy stream and logits within 1e-4."""
    w = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"]
    s = w.shape
    model, orc = build_pair(s, w.seed, batch=1, max_tokens=w.prompt_len, flags=flags)
    prompt = S.make_tokens(w.seed, 1, w.prompt_len, s.vocab)
    nxt = torch.empty(1, dtype=torch.int32, device=DEV)
    logits = torch.empty(1, s.vocab, device=DEV)
    L.llm_prefill(model.h, prompt.to(DEV), nxt, logits)
    L.llm_synchronize(model.h)
    o_taps = []
    o_next, o_logits = orc.prefill(prompt.numpy(), o_taps)
    check_taps(gpu_taps(model, w.prompt_len), o_taps, tol=1e-5, what="prefill")
    gpu_stream, orc_stream = [int(nxt[0])], [int(o_next[0])]
    for step in range(w.decode_steps + 1):
        g = logits.cpu().numpy()
        err = np.abs(g - o_logits).max() / np.abs(o_logits).max()
        assert err <= F32_LOGIT_REL, f"step {step}: logits rel err {err:.2e}"
        assert gpu_stream[-1] == orc_stream[-1], f"step {step}: token {gpu_stream[-1]} vs {orc_stream[-1]}"
        if step == w.decode_steps:
            break
        cur = nxt.clone()
        L.llm_decode_step(model.h, cur, nxt, logits)     # the GPU feeds itself its own token
        L.llm_synchronize(model.h)
        o_next, o_logits = orc.decode(o_next)
        gpu_stream.append(int(nxt[0]))
        orc_stream.append(int(o_next[0]))
    assert gpu_stream == orc_stream
    assert L.llm_kv_cache_get_lens(model.h, 1) == [w.prompt_len + w.decode_steps]
    model.free()


def test_llama3_layer_hidden_prefill_and_decode(lib):
    """One Llama-3-8B-shaped layer: 512 hidden states, then 64 cached decode steps."""
    w = S.WORKLOADS["llama3-8b-1layer-bf16-b1-h512-d64"]
    s = w.shape
    model, orc = build_pair(s, w.seed, batch=1, max_tokens=w.prompt_len)
    h_all = S.make_hidden(w.seed, 1, w.prompt_len + w.decode_steps, s.dim)
    h_in = h_all[:, :w.prompt_len].contiguous()
    out = torch.empty(1, w.prompt_len, s.dim, device=DEV)
    L.llm_prefill_hidden(model.h, h_in.to(DEV), out)
    L.llm_synchronize(model.h)
    ref = orc.forward_hidden(h_in)
    r = rel_l2(out.cpu().numpy(), ref)
    assert r <= BF16_REL_L2, r
    worst = r
    o1 = torch.empty(1, s.dim, device=DEV)
    for step in range(w.decode_steps):
        x = h_all[:, w.prompt_len + step].contiguous()
        L.llm_decode_step_hidden(model.h, x.to(DEV), o1)
        L.llm_synchronize(model.h)
        ref = orc.forward_hidden(x.reshape(1, 1, s.dim))
        r = rel_l2(o1.cpu().numpy(), ref.reshape(1, s.dim))
        assert r <= BF16_REL_L2, f"decode step {step}: {r}"
        worst = max(worst, r)
    print(f"worst rel L2 {worst:.3e}")
    model.free()


def _run_tokens_case(shape, seed, B, T, steps, flags=0):
    model, orc = build_pair(shape, seed, batch=B, max_tokens=B * T, flags=flags)
    prompt = S.make_tokens(seed, B, T, shape.vocab)
    nxt = torch.empty(B, dtype=torch.int32, device=DEV)
    logits = torch.empty(B, shape.vocab, device=DEV)
    L.llm_prefill(model.h, prompt.to(DEV), nxt, logits)
    L.llm_synchronize(model.h)
    o_taps = []
    o_next, o_logits = orc.prefill(prompt.numpy(), o_taps)
    worst = check_taps(gpu_taps(model, B * T), [t.reshape(B * T, -1) for t in o_taps], what="prefill")
    checked = check_argmax(nxt.cpu().numpy(), o_logits)
    assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
    for step in range(steps):
        tok = torch.as_tensor(o_next, dtype=torch.int32).to(DEV)   # oracle's token into both sides
        L.llm_decode_step(model.h, tok, nxt, logits)
        L.llm_synchronize(model.h)
        o_taps = []
        o_next, o_logits = orc.decode(o_next, o_taps)
        worst = max(worst, check_taps(gpu_taps(model, B), [t.reshape(B, -1) for t in o_taps], what=f"decode {step}"))
        checked += check_argmax(nxt.cpu().numpy(), o_logits)
        assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
    assert checked >= (steps + 1) * B // 2, "too few argmax checks above the margin bar"
    print(f"worst per-layer rel L2 {worst:.3e}; argmax checked {checked}")
    model.free()


@pytest.mark.parametrize("flags", [0, L.LLM_FLAG_CUDA_GRAPH])
def test_llama3_shape_two_layers_ragged_prefill_then_decode(lib, flags):
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=512)
    _run_tokens_case(shape, seed=77, B=2, T=200, steps=6, flags=flags)


def test_llama3_shape_small_prompt_uses_decode_kernels(lib):
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=64)
    _run_tokens_case(shape, seed=78, B=3, T=5, steps=3)


def test_llama2_mha_shape_two_layers(lib):
    shape = S.WORKLOADS["llama2-7b-mha-bf16-b8-p1024-g256"].shape.replace(n_layers=2, max_seq_len=256)
    _run_tokens_case(shape, seed=79, B=3, T=77, steps=4)


def test_multi_query_llama3_layer_shape_two_layers(lib):
    """One KV head for all 32 query heads (MQA, G = 32): the prefill runs the flash
    kernel with 32 heads per KV head, decode splits each token's heads into two
    16-row work items."""
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, n_kv_heads=1, max_seq_len=256)
    _run_tokens_case(shape, seed=80, B=2, T=40, steps=4)


def test_multi_query_f32_greedy_stream_and_logits(lib):
    """fp32 MQA model (32 query heads of 16 dims, one KV head): the decode kernel
    also runs the prefill, with (token, head) rows chunked 16 at a time; the same
    greedy stream as the oracle and logits within 1e-4."""
    s = S.ModelShape(dim=512, n_layers=2, n_heads=32, n_kv_heads=1, head_dim=16, ffn_hidden=1024, vocab=512,
                     max_seq_len=64, norm_eps=1e-5, rope_theta=10000.0, dtype="f32", tie_embeddings=False)
    T, steps = 9, 12
    model, orc = build_pair(s, 81, batch=1, max_tokens=T)
    prompt = S.make_tokens(81, 1, T, s.vocab)
    nxt = torch.empty(1, dtype=torch.int32, device=DEV)
    logits = torch.empty(1, s.vocab, device=DEV)
    L.llm_prefill(model.h, prompt.to(DEV), nxt, logits)
    L.llm_synchronize(model.h)
    o_taps = []
    o_next, o_logits = orc.prefill(prompt.numpy(), o_taps)
    check_taps(gpu_taps(model, T), o_taps, tol=1e-5, what="prefill")
    for step in range(steps + 1):
        g = logits.cpu().numpy()
        err = np.abs(g - o_logits).max() / np.abs(o_logits).max()
        assert err <= F32_LOGIT_REL, f"step {step}: logits rel err {err:.2e}"
        assert int(nxt[0]) == int(o_next[0]), f"step {step}: token {int(nxt[0])} vs {int(o_next[0])}"
        if step == steps:
            break
        cur = nxt.clone()
        L.llm_decode_step(model.h, cur, nxt, logits)
        L.llm_synchronize(model.h)
        o_next, o_logits = orc.decode(o_next)
    model.free()


def test_batched_decode_over_prefilled_ragged_caches(lib):
    """Llama-3-8B shape, batch 16, caches pre-filled with N(0,1) to ragged lengths."""
    w = S.WORKLOADS["llama3-8b-bf16-b16-kv4k8k-g128"]
    lo, hi = 40, 300   # ragged lengths, shortened so the oracle stays fast
    shape = w.shape.replace(n_layers=2, max_seq_len=hi + 16)
    B = w.batch
    model, orc = build_pair(shape, w.seed, batch=B, max_tokens=B)
    lens, caches = S.make_kv_prefill(shape, w.seed, B, lo, hi)
    install_prefilled_cache(model, orc, lens.numpy(), caches)
    tok = S.make_tokens(w.seed, B, 1, shape.vocab, tag="decode0")[:, 0].numpy()
    nxt = torch.empty(B, dtype=torch.int32, device=DEV)
    logits = torch.empty(B, shape.vocab, device=DEV)
    checked = 0
    for step in range(4):
        L.llm_decode_step(model.h, torch.as_tensor(tok, dtype=torch.int32).to(DEV), nxt, logits)
        L.llm_synchronize(model.h)
        o_taps = []
        tok, o_logits = orc.decode(tok, o_taps)
        check_taps(gpu_taps(model, B), [t.reshape(B, -1) for t in o_taps], what=f"step {step}")
        checked += check_argmax(nxt.cpu().numpy(), o_logits)
    assert L.llm_kv_cache_get_lens(model.h, B) == [int(x) + 4 for x in lens]
    assert checked >= 4 * B // 2
    model.free()


def test_batched_decode_at_the_workload_cache_lengths(lib):
    """The batched-decode workload at its own sizes (two Llama-3-8B layers): 16
    sequences whose caches hold 4096-8192 N(0,1) positions, decoded through the
    CUDA graph; per-layer hidden states, logits and argmax against the oracle
    (which feeds its own tokens to both sides)."""
    w = S.WORKLOADS["llama3-8b-bf16-b16-kv4k8k-g128"]
    shape = w.shape.replace(n_layers=2)
    B = w.batch
    model, orc = build_pair(shape, w.seed, batch=B, max_tokens=B, flags=L.LLM_FLAG_CUDA_GRAPH)
    lens, caches = S.make_kv_prefill(shape, w.seed, B, *w.kv_len_range)
    assert int(lens.min()) >= 4096 and int(lens.max()) <= 8192
    install_prefilled_cache(model, orc, lens.numpy(), caches)
    del caches
    tok = S.make_tokens(w.seed, B, 1, shape.vocab, tag="decode0")[:, 0].numpy()
    nxt = torch.empty(B, dtype=torch.int32, device=DEV)
    logits = torch.empty(B, shape.vocab, device=DEV)
    checked = 0
    for step in range(2):
        L.llm_decode_step(model.h, torch.as_tensor(tok, dtype=torch.int32).to(DEV), nxt, logits)
        L.llm_synchronize(model.h)
        o_taps = []
        tok, o_logits = orc.decode(tok, o_taps)
        check_taps(gpu_taps(model, B), [t.reshape(B, -1) for t in o_taps], what=f"step {step}")
        assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
        checked += check_argmax(nxt.cpu().numpy(), o_logits)
    assert L.llm_kv_cache_get_lens(model.h, B) == [int(x) + 2 for x in lens]
    assert checked >= B
    model.free()


def test_llama2_mha_at_the_workload_batch_and_prompt(lib):
    """The Llama-2-7B multi-head workload at its own batch and prompt length (two
    layers): 8 sequences of 1024 tokens through the tensor-core prefill, then
    decode steps; per-layer hidden states, logits and argmax against the oracle."""
    w = S.WORKLOADS["llama2-7b-mha-bf16-b8-p1024-g256"]
    shape = w.shape.replace(n_layers=2, max_seq_len=w.prompt_len + 8)
    _run_tokens_case(shape, seed=w.seed, B=w.batch, T=w.prompt_len, steps=2, flags=L.LLM_FLAG_CUDA_GRAPH)


def test_long_context_decode_up_to_the_8192_context(lib):
    """Batch-1 decode against a cache of 8064 positions (two Llama-3-8B layers):
    many 32-key groups per attention warp and the longest cache the context allows."""
    w = S.WORKLOADS["llama3-8b-bf16-b1-kv8k-g128"]
    shape = w.shape.replace(n_layers=2)
    model, orc = build_pair(shape, w.seed, batch=1, max_tokens=1, flags=L.LLM_FLAG_CUDA_GRAPH)
    lens, caches = S.make_kv_prefill(shape, w.seed, 1, *w.kv_len_range)
    install_prefilled_cache(model, orc, lens.numpy(), caches)
    del caches
    tok = S.make_tokens(w.seed, 1, 1, shape.vocab, tag="decode0")[:, 0].numpy()
    nxt = torch.empty(1, dtype=torch.int32, device=DEV)
    logits = torch.empty(1, shape.vocab, device=DEV)
    for step in range(3):
        L.llm_decode_step(model.h, torch.as_tensor(tok, dtype=torch.int32).to(DEV), nxt, logits)
        L.llm_synchronize(model.h)
        o_taps = []
        tok, o_logits = orc.decode(tok, o_taps)
        check_taps(gpu_taps(model, 1), [t.reshape(1, -1) for t in o_taps], what=f"step {step}")
        check_argmax(nxt.cpu().numpy(), o_logits)
        assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
    assert L.llm_kv_cache_get_lens(model.h, 1) == [int(lens[0]) + 3]
    model.free()


def test_graph_replay_is_bitwise_identical_to_direct_launches(lib):
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=128)
    prompt = S.make_tokens(5, 2, 40, shape.vocab).to(DEV)
    results = []
    for flags in (0, L.LLM_FLAG_CUDA_GRAPH):
        glob, layers = S.make_weights(shape, 5)
        m = L.Model(shape, glob, layers, max_batch=2, max_tokens=80, flags=flags)
        nxt = torch.empty(2, dtype=torch.int32, device=DEV)
        lg = torch.empty(2, shape.vocab, device=DEV)
        L.llm_prefill(m.h, prompt, nxt, lg)
        seq = []
        for _ in range(5):
            cur = nxt.clone()
            L.llm_decode_step(m.h, cur, nxt, lg)
            L.llm_synchronize(m.h)
            seq.append((nxt.cpu().clone(), lg.cpu().clone()))
        results.append(seq)
        m.free()
    for (a, la), (b, lb) in zip(*results):
        assert torch.equal(a, b) and torch.equal(la, lb)


def test_host_side_errors_and_cache_reset(lib):
    shape = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"].shape.replace(max_seq_len=16)
    glob, layers = S.make_weights(shape, 9)
    m = L.Model(shape, glob, layers, max_batch=2, max_tokens=20)
    nxt = torch.empty(2, dtype=torch.int32, device=DEV)
    lg = torch.empty(2, shape.vocab, device=DEV)
    toks = S.make_tokens(9, 2, 10, shape.vocab).to(DEV)
    with pytest.raises(L.LlmError) as e:
        L.llm_prefill(m.h, S.make_tokens(9, 3, 2, shape.vocab).to(DEV), nxt, lg)   # B > max_batch
    assert e.value.code == L.LLM_ERR_BATCH
    L.llm_prefill(m.h, toks, nxt, lg)
    L.llm_synchronize(m.h)
    first = (nxt.cpu().clone(), lg.cpu().clone())
    with pytest.raises(L.LlmError) as e:
        L.llm_prefill(m.h, toks, nxt, lg)                                            # 10 + 10 > 16
    assert e.value.code == L.LLM_ERR_SEQ_OVERFLOW
    L.llm_kv_cache_reset(m.h)
    L.llm_prefill(m.h, toks, nxt, lg)
    L.llm_synchronize(m.h)
    assert torch.equal(first[0], nxt.cpu()) and torch.equal(first[1], lg.cpu())
    m.free()
