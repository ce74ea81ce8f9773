"""Run under LLM_LIB_VARIANT=checked by test_gpu_bounds_checked.py (not a test module).

Loads the bounds-checking build of the library and runs small cases of every
kernel family against the oracle with the device error word left at zero, then
one out-of-range token id, which the checked embedding must report as
LLM_ERR_DEVICE_BOUNDS without touching memory outside the table, after which
the model keeps working, and a prefill attention whose new tokens would run past
the cache, reported the same way.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import llama_decoder_forward_fwd_b200 as L  # noqa: E402
import oracle as O  # noqa: E402
import seeded_inputs as S  # noqa: E402
from model_util import BF16_REL_L2, build_pair, check_taps, gpu_taps, rel_l2  # noqa: E402

DEV = "cuda"


def ops():
    g = torch.Generator().manual_seed(5)
    # GEMV and tensor-core GEMM against fp64 products of the same bf16 operands
    x = torch.randn(3, 512, generator=g).to(torch.bfloat16)
    W = torch.randn(640, 512, generator=g).to(torch.bfloat16)
    ws = torch.empty(L.llm_op_gemv_workspace(640, 512), dtype=torch.uint8, device=DEV)
    y = torch.empty(3, 640, device=DEV)
    L.llm_op_gemv_bf16(x.to(DEV), W.to(DEV), y, ws)
    L.llm_op_synchronize()
    ref = O.f64(x) @ O.f64(W).T
    assert np.abs(y.cpu().numpy() - ref).max() <= 1e-3 * np.abs(ref).max()
    A = torch.randn(200, 256, generator=g).to(torch.bfloat16)
    Bm = torch.randn(512, 256, generator=g).to(torch.bfloat16)
    C = torch.empty(200, 512, device=DEV)
    L.llm_op_gemm_bf16(A.to(DEV), Bm.to(DEV), C)
    L.llm_op_synchronize()
    ref = O.f64(A) @ O.f64(Bm).T
    assert np.abs(C.cpu().numpy() - ref).max() <= 1e-3 * np.abs(ref).max()
    # attention: prefill (tcgen05), split-KV decode, allocation-free decode
    B, T, H, Hk, d, Smax, pos0 = 2, 9, 8, 2, 128, 256, [0, 100]
    q = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)
    kc = torch.randn(B, Hk, Smax, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(B, Hk, Smax, d, generator=g).to(torch.bfloat16)
    ref = np.empty((B, T, H * d))
    for b in range(B):
        n = pos0[b] + T
        ref[b] = O.attention(O.f64(q[b]), O.f64(kc[b, :, :n]).transpose(1, 0, 2),
                             O.f64(vc[b, :, :n]).transpose(1, 0, 2), pos0[b] + np.arange(T), np.arange(n))
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    out = torch.empty(B, T, H * d, dtype=torch.bfloat16, device=DEV)
    bound = 8e-3 * float(vc.abs().max())
    L.llm_op_attention_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out)
    L.llm_op_synchronize()
    assert np.abs(O.f64(out.cpu()) - ref).max() <= bound
    wsa = torch.empty(L.llm_op_attention_decode_workspace(B, T, H, Hk, d), dtype=torch.uint8, device=DEV)
    out.zero_()
    L.llm_op_attention_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out, wsa)
    L.llm_op_synchronize()
    assert np.abs(O.f64(out.cpu()) - ref).max() <= bound
    out.zero_()
    L.llm_op_attention_decode_static(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out)
    L.llm_op_synchronize()
    assert np.abs(O.f64(out.cpu()) - ref).max() <= bound
    # new tokens that would run past the cache: the attention kernels read only
    # inside it (their positions are clamped) and the checked build reports them
    bad = torch.tensor([0, Smax - T + 1], dtype=torch.int32, device=DEV)
    L.llm_op_attention_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), bad, out)
    try:
        L.llm_op_synchronize()
        raise AssertionError("the checked build did not report the attention positions")
    except L.LlmError as e:
        assert e.code == L.LLM_ERR_DEVICE_BOUNDS and "attention" in str(e), (e.code, str(e))
    L.llm_op_attention_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), p, out)
    L.llm_op_synchronize()
    assert np.abs(O.f64(out.cpu()) - ref).max() <= bound


def bf16_model():
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=2, max_seq_len=128)
    B, T, seed = 2, 40, 81
    model, orc = build_pair(shape, seed, batch=B, max_tokens=B * T, flags=L.LLM_FLAG_CUDA_GRAPH)
    prompt = S.make_tokens(seed, B, T, shape.vocab)
    nxt = torch.empty(B, dtype=torch.int32, device=DEV)
    logits = torch.empty(B, shape.vocab, device=DEV)
    L.llm_prefill(model.h, prompt.to(DEV), nxt, logits)
    L.llm_synchronize(model.h)
    o_taps = []
    o_next, o_logits = orc.prefill(prompt.numpy(), o_taps)
    check_taps(gpu_taps(model, B * T), [t.reshape(B * T, -1) for t in o_taps], what="prefill")
    assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
    for step in range(3):
        tok = torch.as_tensor(o_next, dtype=torch.int32).to(DEV)
        L.llm_decode_step(model.h, tok, nxt, logits)
        L.llm_synchronize(model.h)
        o_taps = []
        o_next, o_logits = orc.decode(o_next, o_taps)
        check_taps(gpu_taps(model, B), [t.reshape(B, -1) for t in o_taps], what=f"decode {step}")
        assert rel_l2(logits.cpu().numpy(), o_logits) <= BF16_REL_L2
    # an out-of-range token id: reported, nothing read outside the table, model still usable
    bad = torch.tensor([shape.vocab + 5, 3], dtype=torch.int32, device=DEV)
    L.llm_decode_step(model.h, bad, nxt, logits)
    try:
        L.llm_synchronize(model.h)
        raise AssertionError("the checked build did not report the token id")
    except L.LlmError as e:
        assert e.code == L.LLM_ERR_DEVICE_BOUNDS, e.code
        assert "token id" in str(e), str(e)
    L.llm_decode_step(model.h, torch.tensor([1, 2], dtype=torch.int32, device=DEV), nxt, logits)
    L.llm_synchronize(model.h)
    assert L.llm_kv_cache_get_lens(model.h, B) == [T + 5, T + 5]
    model.free()


def f32_model():
    w = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"]
    s = w.shape
    model, orc = build_pair(s, w.seed, batch=1, max_tokens=w.prompt_len, taps=False)
    prompt = S.make_tokens(w.seed, 1, w.prompt_len, s.vocab)
    nxt = torch.empty(1, dtype=torch.int32, device=DEV)
    L.llm_prefill(model.h, prompt.to(DEV), nxt)
    L.llm_synchronize(model.h)
    o_next, _ = orc.prefill(prompt.numpy())
    stream, o_stream = [int(nxt[0])], [int(o_next[0])]
    for _ in range(10):
        L.llm_decode_step(model.h, nxt.clone(), nxt)
        L.llm_synchronize(model.h)
        o_next, _ = orc.decode(o_next)
        stream.append(int(nxt[0]))
        o_stream.append(int(o_next[0]))
    assert stream == o_stream, (stream, o_stream)
    model.free()


if __name__ == "__main__":
    assert os.path.basename(L.LIB_PATH) == "liblfwd_checked.so", L.LIB_PATH
    L.load()
    assert L.llm_build_flags() == L.LLM_BUILD_BOUNDS_CHECK
    ops()
    f32_model()
    bf16_model()
    print("CHECKED OK")
