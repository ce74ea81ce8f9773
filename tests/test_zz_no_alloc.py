"""The allocation-free split-KV attention entry point, through the C ABI (GPU).

llm_op_attention_decode_static serves callers that cannot allocate device
memory (code inside a CUDA graph capture, plug-ins whose host owns every
allocation, latency-critical loops): it uses a fixed scratch array inside the
library instead of a caller-provided workspace. Here, on two calls in a row (the
second call finds the first call's leftovers in the shared scratch), it must
agree with the oracle's causal grouped-query attention and with
llm_op_attention_decode on the same inputs, within the split-KV tolerance of the
other attention tests. This file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, T, H, Hk, d, S, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, H, d, generator=g).to(dtype).to(DEV)
    kc = torch.randn(B, Hk, S, d, generator=g).to(dtype).to(DEV)
    vc = torch.randn(B, Hk, S, d, generator=g).to(dtype).to(DEV)
    return q, kc, vc


def _oracle(q, kc, vc, pos0):
    """Attention of each sequence's T new tokens (positions pos0 .. pos0+T-1) over keys 0 .. pos0+T-1."""
    B, T = q.shape[:2]
    out = []
    for b in range(B):
        n = pos0[b] + T
        k = O.f64(kc[b, :, :n]).transpose(1, 0, 2)
        v = O.f64(vc[b, :, :n]).transpose(1, 0, 2)
        out.append(O.attention(O.f64(q[b]), k, v, pos0[b] + np.arange(T), np.arange(n)))
    return np.stack(out)


@pytest.mark.parametrize("dtype,d,tol", [(torch.bfloat16, 128, 6e-3), (torch.float32, 48, 2e-5)])
@pytest.mark.parametrize("B,T,H,Hk,S,pos0", [(1, 1, 32, 8, 2304, [2047]), (3, 1, 32, 8, 2304, [0, 37, 700]),
                                              (2, 4, 8, 2, 2304, [9, 0]), (8, 1, 32, 8, 160, [0, 5, 31, 64, 99, 120, 150, 158])])
def test_static_scratch_matches_oracle_and_workspace_entry_point(lib, dtype, d, tol, B, T, H, Hk, S, pos0):
    import llama_decoder_forward_fwd_b200 as L
    p = torch.tensor(pos0, dtype=torch.int32, device=DEV)
    ws = torch.empty(L.llm_op_attention_decode_workspace(B, T, H, Hk, d), dtype=torch.uint8, device=DEV)
    for call in range(2):
        q, kc, vc = _inputs(B, T, H, Hk, d, S, dtype, 100 + call)
        ref = torch.full((B, T, H * d), float("nan"), dtype=dtype, device=DEV)
        got = torch.full((B, T, H * d), float("nan"), dtype=dtype, device=DEV)
        L.llm_op_attention_decode(q, kc, vc, p, ref, ws)
        L.llm_op_attention_decode_static(q, kc, vc, p, got)
        torch.cuda.synchronize()
        r, g = ref.float().cpu().numpy(), got.float().cpu().numpy()
        bound = tol * float(vc.abs().max())
        assert np.isfinite(g).all()
        assert np.abs(g - r).max() <= bound, (call, np.abs(g - r).max())
        want = _oracle(q.cpu(), kc.cpu(), vc.cpu(), pos0)
        assert np.abs(g - want).max() <= bound, (call, np.abs(g - want).max())


def test_static_scratch_rejects_shapes_beyond_its_size(lib):
    import llama_decoder_forward_fwd_b200 as L
    # 16 sequences of 8 new tokens over caches of 4096 positions: 6 splits of 256
    # groups of 16 rows, about 13 MB of partial results, more than the fixed 8 MiB
    B, T, H, Hk, d, S = 16, 8, 32, 8, 128, 4096
    q, kc, vc = _inputs(B, T, H, Hk, d, S, torch.bfloat16, 5)
    out = torch.zeros(B, T, H * d, dtype=torch.bfloat16, device=DEV)
    p = torch.zeros(B, dtype=torch.int32, device=DEV)
    with pytest.raises(L.LlmError) as e:
        L.llm_op_attention_decode_static(q, kc, vc, p, out)
    assert e.value.code == L.LLM_ERR_BAD_ARG
    assert "static scratch" in str(e.value)
