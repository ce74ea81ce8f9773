"""Failure detection on the device, without a fault (GPU).

Every wait in the library's kernels (mbarrier waits of the TMA pipelines, the
grid barriers of the cooperative launches, the split-tile counters) is bounded:
when it runs out the kernel records a code in the model's device error word and
returns, and llm_synchronize() reports LLM_ERR_DEVICE_TIMEOUT. Here that path
runs on purpose: llm_debug_wait_probe queues a wait whose target is never
reached, bounded by 1 ms, on the library's own wait code. Nothing faults or
hangs; the model keeps working and gives the same results afterwards.
"""
import time

import numpy as np
import pytest
import torch

import llama_decoder_forward_fwd_b200 as L
import seeded_inputs as S
from model_util import build_pair

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier", "grid-barrier"])
def test_bounded_wait_runs_out_and_the_model_recovers(lib, which):
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=1, max_seq_len=64, vocab=1000)
    model, orc = build_pair(shape, 5, batch=1, max_tokens=8, flags=L.LLM_FLAG_CUDA_GRAPH, taps=False)
    prompt = S.make_tokens(5, 1, 8, shape.vocab).to(DEV)
    nxt = torch.empty(1, dtype=torch.int32, device=DEV)
    logits = torch.empty(1, shape.vocab, device=DEV)

    def step():
        L.llm_kv_cache_reset(model.h)
        L.llm_prefill(model.h, prompt, nxt)
        L.llm_decode_step(model.h, nxt.clone(), nxt, logits)
        L.llm_synchronize(model.h)
        return int(nxt[0]), logits.cpu().numpy().copy()

    tok0, lg0 = step()
    t0 = time.monotonic()
    L.llm_debug_wait_probe(model.h, which, 1.0)
    with pytest.raises(L.LlmError) as e:
        L.llm_synchronize(model.h)
    waited = time.monotonic() - t0
    assert e.value.code == L.LLM_ERR_DEVICE_TIMEOUT
    assert "0x501" in str(e.value)
    assert waited < 2.0, f"the 1 ms bound, not the 4 s default, should end the wait ({waited:.2f} s)"
    L.llm_synchronize(model.h)  # the word was cleared: no error left behind
    tok1, lg1 = step()          # the same model, the same result
    assert tok1 == tok0 and np.array_equal(lg1, lg0)
    model.free()


def test_wait_probe_rejects_bad_arguments(lib):
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape.replace(n_layers=1, max_seq_len=64, vocab=1000)
    model, _ = build_pair(shape, 6, batch=1, max_tokens=1, taps=False)
    for which, ms in ((2, 1.0), (0, 0.0), (1, -1.0), (0, 20000.0)):
        with pytest.raises(L.LlmError) as e:
            L.llm_debug_wait_probe(model.h, which, ms)
        assert e.value.code == L.LLM_ERR_BAD_ARG
    model.free()
