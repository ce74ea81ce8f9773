"""A model loaded from Meta's checkpoint layout runs through the C ABI (GPU).

The tiny fp32 model's seeded weights are written under the checkpoint's key
names (consolidated.00.pth) with a params.json, loaded with
checkpoint.load_model, and its prefill is checked against the fp64 oracle on
the same weights: the same next token and logits within 1e-4.
"""
import json

import numpy as np
import pytest
import torch

import llama_decoder_forward_fwd_b200 as L
import oracle as O
import seeded_inputs as S
from llama_decoder_forward_fwd_b200 import checkpoint as C
from model_util import F32_LOGIT_REL

pytestmark = pytest.mark.gpu


def test_tiny_model_from_checkpoint_files(lib, tmp_path):
    w = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"]
    s = w.shape
    glob, layers = S.make_weights(s, w.seed)
    sd = {C.GLOBAL_KEYS[k]: v for k, v in glob.items()}
    for i, lw in enumerate(layers):
        for k, v in lw.items():
            sd[C.LAYER_KEYS[k].format(i=i)] = v
    torch.save(sd, tmp_path / "consolidated.00.pth")
    (tmp_path / "params.json").write_text(json.dumps(
        {"dim": s.dim, "n_layers": s.n_layers, "n_heads": s.n_heads, "n_kv_heads": s.n_kv_heads,
         "vocab_size": s.vocab, "norm_eps": s.norm_eps, "rope_theta": s.rope_theta}))
    m = C.load_model(str(tmp_path / "params.json"), str(tmp_path / "consolidated.00.pth"),
                     max_seq_len=s.max_seq_len, max_batch=1, max_tokens=w.prompt_len)
    prompt = S.make_tokens(w.seed, 1, w.prompt_len, s.vocab)
    nxt = torch.empty(1, dtype=torch.int32, device="cuda")
    logits = torch.empty(1, s.vocab, device="cuda")
    L.llm_prefill(m.h, prompt.to("cuda"), nxt, logits)
    L.llm_synchronize(m.h)
    o_next, o_logits = O.OracleModel(s, glob, layers, 1).prefill(prompt.numpy())
    err = np.abs(logits.cpu().numpy() - o_logits).max() / np.abs(o_logits).max()
    assert err <= F32_LOGIT_REL, err
    assert int(nxt[0]) == int(o_next[0])
    m.free()
