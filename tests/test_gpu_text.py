"""Text in, text out through the GPU path (GPU).

The walkthrough's tokenizer section turns its prompt into ids (with
<|begin_of_text|> in front), runs the model, and turns the predicted id back into
text. Here a small byte-level BPE vocabulary is trained and written in the
tokenizer.model format (the trained Llama-3 file is not available), the page's
prompt is encoded with it, the ids go through llm_prefill and llm_decode_step
of an fp32 model whose vocabulary is that tokenizer's, and the generated ids are
decoded back to text. The fp32 model must give exactly the oracle's greedy ids,
hence exactly its text.
"""
import base64
import json
import os

import pytest
import torch

import llama_decoder_forward_fwd_b200 as L
import seeded_inputs as S
from llama_decoder_forward_fwd_b200 import tokenizer as T
from model_util import build_pair
from test_tokenizer import CORPUS, _trained_vocab

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_tokenizer.json"), encoding="utf-8"))


def test_prompt_text_to_generated_text_matches_the_oracle(lib, tmp_path):
    ranks = _trained_vocab(CORPUS, 120)
    path = tmp_path / "tokenizer.model"
    with open(path, "wb") as f:
        for b, r in sorted(ranks.items(), key=lambda kv: kv[1]):
            f.write(base64.b64encode(b) + b" " + str(r).encode() + b"\n")
    tok = T.Tokenizer.from_file(str(path))
    ids = tok.encode(GOLD["prompt"], bos=True)
    assert ids[0] == tok.special["<|begin_of_text|>"] == tok.n_vocab_base
    assert tok.decode(ids[1:]) == GOLD["prompt"]

    steps = 16
    shape = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"].shape.replace(vocab=tok.n_vocab,
                                                                         max_seq_len=len(ids) + steps + 1)
    model, orc = build_pair(shape, 2025, batch=1, max_tokens=len(ids), flags=L.LLM_FLAG_CUDA_GRAPH, taps=False)
    prompt = torch.tensor([ids], dtype=torch.int32, device=DEV)
    nxt = torch.empty(1, dtype=torch.int32, device=DEV)
    L.llm_prefill(model.h, prompt, nxt)
    gen = [int(nxt.cpu()[0])]
    for _ in range(steps):
        L.llm_decode_step(model.h, nxt.clone(), nxt)
        gen.append(int(nxt.cpu()[0]))
    L.llm_synchronize(model.h)
    model.free()

    o_toks, _ = orc.generate([ids], steps)
    o_gen = [int(t[0]) for t in o_toks]
    assert gen == o_gen, f"GPU ids {gen} vs oracle ids {o_gen}"
    text = tok.decode(gen)
    assert text == tok.decode(o_gen)
    print(f"prompt {GOLD['prompt']!r} -> {len(ids)} ids -> generated {text!r}")
