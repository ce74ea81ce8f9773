"""The seeded synthetic inputs both sides read (CPU).

The recipe: every tensor drawn from its own generator, seeded from (workload
seed, tensor name); weights N(0, 0.02) rounded to the model dtype with the
checkpoint's [out, in] shapes; norm weights 1; token ids uniform in [0, vocab);
hidden states N(0, 1) rounded to bf16-representable values; KV caches N(0, 1)
with per-sequence lengths uniform in the workload's range.
"""
import numpy as np
import pytest
import torch

import seeded_inputs as S

L3 = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape
TINY = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"].shape


def test_same_seed_same_bits_and_distinct_tensors_differ():
    a = S.make_layer_weights(TINY, 7, 1)
    b = S.make_layer_weights(TINY, 7, 1)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    other_layer = S.make_layer_weights(TINY, 7, 2)
    other_seed = S.make_layer_weights(TINY, 8, 1)
    for k in ("wq", "wk", "wv", "wo", "w1", "w2", "w3"):
        assert not torch.equal(a[k], other_layer[k]), k
        assert not torch.equal(a[k], other_seed[k]), k
    assert not torch.equal(a["w1"], a["w3"])          # same shape, different names


def test_weight_shapes_dtype_and_distribution():
    lw = S.make_layer_weights(L3, 0, 0)
    shapes = {"wq": (4096, 4096), "wk": (1024, 4096), "wv": (1024, 4096), "wo": (4096, 4096),
              "w1": (14336, 4096), "w3": (14336, 4096), "w2": (4096, 14336)}
    for k, shp in shapes.items():
        assert tuple(lw[k].shape) == shp, k            # [out, in]: y = x W^T
        assert lw[k].dtype == torch.bfloat16
    w = lw["wk"].float()
    assert abs(w.mean().item()) < 1e-4
    assert w.std().item() == pytest.approx(0.02, rel=0.01)
    for k in ("attention_norm", "ffn_norm"):
        assert torch.all(lw[k] == 1)
    g = S.make_global_weights(L3, 0)
    assert tuple(g["tok_embeddings"].shape) == (128256, 4096)
    assert tuple(g["output"].shape) == (128256, 4096)
    assert torch.all(g["norm"] == 1)
    assert "output" not in S.make_global_weights(TINY, 0)   # tied lm_head
    assert S.make_global_weights(L3.replace(has_embed_and_head=False), 0) == {}


def test_tokens_uniform_in_vocab():
    t = S.make_tokens(3, 4, 5000, 1000)
    assert t.dtype == torch.int32 and tuple(t.shape) == (4, 5000)
    assert int(t.min()) >= 0 and int(t.max()) < 1000
    counts = np.bincount(t.flatten().numpy(), minlength=1000)
    # 20000 draws over 1000 ids: every decile of ids holds about a tenth
    dec = counts.reshape(10, 100).sum(1) / counts.sum()
    assert np.all(np.abs(dec - 0.1) < 0.02)
    assert not torch.equal(S.make_tokens(3, 1, 16, 1000), S.make_tokens(3, 1, 16, 1000, tag="decode0"))


def test_hidden_states_are_bf16_representable_standard_normal():
    h = S.make_hidden(5, 2, 64, 512)
    assert h.dtype == torch.float32 and tuple(h.shape) == (2, 64, 512)
    assert torch.equal(h, h.to(torch.bfloat16).to(torch.float32))
    assert abs(h.mean().item()) < 0.02
    assert h.std().item() == pytest.approx(1.0, rel=0.02)


def test_kv_prefill_lengths_and_values():
    w = S.WORKLOADS["llama3-8b-bf16-b16-kv4k8k-g128"]
    shape = w.shape.replace(n_layers=1)
    lens, caches = S.make_kv_prefill(shape, w.seed, 16, 40, 300)
    assert lens.dtype == torch.int32 and len(lens) == 16
    assert int(lens.min()) >= 40 and int(lens.max()) <= 300
    assert len(set(lens.tolist())) > 8                 # ragged
    K, V = caches[0]
    assert tuple(K.shape) == (16, 8, 300, 128) and K.dtype == torch.bfloat16
    assert K.float().std().item() == pytest.approx(1.0, rel=0.02)
    assert not torch.equal(K, V)
    # the lengths depend only on the seed and the range, not on which layers are drawn
    lens2, none = S.make_kv_prefill(shape, w.seed, 16, 40, 300, layers=[])
    assert torch.equal(lens, lens2) and none == {}
    lo, hi = w.kv_len_range
    full = S.make_kv_prefill(w.shape, w.seed, w.batch, lo, hi, layers=[])[0]
    assert int(full.min()) >= 4096 and int(full.max()) <= 8192


def test_workload_caches_fit_the_context():
    for w in S.WORKLOADS.values():
        top = (w.kv_len_range[1] if w.input_kind == "kv_prefilled" else w.prompt_len) + w.decode_steps
        assert top <= w.shape.max_seq_len, w.name
