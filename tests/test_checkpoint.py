"""The loader for Meta's checkpoint layout (CPU).

The trained weights are not here, so the loader is checked on tensors with the
checkpoint's names: its key layout against the keys "Building llama3 from
scratch" prints for consolidated.00.pth, its config against the params.json the
same page prints, and its output against the seeded weights the parity tests
run (a model loaded from a checkpoint that holds the seeded tensors under
Meta's names gets exactly those tensors).
"""
import json
import os

import pytest
import torch

import seeded_inputs as S
from llama_decoder_forward_fwd_b200 import checkpoint as C

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_shapes.json")))


def _as_checkpoint(shape, seed):
    """The seeded weights of `shape` stored under Meta's key names."""
    glob, layers = S.make_weights(shape, seed)
    sd = {C.GLOBAL_KEYS[k]: v for k, v in glob.items()}
    for i, lw in enumerate(layers):
        for k, v in lw.items():
            sd[C.LAYER_KEYS[k].format(i=i)] = v
    return sd, glob, layers


def _meta_llama3_8b(n_layers=32, ffn=14336):
    """Shapes-only tensors of the Llama-3-8B checkpoint (no storage)."""
    p = GOLD["llama3_8b_params"]
    D, V = p["dim"], p["vocab_size"]
    kvd = p["n_kv_heads"] * D // p["n_heads"]
    sd = {"tok_embeddings.weight": torch.empty(V, D, dtype=torch.bfloat16, device="meta"),
          "norm.weight": torch.empty(D, dtype=torch.bfloat16, device="meta"),
          "output.weight": torch.empty(V, D, dtype=torch.bfloat16, device="meta")}
    shp = {"wq": (D, D), "wk": (kvd, D), "wv": (kvd, D), "wo": (D, D), "w1": (ffn, D), "w3": (ffn, D),
           "w2": (D, ffn), "attention_norm": (D,), "ffn_norm": (D,)}
    for i in range(n_layers):
        for k, s in shp.items():
            sd[C.LAYER_KEYS[k].format(i=i)] = torch.empty(*s, dtype=torch.bfloat16, device="meta")
    return p, sd


def test_key_layout_matches_the_printed_checkpoint_keys():
    assert C.key_order(32)[:11] == GOLD["llama3_8b_first_11_checkpoint_keys"]
    assert len(C.key_order(32)) == 1 + 9 * 32 + 2


def test_config_of_the_printed_llama3_8b_params():
    params, sd = _meta_llama3_8b()
    cfg = C.config_from_checkpoint(params, sd, max_seq_len=8192)
    assert (cfg.dim, cfg.n_layers, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim) == (4096, 32, 32, 8, 128)
    assert (cfg.vocab, cfg.ffn_hidden, cfg.max_seq_len) == (128256, 14336, 8192)
    assert cfg.norm_eps == pytest.approx(1e-5) and cfg.rope_theta == 500000.0
    assert cfg.dtype == "bf16" and not cfg.tie_embeddings and cfg.has_embed_and_head
    shapes = C.expected_shapes(cfg)
    for k, s in GOLD["llama3_8b_layer0_weight_shapes"].items():
        assert shapes[C.LAYER_KEYS[k].format(i=0)] == tuple(s)
    for key, t in sd.items():
        assert shapes[key] == tuple(t.shape), key
    assert set(shapes) == set(sd)
    # the config is what the benchmark's Llama-3-8B workload runs
    w = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape
    for f in ("dim", "n_layers", "n_heads", "n_kv_heads", "head_dim", "ffn_hidden", "vocab", "rope_theta"):
        assert getattr(cfg, f) == getattr(w, f), f


@pytest.mark.parametrize("name", ["tiny-llama2-f32-d288-b1-p8-g50", "llama3-8b-1layer-bf16-b1-h512-d64"])
def test_split_returns_exactly_the_seeded_tensors(name):
    shape = S.WORKLOADS[name].shape
    if not shape.has_embed_and_head:      # the loader reads full models: give the layer an embedding and head
        shape = shape.replace(has_embed_and_head=True, vocab=64)
    shape = shape.replace(ffn_hidden=min(shape.ffn_hidden, 256))
    sd, glob, layers = _as_checkpoint(shape, 3)
    params = {"dim": shape.dim, "n_layers": shape.n_layers, "n_heads": shape.n_heads,
              "n_kv_heads": shape.n_kv_heads, "vocab_size": shape.vocab, "norm_eps": shape.norm_eps,
              "rope_theta": shape.rope_theta}
    cfg = C.config_from_checkpoint(params, sd, max_seq_len=shape.max_seq_len)
    assert cfg.tie_embeddings == shape.tie_embeddings and cfg.dtype == shape.dtype
    g2, l2 = C.split_state_dict(sd, cfg)
    assert set(g2) == set(glob)
    for k in glob:
        assert torch.equal(g2[k], glob[k]), k
    for a, b in zip(l2, layers):
        assert set(a) == set(b)
        for k in a:
            assert torch.equal(a[k], b[k]) and a[k].is_contiguous(), k


def test_llama2_style_params_and_missing_or_misshapen_keys():
    shape = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"].shape.replace(ffn_hidden=64)
    sd, _, _ = _as_checkpoint(shape, 4)
    params = {"dim": 288, "n_layers": 6, "n_heads": 6, "vocab_size": -1, "norm_eps": 1e-5}
    cfg = C.config_from_checkpoint(params, sd, max_seq_len=256)
    assert cfg.n_kv_heads == 6 and cfg.vocab == 32000 and cfg.rope_theta == 10000.0 and cfg.tie_embeddings
    broken = dict(sd)
    del broken["layers.3.feed_forward.w2.weight"]
    with pytest.raises(ValueError, match="layers.3.feed_forward.w2.weight"):
        C.split_state_dict(broken, cfg)
    broken = dict(sd)
    broken["layers.0.feed_forward.w1.weight"] = broken["layers.0.feed_forward.w1.weight"].t()   # [in, out]
    with pytest.raises(ValueError, match="layers.0.feed_forward.w1.weight"):
        C.split_state_dict(broken, C.config_from_checkpoint(params, sd, 256))
    with pytest.raises(ValueError, match="n_heads"):
        C.config_from_checkpoint({"dim": 288, "n_layers": 6}, sd, 256)
    with pytest.raises(ValueError, match="do not divide"):
        C.config_from_checkpoint(dict(params, n_kv_heads=4), sd, 256)


def test_files_on_disk(tmp_path):
    shape = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"].shape.replace(ffn_hidden=64, n_layers=2)
    sd, glob, _ = _as_checkpoint(shape, 5)
    torch.save(sd, tmp_path / "consolidated.00.pth")
    (tmp_path / "params.json").write_text(json.dumps({"dim": 288, "n_layers": 2, "n_heads": 6, "vocab_size": 32000}))
    params = C.read_params(str(tmp_path / "params.json"))
    sd2 = C.read_state_dict(str(tmp_path / "consolidated.00.pth"))
    cfg = C.config_from_checkpoint(params, sd2, 256)
    g2, _ = C.split_state_dict(sd2, cfg)
    assert torch.equal(g2["tok_embeddings"], glob["tok_embeddings"])


def test_load_model_hands_the_config_and_weights_to_the_binding(tmp_path, monkeypatch):
    import llama_decoder_forward_fwd_b200 as L
    shape = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"].shape.replace(ffn_hidden=64, n_layers=2)
    sd, glob, layers = _as_checkpoint(shape, 6)
    torch.save(sd, tmp_path / "consolidated.00.pth")
    (tmp_path / "params.json").write_text(json.dumps({"dim": 288, "n_layers": 2, "n_heads": 6, "vocab_size": 32000}))
    seen = {}

    class Recorder:
        def __init__(self, cfg, glob, layers, **kw):
            seen.update(cfg=cfg, glob=glob, layers=layers, **kw)

    monkeypatch.setattr(L, "Model", Recorder)
    C.load_model(str(tmp_path / "params.json"), str(tmp_path / "consolidated.00.pth"), max_seq_len=256,
                 max_batch=2, max_tokens=16, flags=L.LLM_FLAG_CUDA_GRAPH, device="cpu")
    assert seen["max_batch"] == 2 and seen["max_tokens"] == 16 and seen["flags"] == L.LLM_FLAG_CUDA_GRAPH
    assert seen["cfg"].max_seq_len == 256 and seen["cfg"].tie_embeddings
    assert torch.equal(seen["layers"][1]["w2"], layers[1]["w2"])
    cfg = L.make_config(seen["cfg"], max_batch=2)
    assert (cfg.dim, cfg.n_kv_heads, cfg.ffn_hidden, cfg.tie_embeddings, cfg.dtype) == (288, 6, 64, 1, L.LLM_F32)
