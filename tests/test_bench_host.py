"""Host-side arithmetic of bench.py (CPU): the algorithmic work behind the rooflines.

`achieved` in the bench line is algorithmic bytes (or FLOPs) per launch over the
measured launch time, so the counts are checked here against closed forms
written out from the Llama-3-8B shape ("Building llama3 from scratch": dim 4096,
32 layers, 32 query / 8 KV heads of 128, FFN 14336, vocabulary 128256), not
against bench.py's own formula.
"""
import pytest

import bench
import seeded_inputs as S

W = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"]


def test_llama3_8b_parameter_counts():
    s = W.shape
    per_layer = (4096 * 4096          # wq
                 + 2 * 1024 * 4096    # wk, wv (8 KV heads x 128)
                 + 4096 * 4096        # wo
                 + 3 * 14336 * 4096)  # w1, w3, w2
    assert per_layer == 218_103_808
    embed = 128256 * 4096
    # 32 layers + embedding + lm_head = the 8.03 B parameters of the model file
    assert 32 * per_layer + 2 * embed == pytest.approx(8.03e9, rel=1e-3)
    assert s.n_layers * per_layer == 6_979_321_856


def test_decode_bytes_per_step_are_weights_once_plus_the_cache_once():
    s = W.shape
    for S_mean in (1.0, 2048.0, 2176.0):
        _, step_bytes, kinds, _ = bench.work_model(s, 1, W.prompt_len, S_mean)
        weights = 2 * (32 * 218_103_808 + 128256 * 4096)     # bf16, lm_head read, embedding row not counted
        kv_per_position = 32 * 2 * 8 * 128 * 2                 # layers x (K, V) x heads x dims x bf16
        assert kv_per_position == 128 * 1024
        assert step_bytes == pytest.approx(weights + kv_per_position * S_mean, rel=1e-12)
    # one launch of each decode projection reads its weight matrix once
    assert kinds["qkv"] == 2 * 6144 * 4096
    assert kinds["wo"] == 2 * 4096 * 4096
    assert kinds["w13"] == 2 * 2 * 14336 * 4096 == 234_881_024
    assert kinds["w2"] == 2 * 14336 * 4096
    assert kinds["head"] == 2 * 128256 * 4096
    assert kinds["attn"] == pytest.approx(2 * 8 * 128 * 2 * 2176.0)   # one layer's K and V at S = 2176


def test_prefill_flops_are_linear_plus_causal_attention_plus_last_position_head():
    s = W.shape
    T = W.prompt_len
    flops, _, _, kinds = bench.work_model(s, 1, T, T)
    linear = 2 * T * 32 * 218_103_808
    attention = 32 * 4 * 32 * 128 * T * T / 2        # QK^T and PV over the causal half, 32 heads, 32 layers
    head = 2 * 4096 * 128256                           # lm_head on the last position only
    assert flops == pytest.approx(linear + attention + head, rel=1e-12)
    assert linear == pytest.approx(28.6e12, rel=2e-3)
    assert attention == pytest.approx(1.1e12, rel=3e-2)
    assert kinds["w13"] == 2 * T * 2 * 14336 * 4096


def test_batched_workload_bytes_scale_the_cache_by_the_batch():
    w = S.WORKLOADS["llama3-8b-bf16-b16-kv4k8k-g128"]
    _, b1, _, _ = bench.work_model(w.shape, 1, 0, 6144.0)
    _, b16, _, _ = bench.work_model(w.shape, 16, 0, 6144.0)
    assert b16 - b1 == pytest.approx(15 * 128 * 1024 * 6144.0, rel=1e-12)   # weights once, 16 caches


def test_replica_throughput_counts_every_rank():
    assert bench.replica_throughput(4, 5, 2304, 2.0) == pytest.approx(4 * 5 * 2304 / 2.0)


def test_peaks_come_from_the_measured_file_and_fall_back_when_it_is_unusable(tmp_path):
    import json

    p = tmp_path / "peaks.json"
    p.write_text(json.dumps({"hbm_gbs": 6547.5, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1363.4,
                             "clocks": {"sm_mhz": 1965}}))
    peaks, src = bench.load_peaks(str(p))
    assert src == "measured"
    assert peaks == {"hbm_gbs": 6547.5, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1363.4}
    p.write_text(json.dumps({"hbm_gbs": 6547.5, "bf16_tflops": 1674.6}))
    assert bench.load_peaks(str(p))[0]["bf16_tflops_sustained"] == 1674.6
    for bad in ('{"hbm_gbs": 6547.5}', '{"hbm_gbs": "n/a", "bf16_tflops": 1}', "[1, 2]", "not json",
                '{"hbm_gbs": 0, "bf16_tflops": 1674.6}'):
        p.write_text(bad)
        peaks, src = bench.load_peaks(str(p))
        assert src == "fallback" and peaks == bench.PEAKS_FALLBACK
    assert bench.load_peaks(str(tmp_path / "absent.json"))[1] == "fallback"
