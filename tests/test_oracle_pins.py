"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

None of these re-types an oracle formula: they check closed forms, invariants,
special cases, page-printed shapes, and an independently written scalar
(pure-Python) model. Each is chosen so that a plausible slip in the oracle (a
dropped eps, a rotation sign, a wrong pair or frequency index, an off-by-one
mask, a transposed projection, a wrong GQA head map, a swapped w1/w3) fails at
least one of them.
"""
import cmath
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import seeded_inputs as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(7)


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_output_has_unit_rms_before_weight():
    # RMS of x * rsqrt(mean(x^2) + eps) is sqrt(ms / (ms + eps)): exactly 1 when eps = 0.
    for scale in (1e-3, 1.0, 37.0):
        x = RNG.standard_normal((5, 64)) * scale
        ones = np.ones(64)
        y0 = O.rmsnorm(x, ones, 0.0)
        np.testing.assert_allclose(np.sqrt(np.mean(y0 ** 2, -1)), 1.0, rtol=1e-14)
        eps = 1e-5
        y = O.rmsnorm(x, ones, eps)
        ms = np.mean(x ** 2, -1)
        np.testing.assert_allclose(np.sqrt(np.mean(y ** 2, -1)), np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_rmsnorm_constant_vector_and_weight():
    c, eps = 0.01, 1e-5       # small c makes eps visible: a dropped eps fails here
    y = O.rmsnorm(np.full(8, c), np.ones(8), eps)
    np.testing.assert_allclose(y, c / math.sqrt(c * c + eps), rtol=1e-15)
    w = RNG.standard_normal(8)
    x = RNG.standard_normal(8)
    np.testing.assert_allclose(O.rmsnorm(x, w, eps), O.rmsnorm(x, np.ones(8), eps) * w, rtol=1e-15)


# ---------------------------------------------------------------- RoPE
def _rope_complex(x, pos, theta):
    """RoPE in its complex form: pair (x[2i], x[2i+1]) as x[2i] + j x[2i+1] times e^{j p theta^(-2i/d)}."""
    d = x.shape[-1]
    out = np.empty_like(x)
    for t in range(x.shape[0]):
        for h in range(x.shape[1]):
            for i in range(d // 2):
                z = complex(x[t, h, 2 * i], x[t, h, 2 * i + 1])
                z *= cmath.exp(1j * pos[t] * theta ** (-2.0 * i / d))
                out[t, h, 2 * i], out[t, h, 2 * i + 1] = z.real, z.imag
    return out


def test_rope_matches_complex_rotation():
    x = RNG.standard_normal((6, 3, 8))
    pos = np.array([0, 1, 2, 5, 17, 300])
    np.testing.assert_allclose(O.rope(x, pos, 10000.0), _rope_complex(x, pos, 10000.0), atol=1e-13)


def test_rope_pair0_rotates_by_position_radians():
    # Pair 0 has frequency theta^0 = 1, so position p rotates it by p radians: (1, 0) -> (cos p, sin p).
    x = np.zeros((1, 1, 4))
    x[0, 0, 0] = 1.0
    y = O.rope(x, np.array([3]), 500000.0)
    np.testing.assert_allclose(y[0, 0, :2], [math.cos(3.0), math.sin(3.0)], atol=1e-15)


def test_rope_identity_at_position_zero_and_preserves_pair_norms():
    x = RNG.standard_normal((4, 2, 16))
    np.testing.assert_array_equal(O.rope(x[:1], np.array([0]), 500000.0), x[:1])
    y = O.rope(x, np.array([1, 9, 100, 4095]), 500000.0)
    n_in = np.hypot(x[..., 0::2], x[..., 1::2])
    n_out = np.hypot(y[..., 0::2], y[..., 1::2])
    np.testing.assert_allclose(n_out, n_in, rtol=1e-13)


def test_rope_dot_product_depends_only_on_offset():
    # "LLaMA2" page: q.k after rotation depends only on q, k and the offset m - n.
    q = RNG.standard_normal((1, 1, 128))
    k = RNG.standard_normal((1, 1, 128))
    for (m, n) in [(5, 2), (100, 37), (2047, 0)]:
        base = np.sum(O.rope(q, np.array([m]), 500000.0) * O.rope(k, np.array([n]), 500000.0))
        for delta in (1, 13, 999):
            moved = np.sum(O.rope(q, np.array([m + delta]), 500000.0) * O.rope(k, np.array([n + delta]), 500000.0))
            assert abs(moved - base) < 1e-10 * max(1.0, abs(base))


# ---------------------------------------------------------------- softmax / SiLU / argmax
def test_softmax_rows_sum_to_one_and_shift_invariant():
    s = RNG.standard_normal((7, 33)) * 10
    p = O.softmax(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-15)
    np.testing.assert_allclose(O.softmax(s + 123.0), p, atol=1e-15)
    s[:, 5:] = -np.inf
    p = O.softmax(s)
    assert np.all(p[:, 5:] == 0.0)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-15)


def test_silu_special_values():
    assert O.silu(np.array(0.0)) == 0.0
    np.testing.assert_allclose(O.silu(np.array(1.0)), 1.0 / (1.0 + math.exp(-1.0)), rtol=1e-15)
    np.testing.assert_allclose(O.silu(np.array(40.0)), 40.0, rtol=1e-15)
    assert abs(O.silu(np.array(-40.0))) < 1e-15
    # SwiGLU with a zero linear branch (w3) is zero: w3 multiplies, it is not the gate.
    x = RNG.standard_normal((3, 8))
    w1, w2 = RNG.standard_normal((16, 8)), RNG.standard_normal((8, 16))
    assert np.all(O.swiglu_ffn(x, w1, np.zeros((16, 8)), w2) == 0.0)
    # One-dimensional case: x = 1, w1 = a, w3 = b, w2 = c gives c * silu(a) * b, so the
    # gate is w1 (a swapped w1/w3 would give c * silu(b) * a).
    a, b, c = 2.0, -0.5, 3.0
    got = O.swiglu_ffn(np.array([[1.0]]), np.array([[a]]), np.array([[b]]), np.array([[c]]))
    np.testing.assert_allclose(got, [[c * b * a / (1.0 + math.exp(-a))]], rtol=1e-15)


def test_argmax_ties_take_lowest_index():
    lg = np.array([[0.0, 3.0, 1.0, 3.0], [-1.0, -1.0, -1.0, -2.0]])
    assert list(O.argmax_first(lg)) == [1, 0]
    np.testing.assert_allclose(O.top2_margin(np.array([1.0, 5.0, 4.5])), 0.5)


# ---------------------------------------------------------------- attention
def test_attention_position_zero_returns_first_value():
    q = RNG.standard_normal((1, 4, 8))
    k = RNG.standard_normal((1, 2, 8))
    v = RNG.standard_normal((1, 2, 8))
    out = O.attention(q, k, v, np.array([0]), np.array([0]))
    np.testing.assert_array_equal(out.reshape(4, 8), np.repeat(v[0], 2, axis=0))


def test_attention_equal_scores_average_visible_values():
    T = 6
    q = np.zeros((T, 2, 4))          # zero query: every visible key scores 0
    k = RNG.standard_normal((T, 1, 4))
    v = RNG.standard_normal((T, 1, 4))
    pos = np.arange(T)
    out = O.attention(q, k, v, pos, pos).reshape(T, 2, 4)
    for t in range(T):
        np.testing.assert_allclose(out[t, 0], v[: t + 1, 0].mean(0), atol=1e-15)
        np.testing.assert_allclose(out[t, 1], v[: t + 1, 0].mean(0), atol=1e-15)


def _mha_loops(q, k, v):
    """Independent multi-head causal attention written with explicit loops (H == Hk)."""
    T, H, d = q.shape
    out = np.zeros((T, H, d))
    for h in range(H):
        for t in range(T):
            sc = [float(np.dot(q[t, h], k[j, h])) / math.sqrt(d) for j in range(t + 1)]
            mx = max(sc)
            e = [math.exp(s - mx) for s in sc]
            z = sum(e)
            for j in range(t + 1):
                out[t, h] += e[j] / z * v[j, h]
    return out.reshape(T, H * d)


def test_gqa_reduces_to_mha_and_repeats_kv_heads():
    T, H, d = 5, 4, 6
    q = RNG.standard_normal((T, H, d))
    k = RNG.standard_normal((T, H, d))
    v = RNG.standard_normal((T, H, d))
    pos = np.arange(T)
    np.testing.assert_allclose(O.attention(q, k, v, pos, pos), _mha_loops(q, k, v), atol=1e-13)
    # G = 2: query heads (0,1) read KV head 0, (2,3) read KV head 1.
    k2, v2 = k[:, :2], v[:, :2]
    kr, vr = np.repeat(k2, 2, axis=1), np.repeat(v2, 2, axis=1)
    np.testing.assert_allclose(O.attention(q, k2, v2, pos, pos), _mha_loops(q, kr, vr), atol=1e-13)


# ---------------------------------------------------------------- whole model
TINY = S.ModelShape(dim=16, n_layers=2, n_heads=4, n_kv_heads=2, head_dim=4, ffn_hidden=32,
                    vocab=64, max_seq_len=32, norm_eps=1e-5, rope_theta=10000.0, dtype="f32",
                    tie_embeddings=False)


def _tiny_weights(seed=3):
    g, layers = S.make_weights(TINY, seed)
    # Non-unit norm weights so that a dropped or misplaced norm weight is caught.
    for i, lw in enumerate(layers):
        gen = torch.Generator().manual_seed(100 + i)
        lw["attention_norm"] = 1.0 + 0.1 * torch.randn(16, generator=gen)
        lw["ffn_norm"] = 1.0 + 0.1 * torch.randn(16, generator=gen)
    g["norm"] = 1.0 + 0.1 * torch.randn(16, generator=torch.Generator().manual_seed(99))
    return g, layers


def _scalar_model(glob, layers, tokens):
    """The tiny decoder written with Python scalars and lists only (brute force)."""
    D, H, Hk, d, eps, theta = 16, 4, 2, 4, 1e-5, 10000.0
    G = H // Hk
    tolist = lambda t: t.to(torch.float64).tolist()
    E = tolist(glob["tok_embeddings"])

    def matvec(W, x):
        return [sum(W[r][c] * x[c] for c in range(len(x))) for r in range(len(W))]

    def norm(x, w):
        r = 1.0 / math.sqrt(sum(a * a for a in x) / len(x) + eps)
        return [x[i] * r * w[i] for i in range(len(x))]

    def rot(vec, p):
        out = list(vec)
        for i in range(d // 2):
            a = p * theta ** (-2.0 * i / d)
            x0, x1 = vec[2 * i], vec[2 * i + 1]
            out[2 * i] = math.cos(a) * x0 - math.sin(a) * x1
            out[2 * i + 1] = math.sin(a) * x0 + math.cos(a) * x1
        return out

    hs = [list(E[t]) for t in tokens]
    T = len(tokens)
    for lw in layers:
        W = {k: tolist(v) for k, v in lw.items()}
        K, V, att = [], [], []
        for t in range(T):
            x = norm(hs[t], W["attention_norm"])
            q, k, v = matvec(W["wq"], x), matvec(W["wk"], x), matvec(W["wv"], x)
            K.append([rot(k[j * d:(j + 1) * d], t) for j in range(Hk)])
            V.append([v[j * d:(j + 1) * d] for j in range(Hk)])
            o = []
            for h in range(H):
                qh = rot(q[h * d:(h + 1) * d], t)
                sc = [sum(qh[i] * K[j][h // G][i] for i in range(d)) / math.sqrt(d) for j in range(t + 1)]
                mx = max(sc)
                e = [math.exp(s - mx) for s in sc]
                z = sum(e)
                o += [sum(e[j] / z * V[j][h // G][i] for j in range(t + 1)) for i in range(d)]
            att.append(o)
        for t in range(T):
            a = matvec(W["wo"], att[t])
            hs[t] = [hs[t][i] + a[i] for i in range(D)]
            x = norm(hs[t], W["ffn_norm"])
            g1, g3 = matvec(W["w1"], x), matvec(W["w3"], x)
            gg = [g1[i] / (1.0 + math.exp(-g1[i])) * g3[i] for i in range(len(g1))]
            f = matvec(W["w2"], gg)
            hs[t] = [hs[t][i] + f[i] for i in range(D)]
    x = norm(hs[-1], tolist(glob["norm"]))
    return hs, matvec(tolist(glob["output"]), x)


def test_tiny_model_matches_scalar_bruteforce():
    glob, layers = _tiny_weights()
    toks = S.make_tokens(5, 1, 8, TINY.vocab)[0].tolist()
    hs_ref, logits_ref = _scalar_model(glob, layers, toks)
    m = O.OracleModel(TINY, glob, layers, batch=1)
    taps = []
    nxt, logits = m.prefill(np.array([toks]), taps)
    np.testing.assert_allclose(taps[-1][0], np.array(hs_ref), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(logits[0], np.array(logits_ref), rtol=1e-12, atol=1e-14)
    assert nxt[0] == int(np.argmax(logits_ref))


def test_kv_cached_decode_equals_full_recompute():
    glob, layers = _tiny_weights()
    toks = S.make_tokens(6, 2, 11, TINY.vocab)
    full = O.OracleModel(TINY, glob, layers, batch=2)
    _, lg_full = full.prefill(toks)
    inc = O.OracleModel(TINY, glob, layers, batch=2)
    inc.prefill(toks[:, :7])
    for t in range(7, 11):
        _, lg = inc.decode(toks[:, t])
    np.testing.assert_allclose(lg, lg_full, rtol=1e-12, atol=1e-12)
    for l in range(TINY.n_layers):
        for b in range(2):
            np.testing.assert_allclose(inc.K[l][b], full.K[l][b], atol=1e-12)


def test_changing_future_tokens_leaves_past_outputs_unchanged():
    glob, layers = _tiny_weights()
    toks = S.make_tokens(8, 1, 10, TINY.vocab).numpy()
    alt = toks.copy()
    alt[0, 6:] = (alt[0, 6:] + 17) % TINY.vocab
    ta, tb = [], []
    O.OracleModel(TINY, glob, layers, 1).prefill(toks, ta)
    O.OracleModel(TINY, glob, layers, 1).prefill(alt, tb)
    for a, b in zip(ta, tb):
        np.testing.assert_array_equal(a[:, :6], b[:, :6])
        assert not np.array_equal(a[:, 6:], b[:, 6:])


# ---------------------------------------------------------------- page-printed shapes
def test_page_printed_llama3_8b_shapes():
    gold = json.load(open(os.path.join(GOLDEN, "page_shapes.json")))
    p = gold["llama3_8b_params"]
    wl = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape
    assert (wl.dim, wl.n_layers, wl.n_heads, wl.n_kv_heads, wl.vocab) == \
        (p["dim"], p["n_layers"], p["n_heads"], p["n_kv_heads"], p["vocab_size"])
    assert wl.norm_eps == p["norm_eps"] and wl.rope_theta == p["rope_theta"]
    assert wl.head_dim == p["dim"] // p["n_heads"]
    shapes = gold["llama3_8b_layer0_weight_shapes"]
    lw = S.make_layer_weights(wl.replace(ffn_hidden=8), 0, 0)     # tiny FFN keeps this cheap
    for k in ("wq", "wk", "wv", "wo"):
        assert list(lw[k].shape) == shapes[k]
    # The walkthrough's per-head view and per-token query: head h owns rows h*128 .. h*128+127 of wq.
    T = gold["prompt_tokens"]
    emb = np.random.default_rng(0).standard_normal((T, p["dim"])) * 0.02
    assert list(emb.shape) == gold["token_embeddings_shape"]
    x = O.rmsnorm(emb, O.f64(lw["attention_norm"]), p["norm_eps"])
    assert list(x.shape) == gold["normed_embeddings_shape"]
    wq = O.f64(lw["wq"])
    view = wq.reshape(p["n_heads"], wl.head_dim, p["dim"])
    assert list(view.shape) == gold["wq_per_head_view_shape"]
    assert list(view[0].shape) == gold["wq_head0_shape"]
    q0 = x @ view[0].T
    assert list(q0.shape) == gold["q_per_token_shape"]
    # The oracle's full projection, split into heads, agrees with the per-head view.
    np.testing.assert_allclose((x @ wq.T).reshape(T, p["n_heads"], wl.head_dim)[:, 0, :], q0, rtol=1e-12)


def test_page_printed_tiny_config():
    gold = json.load(open(os.path.join(GOLDEN, "page_shapes.json")))["stories15m_params"]
    w = S.WORKLOADS["tiny-llama2-f32-d288-b1-p8-g50"]
    assert (w.shape.dim, w.shape.n_layers, w.shape.n_heads, w.shape.vocab, w.shape.max_seq_len,
            w.decode_steps) == (gold["dim"], gold["n_layers"], gold["n_heads"], gold["vocab_size"],
                                gold["max_seq_len"], gold["max_new_tokens"])


# ---- bf16 storage emulation ---------------------------------------------------
def test_round_bf16_definition():
    """Nearest value with an 8-bit significand, ties to even; against the definition,
    hand-worked ties, the half-ulp bound, and torch's float32 -> bfloat16 cast."""
    r = O.round_bf16
    exact = np.array([0.0, 1.0, -1.5, 3.25, 2.0 ** -20, -(2.0 ** 30), 1 + 2.0 ** -7])
    assert np.array_equal(r(exact), exact)
    # ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> even significand (1.0);
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6 -> 1 + 2^-6
    assert r(1 + 2.0 ** -8) == 1.0
    assert r(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert r(-(1 + 2.0 ** -8)) == -1.0
    assert r(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7   # just above the tie
    rng = np.random.default_rng(7)
    x = rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))
    y = r(x)
    assert np.all(np.abs(y - x) <= 2.0 ** -8 * np.abs(x))           # half an ulp
    m, _ = np.frexp(y)
    assert np.all(np.ldexp(m, 8) == np.rint(np.ldexp(m, 8)))         # 8 significant bits
    x32 = x.astype(np.float32)
    ref = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(r(x32.astype(np.float64)), ref)


def test_bf16_emulation_rounds_where_stated_and_stays_close():
    shape = S.ModelShape(dim=64, n_layers=2, n_heads=4, n_kv_heads=2, head_dim=16, ffn_hidden=96,
                         vocab=50, max_seq_len=32, norm_eps=1e-5, rope_theta=10000.0, dtype="bf16",
                         tie_embeddings=False)
    glob, layers = S.make_weights(shape, 11)
    tok = S.make_tokens(11, 2, 9, shape.vocab).numpy()
    plain = O.OracleModel(shape, glob, layers, 2)
    emu = O.OracleModel(shape, glob, layers, 2, bf16_activations=True)
    same = O.OracleModel(shape, glob, layers, 2, bf16_activations=False)
    tp, te, ts = [], [], []
    _, lp = plain.prefill(tok, tp)
    _, le = emu.prefill(tok, te)
    _, ls = same.prefill(tok, ts)
    assert np.array_equal(lp, ls) and all(np.array_equal(a, b) for a, b in zip(tp, ts))
    for l in range(shape.n_layers):
        for b in range(2):
            assert np.array_equal(O.round_bf16(emu.K[l][b]), emu.K[l][b])
            assert np.array_equal(O.round_bf16(emu.V[l][b]), emu.V[l][b])
            assert not np.array_equal(O.round_bf16(plain.K[l][b]), plain.K[l][b])
        d = np.linalg.norm(te[l] - tp[l]) / np.linalg.norm(tp[l])
        assert 1e-5 < d < 1e-2, d
    d = np.linalg.norm(le - lp) / np.linalg.norm(lp)
    assert 1e-5 < d < 1e-2, d


def test_bf16_rounding_points_round_only_where_named():
    """Each named storage point rounds its own value and nothing else: the cache
    holds bf16 values exactly when k (or v) is named, and every point alone moves
    the result by a small, nonzero amount; the forced set is every point but q."""
    assert O.BF16_FORCED == O.BF16_POINTS - {"q"}
    shape = S.ModelShape(dim=64, n_layers=2, n_heads=4, n_kv_heads=2, head_dim=16, ffn_hidden=96,
                         vocab=50, max_seq_len=32, norm_eps=1e-5, rope_theta=10000.0, dtype="bf16",
                         tie_embeddings=False)
    glob, layers = S.make_weights(shape, 13)
    tok = S.make_tokens(13, 1, 7, shape.vocab).numpy()
    plain = O.OracleModel(shape, glob, layers, 1)
    _, lp = plain.prefill(tok)
    logits = {}
    for p in sorted(O.BF16_POINTS):
        m = O.OracleModel(shape, glob, layers, 1, rounding={p})
        _, logits[p] = m.prefill(tok)
        for l in range(shape.n_layers):
            for cache, name in ((m.K[l][0], "k"), (m.V[l][0], "v")):
                assert np.array_equal(O.round_bf16(cache), cache) == (p == name), (p, name)
        d = np.linalg.norm(logits[p] - lp) / np.linalg.norm(lp)
        assert 1e-6 < d < 1e-2, (p, d)
    for a in logits:
        for b in logits:
            if a < b:
                assert not np.array_equal(logits[a], logits[b]), (a, b)
    with pytest.raises(AssertionError):
        O.OracleModel(shape, glob, layers, 1, rounding={"w"})
