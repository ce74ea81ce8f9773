"""The token <-> text bridge (CPU).

The trained vocabulary file is not here. The pieces the pattern cuts text into
are pinned by the page's worked example (each printed token of its prompt is
one piece); the special-token ids by the page's list and the id it prepends;
the merging by hand-worked cases and, where the tiktoken package is installed,
by agreement with its independent BPE on a vocabulary trained here.
"""
import base64
import collections
import json
import os
import random

import pytest

from llama_decoder_forward_fwd_b200 import tokenizer as T

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_tokenizer.json"), encoding="utf-8"))


def _byte_vocab():
    return {bytes([i]): i for i in range(256)}


def _trained_vocab(corpus, n_merges, pattern=T.PATTERN):
    """A small byte-level BPE vocabulary: repeatedly add the most frequent adjacent pair."""
    import regex
    ranks = _byte_vocab()
    words = collections.Counter(m.group().encode() for m in regex.finditer(pattern, corpus))
    seqs = {w: [w[i:i + 1] for i in range(len(w))] for w in words}
    for _ in range(n_merges):
        pairs = collections.Counter()
        for w, c in words.items():
            s = seqs[w]
            for a, b in zip(s, s[1:]):
                pairs[a + b] += c
        pairs = {p: c for p, c in pairs.items() if p not in ranks}
        if not pairs:
            break
        best = max(sorted(pairs), key=lambda p: pairs[p])
        ranks[best] = len(ranks)
        for w in words:
            s, i, out = seqs[w], 0, []
            while i < len(s):
                if i + 1 < len(s) and s[i] + s[i + 1] == best:
                    out.append(best)
                    i += 2
                else:
                    out.append(s[i])
                    i += 1
            seqs[w] = out
    return ranks


CORPUS = ("the answer to the ultimate question of life, the universe, and everything is 42. "
          "The model reads the prompt, then predicts the next token again and again. "
          "Attention heads share keys and values; the cache keeps them for every position.\n" * 3)


def test_special_token_table_follows_the_printed_list():
    assert len(T.SPECIAL_TOKENS) == GOLD["n_special"] == len(set(T.SPECIAL_TOKENS))
    tok = T.Tokenizer(_byte_vocab())
    base = tok.n_vocab_base
    assert tok.special["<|begin_of_text|>"] == base
    assert tok.special["<|eot_id|>"] == base + 9
    assert tok.special["<|reserved_special_token_5|>"] == base + 10
    assert tok.special["<|reserved_special_token_250|>"] == base + 255
    assert tok.n_vocab == base + 256
    # with the real 128000-entry vocabulary the first special id is the 128000 the page prepends
    assert GOLD["vocab_base"] + T.SPECIAL_TOKENS.index("<|begin_of_text|>") == GOLD["token_ids"][0]
    assert GOLD["token_strings"][0] == "<|begin_of_text|>"


def test_pattern_cuts_the_printed_prompt_into_the_printed_tokens():
    tok = T.Tokenizer(_byte_vocab())
    pieces = tok.pieces(GOLD["prompt"])
    assert pieces == GOLD["token_strings"][1:]
    assert len(pieces) == len(GOLD["token_ids"]) - 1


def test_pattern_pieces():
    tok = T.Tokenizer(_byte_vocab())
    assert tok.pieces("I'm here, they'll see 12345 apples!!\n\n  end") == \
        ["I", "'m", " here", ",", " they", "'ll", " see", " ", "123", "45", " apples", "!!\n\n", " ", " end"]
    assert "".join(tok.pieces("mixed  spaces\tand\r\nbreaks ")) == "mixed  spaces\tand\r\nbreaks "


def test_merges_worked_by_hand():
    ranks = _byte_vocab()
    ranks.update({b"ab": 256, b"bc": 257, b"abc": 258, b"xyz": 259})
    tok = T.Tokenizer(ranks)
    assert tok.encode("abc") == [258]                 # the whole piece is an entry
    assert tok.encode("abcb") == [258, ord("b")]      # ab (256) before bc (257), then abc
    assert tok.encode("bcab") == [257, 256]           # bc and ab both merge, abc is never adjacent
    assert tok.encode("xyz") == [259]                 # whole piece, though no pair of it merges
    assert tok.encode("xyzx") == [ord("x"), ord("y"), ord("z"), ord("x")]


def test_special_tokens_only_where_allowed():
    tok = T.Tokenizer(_byte_vocab())
    text = "<|begin_of_text|>hi<|eot_id|>"
    assert tok.encode(text, allowed_special="all") == [256, ord("h"), ord("i"), 256 + 9]
    plain = tok.encode(text)
    assert 256 not in plain and tok.decode(plain) == text
    assert tok.encode("hi", bos=True) == [256, ord("h"), ord("i")]
    assert tok.decode([256, ord("h")]) == "<|begin_of_text|>h"


def test_round_trip_on_random_text():
    tok = T.Tokenizer(_trained_vocab(CORPUS, 120))
    assert tok.decode(tok.encode(GOLD["round_trip_text"])) == GOLD["round_trip_text"]   # the page's own check
    rng = random.Random(0)
    alphabet = "abcdefghij ,.!?'\n\t0123456789ÄéßñЖ中文😀 " + "the answer "
    for _ in range(200):
        s = "".join(rng.choice(alphabet) for _ in range(rng.randint(0, 60)))
        assert tok.decode(tok.encode(s)) == s


def test_vocabulary_file_format(tmp_path):
    ranks = _trained_vocab(CORPUS, 30)
    p = tmp_path / "tokenizer.model"
    p.write_bytes(b"".join(base64.b64encode(b) + b" " + str(r).encode() + b"\n" for b, r in ranks.items()))
    tok = T.Tokenizer.from_file(str(p))
    assert tok.ranks == ranks and tok.n_vocab_base == len(ranks)
    with pytest.raises(ValueError):
        T.Tokenizer({b"a": 0, b"b": 2})


def test_agrees_with_tiktoken():
    tiktoken = pytest.importorskip("tiktoken")
    ranks = _trained_vocab(CORPUS, 200)
    ours = T.Tokenizer(ranks)
    ref = tiktoken.Encoding(name="trained-here", pat_str=T.PATTERN, mergeable_ranks=ranks,
                            special_tokens=dict(ours.special))
    rng = random.Random(1)
    words = CORPUS.split(" ") + ["42", "!!", "\n", "  ", "Ж", "😀", "<|eot_id|>"]
    for _ in range(300):
        s = " ".join(rng.choice(words) for _ in range(rng.randint(0, 25)))
        assert ours.encode(s, allowed_special="all") == ref.encode(s, allowed_special="all"), s
        assert ours.encode_ordinary(s) == ref.encode_ordinary(s), s
