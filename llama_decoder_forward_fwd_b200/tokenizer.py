"""Token <-> text bridge for the Llama-3 tokenizer format (byte-level BPE).

What "Building llama3 from scratch" sets up in its tokenizer section:

- a vocabulary file, ``tokenizer.model``, of 128000 (token bytes, rank) pairs,
  one per line as the base64 of the bytes and the rank; the rank is the token
  id;
- 256 special tokens numbered after the vocabulary, in the order the page lists
  them: begin and end of text, four reserved ones, start and end of a header
  id, a fifth reserved one, end of turn, then reserved tokens 5 to 250 (so
  ``<|begin_of_text|>`` is 128000, the id the page prepends to its prompt);
- a regular expression that cuts text into pieces before any merging:
  contractions, letter runs with at most one leading non-letter, runs of one to
  three digits, punctuation runs with an optional leading space, line breaks
  and other whitespace. The page prints it with its backslashes lost (``p{L}``
  for the letter class); here they are restored.

Encoding a piece: if its bytes are a vocabulary entry it is one token;
otherwise it starts as single bytes and the adjacent pair whose concatenation
has the lowest rank is merged, again and again, until no adjacent pair forms a
vocabulary entry; the ids are the ranks of the parts. Special tokens in the
text become their ids where the caller allows them, else they are plain text.
Decoding joins the ids' bytes and reads them as UTF-8.
"""
from __future__ import annotations

import base64
from typing import Dict, Iterable, List, Sequence, Union

import regex

PATTERN = (r"(?i:'s|'t|'re|'ve|'m|'ll|'d)|[^\r\n\p{L}\p{N}]?\p{L}+|\p{N}{1,3}| ?[^\s\p{L}\p{N}]+[\r\n]*"
           r"|\s*[\r\n]+|\s+(?!\S)|\s+")

SPECIAL_TOKENS: List[str] = [
    "<|begin_of_text|>", "<|end_of_text|>",
    "<|reserved_special_token_0|>", "<|reserved_special_token_1|>",
    "<|reserved_special_token_2|>", "<|reserved_special_token_3|>",
    "<|start_header_id|>", "<|end_header_id|>",
    "<|reserved_special_token_4|>", "<|eot_id|>",
] + [f"<|reserved_special_token_{i}|>" for i in range(5, 251)]


def read_ranks(path: str) -> Dict[bytes, int]:
    """The vocabulary file: one ``base64(token bytes) rank`` pair per line."""
    ranks: Dict[bytes, int] = {}
    with open(path, "rb") as f:
        for n, line in enumerate(f, 1):
            line = line.strip()
            if not line:
                continue
            parts = line.split()
            if len(parts) != 2:
                raise ValueError(f"{path}:{n}: expected 'base64 rank'")
            ranks[base64.b64decode(parts[0])] = int(parts[1])
    return ranks


class Tokenizer:
    def __init__(self, ranks: Dict[bytes, int], special_tokens: Sequence[str] = SPECIAL_TOKENS,
                 pattern: str = PATTERN):
        ids = sorted(ranks.values())
        if ids != list(range(len(ranks))):
            raise ValueError("ranks must be 0 .. n-1, each once")
        self.ranks = dict(ranks)
        self.n_vocab_base = len(ranks)
        self.special = {tok: self.n_vocab_base + i for i, tok in enumerate(special_tokens)}
        self.id_bytes: Dict[int, bytes] = {r: b for b, r in ranks.items()}
        for tok, i in self.special.items():
            self.id_bytes[i] = tok.encode()
        self._pieces = regex.compile(pattern)
        self._special_re = regex.compile("|".join(regex.escape(t) for t in sorted(self.special, key=len,
                                                                                    reverse=True)))

    @classmethod
    def from_file(cls, path: str, **kw) -> "Tokenizer":
        return cls(read_ranks(path), **kw)

    @property
    def n_vocab(self) -> int:
        return self.n_vocab_base + len(self.special)

    def _merge(self, piece: bytes) -> List[int]:
        r = self.ranks.get(piece)
        if r is not None:
            return [r]
        parts = [piece[i:i + 1] for i in range(len(piece))]
        while len(parts) > 1:
            best, at = None, -1
            for i in range(len(parts) - 1):
                rr = self.ranks.get(parts[i] + parts[i + 1])
                if rr is not None and (best is None or rr < best):
                    best, at = rr, i
            if best is None:
                break
            parts[at:at + 2] = [parts[at] + parts[at + 1]]
        try:
            return [self.ranks[p] for p in parts]
        except KeyError as e:
            raise ValueError(f"byte {e.args[0]!r} has no rank: the vocabulary must hold every single byte") from None

    def encode_ordinary(self, text: str) -> List[int]:
        """Ids of text with no special tokens recognised."""
        out: List[int] = []
        for m in self._pieces.finditer(text):
            out += self._merge(m.group().encode("utf-8"))
        return out

    def encode(self, text: str, allowed_special: Union[str, Iterable[str]] = (), bos: bool = False) -> List[int]:
        """Ids of text; special-token strings listed in allowed_special (or all of
        them, with "all") become their ids; bos prepends <|begin_of_text|>."""
        allowed = set(self.special) if allowed_special == "all" else set(allowed_special)
        out: List[int] = [self.special["<|begin_of_text|>"]] if bos else []
        start = 0
        if allowed:
            for m in self._special_re.finditer(text):
                if m.group() not in allowed:
                    continue
                out += self.encode_ordinary(text[start:m.start()])
                out.append(self.special[m.group()])
                start = m.end()
        return out + self.encode_ordinary(text[start:])

    def decode_bytes(self, ids: Iterable[int]) -> bytes:
        try:
            return b"".join(self.id_bytes[int(i)] for i in ids)
        except KeyError as e:
            raise ValueError(f"token id {e.args[0]} out of range") from None

    def decode(self, ids: Iterable[int]) -> str:
        return self.decode_bytes(ids).decode("utf-8", errors="replace")

    def pieces(self, text: str) -> List[str]:
        """The pieces the pattern cuts text into (before any merging)."""
        return [m.group() for m in self._pieces.finditer(text)]
