"""Oracle of the LZW-based embedding allocation — test infrastructure.

Only `tests/` may import this module; the library never calls it.

The allocation decides d_t, the number of embedding rows of each token ID
(kimjy99 review, §1 Embedding Allocation; papernotes note, LZW 分配):

  1. Scan a token corpus and grow a set of codewords (token tuples) with a
     frequency each. At every position the codeword set is searched for the
     longest suffix of the text ending there; that suffix extended by one
     more token to the left is a suffix not seen before: it becomes a new
     codeword with frequency 1, and the suffix it extends (the new one minus
     its first token) gains 1.
  2. Walk the codewords from the most to the least frequent; a codeword
     that ends with token t gives t one embedding.
  3. Repeat the walk until the embeddings add up to the budget v; every
     token holds at least one embedding and at most k.

Readings where the pages are silent (listed in the design notes):
  - every token starts with its one guaranteed embedding, so the walk hands
    out v - |vocab| more;
  - codewords of equal frequency are walked in the order they were created;
  - a suffix never reaches back past the start of the corpus;
  - a token already at k is skipped by the walk.

Written as plain dictionaries and loops, for small corpora.
"""
from __future__ import annotations


def build_codewords(corpus) -> tuple[list[tuple[int, ...]], dict[tuple[int, ...], int]]:
    """Codewords in creation order, and their frequencies (step 1)."""
    freq: dict[tuple[int, ...], int] = {}
    order: list[tuple[int, ...]] = []
    tokens = [int(t) for t in corpus]
    for i in range(len(tokens)):
        # longest suffix ending at i that is already a codeword
        length = 0
        while length < i + 1 and tuple(tokens[i - length:i + 1]) in freq:
            length += 1
        if length == i + 1:
            # the whole text up to i is a codeword: nothing new can start here
            freq[tuple(tokens[0:i + 1])] += 1
            continue
        new = tuple(tokens[i - length:i + 1])
        freq[new] = 1
        order.append(new)
        if length > 0:
            freq[new[1:]] += 1
    return order, freq


def allocate(corpus, vocab: int, v: int, k: int) -> list[int]:
    """d_t for t in [0, vocab): steps 2-3."""
    if not (vocab <= v <= vocab * k):
        raise ValueError("need vocab <= v <= vocab * k")
    order, freq = build_codewords(corpus)
    # most frequent first; equal frequencies in creation order
    walk = sorted(range(len(order)), key=lambda j: (-freq[order[j]], j))
    d = [1] * vocab
    total = vocab
    while total < v:
        gave = False
        for j in walk:
            t = order[j][-1]
            if d[t] < k:
                d[t] += 1
                total += 1
                gave = True
                if total == v:
                    break
        if not gave:
            raise ValueError("every token that ends a codeword is at k; the budget cannot be met")
    return d
