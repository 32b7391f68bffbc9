"""Pins of the LZW allocation oracle (kimjy99 review, §1 Embedding Allocation):
hand-worked examples, closed forms and invariants that do not reuse the
oracle's own code."""
import numpy as np
import pytest

from oracle import lzw_allocation as lzw


def test_hand_worked_alternating_corpus():
    # a b a b a b with a = 0, b = 1 (worked by hand):
    #   pos 0: (a) new                pos 1: (b) new
    #   pos 2: (a) seen, (b a) new, (a) +1
    #   pos 3: (b) seen, (a b) new, (b) +1
    #   pos 4: (a), (b a) seen, (a b a) new, (b a) +1
    #   pos 5: (b), (a b) seen, (b a b) new, (a b) +1
    order, freq = lzw.build_codewords([0, 1, 0, 1, 0, 1])
    assert order == [(0,), (1,), (1, 0), (0, 1), (0, 1, 0), (1, 0, 1)]
    assert [freq[c] for c in order] == [2, 2, 2, 2, 1, 1]
    # walk: (a) (b) (b a) (a b) (a b a) (b a b), ending tokens 0 1 0 1 0 1;
    # token 2 never appears and keeps its one guaranteed embedding
    assert lzw.allocate([0, 1, 0, 1, 0, 1], vocab=3, v=6, k=3) == [3, 2, 1]
    assert lzw.allocate([0, 1, 0, 1, 0, 1], vocab=3, v=7, k=3) == [3, 3, 1]
    # v = 10, k = 9: one full walk gives 0 +3 and 1 +3 (total 9), the second
    # walk starts again at (a)
    assert lzw.allocate([0, 1, 0, 1, 0, 1], vocab=3, v=10, k=9) == [5, 4, 1]
    with pytest.raises(ValueError):  # tokens 0 and 1 at k, token 2 ends no codeword
        lzw.allocate([0, 1, 0, 1, 0, 1], vocab=3, v=8, k=3)


def test_repeated_token_closed_form():
    # t t t ... t (n times): position i adds the codeword of length i + 1 and
    # the one of length i is matched once more
    n = 9
    order, freq = lzw.build_codewords([5] * n)
    assert order == [(5,) * m for m in range(1, n + 1)]
    assert [freq[c] for c in order] == [2] * (n - 1) + [1]


def test_budget_edges():
    corpus = [0, 1, 2, 0, 1, 2, 2, 2]
    assert lzw.allocate(corpus, vocab=4, v=4, k=5) == [1, 1, 1, 1]
    with pytest.raises(ValueError):
        lzw.allocate(corpus, vocab=4, v=3, k=5)   # below one row per token
    with pytest.raises(ValueError):
        lzw.allocate(corpus, vocab=4, v=21, k=5)  # above k rows per token


def _suffix_trie_reference(tokens):
    """The same scan written on a reversed trie (node = codeword read from its
    last token backwards), as an independent check of step 1."""
    children = [{}]   # node 0 = root (empty suffix)
    count = [0]
    word = [()]
    order = []
    for i in range(len(tokens)):
        node, depth = 0, 0
        while depth <= i and tokens[i - depth] in children[node]:
            node = children[node][tokens[i - depth]]
            depth += 1
        if depth == i + 1:
            count[node] += 1
            continue
        new = len(children)
        children.append({})
        count.append(1)
        word.append(tuple(tokens[i - depth:i + 1]))
        children[node][tokens[i - depth]] = new
        order.append(new)
        if node != 0:
            count[node] += 1
    return [word[j] for j in order], {word[j]: count[j] for j in order}


@pytest.mark.parametrize("seed", range(6))
def test_scan_matches_a_reversed_trie_and_invariants(seed):
    rng = np.random.default_rng(seed)
    vocab = int(rng.integers(2, 40))
    n = int(rng.integers(1, 400))
    p = 1.0 / np.arange(1, vocab + 1) ** 1.1
    tokens = [int(t) for t in rng.choice(vocab, size=n, p=p / p.sum())]
    order, freq = lzw.build_codewords(tokens)
    ref_order, ref_freq = _suffix_trie_reference(tokens)
    assert order == ref_order and freq == ref_freq
    # suffix-closed: dropping a codeword's first token gives a codeword
    assert all(len(c) == 1 or c[1:] in freq for c in order)
    # frequencies: one per position, plus one per position that extended a
    # non-empty match into a new codeword
    extended = sum(1 for c in order if len(c) > 1)
    assert sum(freq.values()) == n + extended
    # the allocation meets the constraints whenever it can
    k = int(rng.integers(1, 12))
    cap = vocab + sum(min(k, 1 + 10 ** 9) - 1 for t in set(c[-1] for c in order))
    v = int(rng.integers(vocab, max(vocab, min(vocab * k, cap)) + 1))
    d = lzw.allocate(tokens, vocab, v, k)
    assert sum(d) == v and min(d) >= 1 and max(d) <= k
    # a token that ends no codeword keeps exactly one row
    ends = {c[-1] for c in order}
    assert all(d[t] == 1 for t in range(vocab) if t not in ends)
