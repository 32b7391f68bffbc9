"""The library's LZW allocation (l3_lzw_allocate, host code) against the
plain-Python oracle of kimjy99 review, 1. Embedding Allocation: the same d_t,
bit for bit, and the same number of codewords."""
import numpy as np
import pytest

import static_token_routed_b200 as l3
from oracle import lzw_allocation as lzw


def test_hand_worked_corpus():
    d, nw = l3.l3_lzw_allocate([0, 1, 0, 1, 0, 1], vocab=3, v=10, k=9)
    assert d.tolist() == [5, 4, 1] and nw == 6


@pytest.mark.parametrize("seed", range(12))
def test_matches_oracle_on_zipf_corpora(seed):
    rng = np.random.default_rng(100 + seed)
    vocab = int(rng.integers(1, 300))
    n = int(rng.integers(0, 3000))
    p = 1.0 / np.arange(1, vocab + 1) ** float(rng.uniform(0.8, 1.4))
    corpus = rng.choice(vocab, size=n, p=p / p.sum()).astype(np.int32)
    if seed % 3 == 0 and n > 10:  # repeated stretches: long matched suffixes
        corpus[n // 2:n // 2 + n // 4] = corpus[:n // 4]
    order, _ = lzw.build_codewords(corpus)
    ends = {c[-1] for c in order}
    k = int(rng.integers(1, 40))
    top = vocab + (k - 1) * len(ends)
    v = int(rng.integers(vocab, top + 1))
    d, nw = l3.l3_lzw_allocate(corpus, vocab, v, k)
    assert nw == len(order)
    assert d.tolist() == lzw.allocate(corpus, vocab, v, k)


def test_errors():
    with pytest.raises(l3.L3Error):
        l3.l3_lzw_allocate([0, 5], vocab=3, v=3, k=2)       # token out of range
    with pytest.raises(l3.L3Error):
        l3.l3_lzw_allocate([0, 1], vocab=3, v=2, k=2)       # v < vocab
    with pytest.raises(l3.L3Error):
        l3.l3_lzw_allocate([0, 1], vocab=3, v=7, k=2)       # v > vocab * k
    with pytest.raises(l3.L3Error):
        l3.l3_lzw_allocate([0, 0, 0], vocab=3, v=6, k=2)    # only token 0 ends codewords
    d, nw = l3.l3_lzw_allocate([], vocab=4, v=4, k=3)        # empty corpus, one row each
    assert d.tolist() == [1, 1, 1, 1] and nw == 0
