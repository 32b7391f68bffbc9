"""The LZW allocation with its codeword walk on the GPU
(l3_lzw_allocate_device; kimjy99 review, 1. Embedding Allocation) against
the plain-Python oracle and the host entry point, bit for bit: the same d_t
for every token and the same number of codewords. The cases cover a walk
that ends inside a pass, one that ends exactly at the end of a complete
pass, several complete passes, k = 1, an empty corpus and the unreachable
budget."""
from collections import Counter

import numpy as np
import pytest
import torch

import static_token_routed_b200 as l3
from oracle import lzw_allocation as lzw

pytestmark = pytest.mark.gpu


def device_alloc(corpus, vocab, v, k):
    d, nw = l3.l3_lzw_allocate_device(corpus, vocab, v, k)
    torch.cuda.synchronize()
    return d.cpu().numpy().tolist(), nw


def test_hand_worked_corpus():
    # codewords (0), (1), (1,0), (0,1), (1,0,1)... the oracle's pinned example
    assert device_alloc([0, 1, 0, 1, 0, 1], 3, 10, 9) == ([5, 4, 1], 6)


def zipf_corpus(seed, vocab, n, s):
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, vocab + 1) ** s
    c = rng.choice(vocab, size=n, p=p / p.sum()).astype(np.int32)
    if seed % 3 == 0 and n > 10:  # repeated stretches: long matched suffixes
        c[n // 2:n // 2 + n // 4] = c[:n // 4]
    return c


@pytest.mark.parametrize("seed", range(10))
def test_matches_oracle(seed):
    rng = np.random.default_rng(500 + seed)
    vocab = int(rng.integers(1, 400))
    n = int(rng.integers(0, 4000))
    corpus = zipf_corpus(seed, vocab, n, float(rng.uniform(0.8, 1.4)))
    order, _ = lzw.build_codewords(corpus)
    ends = {c[-1] for c in order}
    k = int(rng.integers(1, 40))
    top = vocab + (k - 1) * len(ends)
    v = int(rng.integers(vocab, top + 1))
    want = lzw.allocate(corpus, vocab, v, k)
    got, nw = device_alloc(corpus, vocab, v, k)
    assert nw == len(order)
    assert got == want


def test_walk_ending_at_a_complete_pass():
    """v equal to the rows after exactly two complete walks: no partial walk."""
    corpus = zipf_corpus(7, 300, 5000, 1.1)
    order, _ = lzw.build_codewords(corpus)
    k = 30
    cnt = Counter(c[-1] for c in order)
    v = sum(min(k, 1 + 2 * cnt.get(t, 0)) for t in range(300))
    want = lzw.allocate(corpus, 300, v, k)
    assert device_alloc(corpus, 300, v, k)[0] == want
    # one row more and one row less: inside the third and the second walk
    for dv in (1, -1):
        assert device_alloc(corpus, 300, v + dv, k)[0] == lzw.allocate(corpus, 300, v + dv, k)


def test_paper_sized_vocab_against_host():
    """The paper-shaped budget (|tau| = 180000, v = 710000, k = 512) on a
    200K-token synthetic corpus: the same d_t as the host walk."""
    from static_token_routed_b200 import workloads as wl
    corpus = wl.zipf_corpus(180000, 200_000, seed=2)
    want, nw_h = l3.l3_lzw_allocate(corpus, 180000, 710000, 512)
    got, nw = device_alloc(corpus, 180000, 710000, 512)
    assert nw == nw_h and got == want.tolist()
    assert sum(got) == 710000 and min(got) >= 1 and max(got) <= 512


def test_edge_cases():
    assert device_alloc([], 4, 4, 3) == ([1, 1, 1, 1], 0)          # empty corpus
    corpus = zipf_corpus(3, 50, 2000, 1.0)
    assert device_alloc(corpus, 50, 50, 1)[0] == [1] * 50          # k = 1
    order, _ = lzw.build_codewords(corpus)
    ends = {c[-1] for c in order}
    v = 50 + 6 * len(ends)                                          # every ending token at k
    assert device_alloc(corpus, 50, v, 7)[0] == lzw.allocate(corpus, 50, v, 7)
    with pytest.raises(l3.L3Error) as e:                            # out of reach
        l3.l3_lzw_allocate_device([0, 0, 0], 3, 6, 2)
    assert e.value.status == 1 and "out of reach" in str(e.value)
    with pytest.raises(l3.L3Error):                                 # token out of range
        l3.l3_lzw_allocate_device([0, 5], 3, 3, 2)
