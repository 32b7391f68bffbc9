"""The seeded input generator: allocation constraints and determinism (no GPU).

papernotes (LZW 信息论 embedding 分配) and the kimjy99 review (Embedding
Allocation): every token gets at least one and at most k embeddings, and the
d_t sum to the budget v.
"""
import numpy as np
import pytest
import torch

from static_token_routed_b200 import workloads as wl


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_allocation_constraints(name):
    w = wl.WORKLOADS[name]
    d = wl.allocation(w)
    assert len(d) == w.vocab
    assert d.min() >= 1 and d.max() <= w.k
    assert int(d.sum()) == w.v
    off = wl.offsets_from_allocation(d)
    assert off[0] == 0 and off[-1] == w.v and np.all(np.diff(off) >= 1)


def test_zipf_allocation_shape():
    """Near-Zipf: the most frequent IDs sit at the cap and most IDs get one
    row (sciencestack Fig. 5 histogram)."""
    w = wl.WORKLOADS["paper_shaped"]
    d = wl.allocation(w)
    assert d[0] == w.k and np.all(np.diff(d) <= 0)
    assert np.mean(d == 1) > 0.5


def test_dense64_and_uniform_allocations():
    d = wl.allocation(wl.WORKLOADS["dense_stress"])
    assert np.all(d[:64] == 512) and set(np.unique(d[64:])) <= {2, 3}
    d = wl.allocation(wl.WORKLOADS["uniform"])
    assert np.all(d == 4)


def test_ids_and_determinism():
    w = wl.WORKLOADS["tiny_fp32"]
    a, b = wl.make_batch(w), wl.make_batch(w)
    assert torch.equal(a.ids, b.ids) and torch.equal(a.x, b.x)
    assert a.ids.dtype == torch.int32 and a.ids.min() >= 0 and a.ids.max() < w.vocab
    dec = wl.make_batch(wl.WORKLOADS["decode"])
    assert len(np.unique(dec.ids.numpy())) == 256
    t = wl.make_tables(w)
    assert t.W_mix.shape == (w.d_out, w.d_up + w.d_in) and t.W_K.dtype == torch.float32


def test_normal_tensor_independent_of_threads():
    a = wl.normal_tensor(3, "W_K", (3 * (1 << 24) // 1000 + 5, 1000), 0.5, torch.bfloat16, threads=1)
    b = wl.normal_tensor(3, "W_K", (3 * (1 << 24) // 1000 + 5, 1000), 0.5, torch.bfloat16, threads=8)
    assert torch.equal(a, b)
    assert abs(float(a.float().std()) - 0.5) < 0.01


def test_tied_tables_share_one_tensor():
    """A tied workload (one table as keys and values: the W_K / W_V tying
    row of the papernotes page's ablation table, 消融实验) hands out the same
    tensor twice."""
    import dataclasses
    w = dataclasses.replace(wl.WORKLOADS["paper_tied"], vocab=300, v=1200, k=16, n_tokens=64)
    t = wl.make_tables(w)
    assert t.W_V is t.W_K and t.W_K.shape == (1200, 512)
    with pytest.raises(ValueError):
        wl.make_tables(dataclasses.replace(w, d_emb=256))


def test_zipf_corpus_is_seeded_and_in_range():
    a = wl.zipf_corpus(500, 20000, seed=3)
    b = wl.zipf_corpus(500, 20000, seed=3)
    assert a.dtype == np.int32 and len(a) == 20000 and np.array_equal(a, b)
    assert a.min() >= 0 and a.max() < 500
    assert not np.array_equal(a, wl.zipf_corpus(500, 20000, seed=4))
    # frequent IDs come first (Zipf ranks)
    counts = np.bincount(a, minlength=500)
    assert counts[:5].sum() > counts[-100:].sum()
