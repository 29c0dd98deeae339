"""Pins for the oracle's top-K selector (CPU only).

The selector keeps, per prompt, the K highest-scoring document tokens plus
every question token (pages: "a top-K selector keeps the highest-scoring
tokens"; "only the document part of the prompt is pruned, the question is never
touched"; budget ``max_kept_prefill_tokens``).  The pins below do not restate
the oracle's sort: they enumerate subsets, call numpy's lexsort, or use
properties any correct selection must have.
"""
import itertools
import math

import numpy as np
import pytest

from learned_token_pruning_gate_b200 import inputs as gen


def _ranks_before(za, ia, zb, ib):
    """True when token a must be preferred over token b (written independently)."""
    if math.isnan(za) and math.isnan(zb):
        return ia < ib
    if math.isnan(za):
        return False
    if math.isnan(zb):
        return True
    return za > zb or (za == zb and ia < ib)


def _brute_force_topk(z, s, e, K):
    """The unique K-subset of the document in which every member beats every non-member."""
    doc = list(range(s, e))
    k = min(K, len(doc))
    winners = []
    for sub in itertools.combinations(doc, k):
        inside = set(sub)
        ok = all(_ranks_before(float(z[a]), a, float(z[b]), b)
                 for a in inside for b in doc if b not in inside)
        if ok:
            winners.append(sub)
    assert len(winners) == 1, "the total order must make the top-K set unique"
    return set(winners[0])


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_small(oracle, seed):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 11))
    z = rng.choice(np.array([0.5, -0.25, 0.0, -0.0, 1.0, np.nan, np.inf, -np.inf, 0.125],
                            np.float32), size=n)
    s = int(rng.integers(0, n + 1))
    e = int(rng.integers(s, n + 1))
    for K in range(0, e - s + 2):
        kept, cu_kept = oracle.topk_select(z, [0, n], [s], [e], [K])
        expect = _brute_force_topk(z, s, e, K) | set(range(0, s)) | set(range(e, n))
        assert list(kept) == sorted(expect)
        assert cu_kept.tolist() == [0, len(expect)]


def test_all_equal_scores_keep_lowest_indices(oracle):
    z = np.full(50, 0.3, np.float32)
    kept, _ = oracle.topk_select(z, [0, 50], [5], [45], [7])
    assert kept.tolist() == list(range(0, 5)) + list(range(5, 12)) + list(range(45, 50))


def test_signed_zero_ties_by_index(oracle):
    z = np.array([-0.0, 0.0, -0.0, 0.0, -1.0], np.float32)
    kept, _ = oracle.topk_select(z, [0, 5], [0], [5], [2])
    assert kept.tolist() == [0, 1]


def test_nan_only_when_forced(oracle):
    z = np.array([np.nan, -np.inf, np.nan, -3.0], np.float32)
    kept, _ = oracle.topk_select(z, [0, 4], [0], [4], [2])
    assert kept.tolist() == [1, 3]
    kept, _ = oracle.topk_select(z, [0, 4], [0], [4], [3])
    assert kept.tolist() == [0, 1, 3]


@pytest.mark.parametrize("n,K", [(100_000, 2048), (40_000, 1), (5_000, 4999)])
def test_against_numpy_lexsort(oracle, n, K):
    z = gen.random_scores(n, seed=n + K, specials=False)
    q = 256
    kept, cu_kept = oracle.topk_select(z, [0, n], [0], [n - q], [K])
    idx = np.arange(n - q)
    order = np.lexsort((idx, -z[: n - q].astype(np.float64)))  # by -z, then index
    expect = np.sort(np.concatenate([order[:K], np.arange(n - q, n)]))
    np.testing.assert_array_equal(kept, expect)
    assert cu_kept[-1] == min(K, n - q) + q


def test_varlen_batch_is_concatenation(oracle):
    lens = [300, 1, 77, 1024, 0, 500]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    z = gen.random_scores(int(cu[-1]), seed=7)
    s = [10, 0, 0, 100, 0, 0]
    e = [290, 1, 70, 1000, 0, 500]
    K = [50, 0, 100, 3, 5, 500]
    kept, cu_kept = oracle.topk_select(z, cu, s, e, K)
    for b in range(len(lens)):
        zb = z[cu[b]:cu[b + 1]]
        kb, _ = oracle.topk_select(zb, [0, lens[b]], [s[b]], [e[b]], [K[b]])
        got = kept[cu_kept[b]:cu_kept[b + 1]]
        np.testing.assert_array_equal(got, kb + cu[b])
        # the question is always a subset of the kept set and the count is M_b
        prot = set(range(0, s[b])) | set(range(e[b], lens[b]))
        assert prot <= set((got - cu[b]).tolist())
        assert len(got) == min(K[b], e[b] - s[b]) + len(prot)
        assert np.all(np.diff(got) > 0)


def test_invalid_arguments_rejected(oracle):
    z = np.zeros(10, np.float32)
    with pytest.raises(ValueError):
        oracle.topk_select(z, [0, 10], [0], [11], [1])
    with pytest.raises(ValueError):
        oracle.topk_select(z, [0, 10], [0], [5], [-1])


@pytest.mark.parametrize("name", ["tiny_fp32", "qwen_16k"])
def test_planted_needle_is_selected(oracle, name):
    w = gen.WORKLOADS[name]
    if w.total_tokens > 4096:
        w = gen.scaled(w, 8)  # same structure, 2048 tokens: keeps the CPU test quick
    inp = gen.make_inputs(w, with_qkv=False)
    z = oracle.gate_score(inp.f32("h"), inp.f32("W1"), inp.b1.numpy(), inp.w2.numpy(), inp.b2)
    for b in range(w.batch):
        rows = inp.needle_rows[b]
        doc = np.arange(inp.cu_seqlens[b] + inp.doc_begin[b], inp.cu_seqlens[b] + inp.doc_end[b])
        rest = np.setdiff1d(doc, rows)
        assert z[rows].min() > z[rest].max() + 1e-2
    kept, _ = oracle.topk_select(z.astype(np.float32), inp.cu_seqlens, inp.doc_begin,
                                 inp.doc_end, inp.budget)
    for rows in inp.needle_rows:
        assert set(rows.tolist()) <= set(kept.tolist())


def load_worked_example():
    import os

    path = os.path.join(os.path.dirname(__file__), "golden", "topk_worked_example.txt")
    scores, doc, cases = None, None, {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = line.split(":", 1)
        if key == "scores":
            scores = np.array([float(x) for x in val.split()], np.float32)
        elif key == "doc":
            doc = tuple(int(x) for x in val.split())
        else:
            cases[int(key[2:])] = [int(x) for x in val.split()]
    return scores, doc, cases


def test_worked_example(oracle):
    z, (s, e), cases = load_worked_example()
    for K, expect in cases.items():
        kept, _ = oracle.topk_select(z, [0, len(z)], [s], [e], [K])
        assert kept.tolist() == expect, K
