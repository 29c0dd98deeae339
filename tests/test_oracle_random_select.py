"""Pins of the oracle's random-K selection (the pages' random-K selector
ablation): the K document tokens with the largest caller-drawn keys, lower
index on ties, question protected.  Checked against brute force, an
independent sort, special cases and the uniformity the ablation relies on."""
import itertools

import numpy as np

import oracle


def _one(keys, s, e, k):
    n = len(keys)
    kept, cu = oracle.select_by_keys(np.asarray(keys, np.uint32), [0, n], [s], [e], [k])
    assert cu.tolist() == [0, len(kept)]
    return kept.tolist()


def test_brute_force_small():
    """Every K-subset of a tiny document: the kept set is the unique subset
    whose every key beats (or ties with a larger index) every dropped key."""
    rng = np.random.default_rng(3)
    for trial in range(200):
        n = int(rng.integers(1, 9))
        s = int(rng.integers(0, n))
        e = int(rng.integers(s, n + 1))
        k = int(rng.integers(0, e - s + 2))
        keys = rng.integers(0, 4, n).astype(np.uint32)  # many ties on purpose
        got = set(_one(keys, s, e, k))
        doc = list(range(s, e))
        kk = min(k, len(doc))
        best = None
        for sub in itertools.combinations(doc, kk):
            rest = [j for j in doc if j not in sub]
            ok = all((keys[a] > keys[r]) or (keys[a] == keys[r] and a < r)
                     for a in sub for r in rest)
            if ok:
                assert best is None, "the order must make the kept set unique"
                best = set(sub)
        protected = set(range(0, s)) | set(range(e, n))
        assert got == best | protected


def test_matches_independent_sort():
    rng = np.random.default_rng(5)
    n, s, e, k = 5000, 100, 4900, 777
    keys = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
    keys[200:260] = keys[200]  # a block of equal keys
    order = np.lexsort((np.arange(s, e), -keys[s:e].astype(np.int64)))
    want = sorted(set((order[:k] + s).tolist()) | set(range(s)) | set(range(e, n)))
    assert _one(keys, s, e, k) == want


def test_special_cases():
    keys = np.full(10, 7, np.uint32)
    assert _one(keys, 2, 8, 3) == [0, 1, 2, 3, 4, 8, 9]        # equal keys: lowest indices
    assert _one(keys, 2, 8, 0) == [0, 1, 8, 9]                 # K = 0: question only
    assert _one(keys, 2, 8, 99) == list(range(10))             # K >= n_doc: everything
    keys = np.arange(10, dtype=np.uint32)
    assert _one(keys, 0, 10, 3) == [7, 8, 9]
    keys = np.array([0xFFFFFFFF, 0, 0x80000000, 1], np.uint32)  # full unsigned range
    assert _one(keys, 0, 4, 2) == [0, 2]


def test_varlen_batch_is_per_prompt():
    rng = np.random.default_rng(7)
    lens = [30, 0, 17, 50]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    keys = rng.integers(0, 2**32, cu[-1], dtype=np.uint64).astype(np.uint32)
    s, e, k = [3, 0, 0, 10], [25, 0, 17, 40], [5, 1, 20, 0]
    kept, cu_kept = oracle.select_by_keys(keys, cu, s, e, k)
    for b in range(4):
        part = kept[cu_kept[b]:cu_kept[b + 1]] - cu[b]
        one, _ = oracle.select_by_keys(keys[cu[b]:cu[b + 1]], [0, lens[b]], [s[b]], [e[b]], [k[b]])
        assert part.tolist() == one.tolist()


def test_uniform_keys_give_uniform_inclusion():
    """With i.i.d. uniform keys every document token is kept with probability
    K / n_doc (the ablation's premise): 4000 draws, each frequency within 5
    standard deviations."""
    rng = np.random.default_rng(11)
    n, s, e, k, draws = 40, 4, 36, 8, 4000
    counts = np.zeros(n)
    for _ in range(draws):
        keys = rng.integers(0, 2**32, n, dtype=np.uint64).astype(np.uint32)
        counts[_one(keys, s, e, k)] += 1
    p = k / (e - s)
    sd = np.sqrt(draws * p * (1 - p))
    assert np.all(np.abs(counts[s:e] - draws * p) < 5 * sd)
    assert np.all(counts[:s] == draws) and np.all(counts[e:] == draws)
