"""Pins of the gated-delta-rule oracle (oracle/delta.py) to facts outside its own code.

- The step-by-step recurrence equals the unrolled closed form, a unit lower-triangular
  solve: two independent statements of the gated delta rule.
- Exact associative memory: with alpha = beta = 1 and orthonormal keys the state is
  sum_t v_t k_t^T, and querying key s returns v_s (scaled by 1/sqrt(d_k)).
- The delta rule overwrites: writing a second value under the same key replaces the first.
- alpha = 0 forgets everything before t; beta = 0 writes nothing.
- Prompts are independent: a batch equals its prompts run one by one.
"""
import numpy as np
import pytest

from oracle import delta


def _inputs(lens, H=3, dk=16, dv=8, seed=0, decay=0.5):
    rng = np.random.default_rng(seed)
    M = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = rng.standard_normal((M, H, dk))
    k = rng.standard_normal((M, H, dk))
    v = rng.standard_normal((M, H, dv))
    la = -rng.uniform(0.0, decay, (M, H))
    be = rng.uniform(0.0, 1.0, (M, H))
    return q, k, v, la, be, cu


@pytest.mark.parametrize("lens,decay", [([37], 0.5), ([10, 0, 27, 1], 0.5), ([64], 3.0), ([50], 0.0)])
def test_recurrence_equals_closed_form(lens, decay):
    q, k, v, la, be, cu = _inputs(lens, decay=decay)
    o1, s1 = delta.scan(q, k, v, la, be, cu)
    o2, s2 = delta.scan_closed_form(q, k, v, la, be, cu)
    assert np.allclose(o1, o2, rtol=1e-10, atol=1e-12)
    assert np.allclose(s1, s2, rtol=1e-10, atol=1e-12)


def test_orthonormal_keys_are_an_exact_memory():
    dk, dv, T = 16, 8, 12
    rng = np.random.default_rng(1)
    k = np.zeros((T, 1, dk))
    k[np.arange(T), 0, np.arange(T)] = 3.0  # e_t, any length (normalised in the layer)
    v = rng.standard_normal((T, 1, dv))
    s = 5
    q = np.zeros((T, 1, dk))
    q[:, 0, s] = 2.0  # every query asks for key s
    o, state = delta.scan(q, k, v, np.zeros((T, 1)), np.ones((T, 1)), [0, T], eps=0.0)
    assert np.allclose(state[0, 0], v[:, 0, :].T @ (k[:, 0, :] / 3.0), atol=1e-12)
    for t in range(T):
        want = v[s, 0] / np.sqrt(dk) if t >= s else np.zeros(dv)
        assert np.allclose(o[t, 0], want, atol=1e-12)


def test_same_key_overwrites():
    dk, dv = 16, 8
    rng = np.random.default_rng(2)
    kk = rng.standard_normal(dk)
    k = np.stack([kk, 0.5 * kk])[:, None, :]
    v = rng.standard_normal((2, 1, dv))
    q = rng.standard_normal((2, 1, dk))
    _, state = delta.scan(q, k, v, np.zeros((2, 1)), np.ones((2, 1)), [0, 2], eps=0.0)
    kh = kk / np.linalg.norm(kk)
    assert np.allclose(state[0, 0], np.outer(v[1, 0], kh), atol=1e-12)


def test_zero_alpha_forgets_and_zero_beta_writes_nothing():
    q, k, v, la, be, cu = _inputs([20], H=2)
    o, state = delta.scan(q, k, v, np.full_like(la, -np.inf), be, cu, eps=0.0)
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True) / np.sqrt(q.shape[-1])
    kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
    want = be[..., None] * v * np.sum(kn * qn, axis=-1, keepdims=True)
    assert np.allclose(o, want, atol=1e-12)
    assert np.allclose(state[0], (be[-1][:, None, None] * v[-1][:, :, None] * kn[-1][:, None, :]),
                       atol=1e-12)
    o0, s0 = delta.scan(q, k, v, la, np.zeros_like(be), cu)
    assert not o0.any() and not s0.any()


def test_prompts_are_independent():
    q, k, v, la, be, cu = _inputs([9, 14, 5], seed=3)
    o, state = delta.scan(q, k, v, la, be, cu)
    for b in range(3):
        r0, r1 = cu[b], cu[b + 1]
        ob, sb = delta.scan(q[r0:r1], k[r0:r1], v[r0:r1], la[r0:r1], be[r0:r1], [0, r1 - r0])
        assert np.array_equal(o[r0:r1], ob)
        assert np.array_equal(state[b], sb[0])



@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_chunked_form_equals_recurrence(chunk):
    """The chunk-by-chunk statement (the form a parallel kernel takes) agrees with the
    recurrence for chunks of one row, uneven chunks and chunks longer than a prompt."""
    q, k, v, la, be, cu = _inputs([37, 0, 50, 1], decay=1.0, seed=7)
    o1, s1 = delta.scan(q, k, v, la, be, cu)
    o2, s2 = delta.scan_chunked(q, k, v, la, be, cu, chunk=chunk)
    assert np.allclose(o1, o2, rtol=1e-10, atol=1e-12)
    assert np.allclose(s1, s2, rtol=1e-10, atol=1e-12)
