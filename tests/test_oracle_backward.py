"""Pins of the oracle's attention backward (the gradient path that trains the
gate through the attention bias).  The analytic fp64 gradient is checked
against central finite differences of the oracle's own fp64 loss, and against
identities that hold for any input:
  - each query row's softmax weights sum to 1, so the gradient of the logits of
    one row sums to 0; hence the log-gate gradients of a prompt sum to 0 when
    every head has the same gain, and the gain gradient vanishes when every key
    of a prompt has the same log-gate;
  - a prompt of one kept row has a single key with weight 1: no gradient.
"""
import numpy as np
import pytest

import oracle


def _case(lens, Hq=4, Hkv=2, dh=8, seed=0, const_l=False):
    rng = np.random.default_rng(seed)
    M = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = rng.standard_normal((M, Hq, dh)).astype(np.float32)
    k = rng.standard_normal((M, Hkv, dh)).astype(np.float32)
    v = rng.standard_normal((M, Hkv, dh)).astype(np.float32)
    dout = rng.standard_normal((M, Hq, dh)).astype(np.float32)
    l = np.full(M, -0.7) if const_l else np.log(1 / (1 + np.exp(-rng.standard_normal(M) * 2)))
    g = rng.uniform(0.2, 1.0, Hq)
    t = rng.uniform(0.8, 1.2, Hq)
    return q, k, v, cu, l, g, t, dout


def test_backward_matches_central_differences():
    q, k, v, cu, l, g, t, dout = _case([5, 9, 1, 12], seed=3)
    d_l, d_g, d_t = oracle.gated_attention_backward(q, k, v, cu, l, g, t, dout)
    loss = lambda l_, g_, t_: oracle.attention_loss(q, k, v, cu, l_, g_, t_, dout)  # noqa: E731
    eps = 1e-5
    fd_l = np.array([(loss(l + eps * e, g, t) - loss(l - eps * e, g, t)) / (2 * eps)
                     for e in np.eye(len(l))])
    fd_g = np.array([(loss(l, g + eps * e, t) - loss(l, g - eps * e, t)) / (2 * eps)
                     for e in np.eye(len(g))])
    fd_t = np.array([(loss(l, g, t + eps * e) - loss(l, g, t - eps * e)) / (2 * eps)
                     for e in np.eye(len(t))])
    for name, a, f in [("d_logsig", d_l, fd_l), ("d_gain", d_g, fd_g), ("d_temp", d_t, fd_t)]:
        scale = np.abs(f).max()
        assert scale > 1e-3, name  # a non-trivial gradient
        np.testing.assert_allclose(a, f, rtol=0, atol=1e-7 * max(scale, 1.0), err_msg=name)


def test_backward_identities():
    lens = [7, 1, 11]
    q, k, v, cu, l, g, t, dout = _case(lens, seed=5)
    # equal gains: the log-gate gradients of every prompt sum to zero
    g_eq = np.full_like(g, 0.6)
    d_l, _, _ = oracle.gated_attention_backward(q, k, v, cu, l, g_eq, t, dout)
    for b in range(len(lens)):
        assert abs(d_l[cu[b]:cu[b + 1]].sum()) < 1e-10
    # the one-row prompt has no gradient at all
    assert d_l[cu[1]] == 0.0
    # equal log-gates: the gain gradient vanishes
    q, k, v, cu, l, g, t, dout = _case(lens, seed=6, const_l=True)
    _, d_g, d_t = oracle.gated_attention_backward(q, k, v, cu, l, g, t, dout)
    assert np.abs(d_g).max() < 1e-10
    assert np.abs(d_t).max() > 1e-3


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_plants_a_mistake(seed):
    """A dropped term must be caught: the gradient of the temperature without its
    1/tau factor differs from the finite difference."""
    q, k, v, cu, l, g, t, dout = _case([9, 6], seed=seed)
    t = t * 1.7  # far from 1, so a missing 1/tau shows
    _, _, d_t = oracle.gated_attention_backward(q, k, v, cu, l, g, t, dout)
    eps = 1e-5
    fd = np.array([(oracle.attention_loss(q, k, v, cu, l, g, t + eps * e, dout)
                    - oracle.attention_loss(q, k, v, cu, l, g, t - eps * e, dout)) / (2 * eps)
                   for e in np.eye(len(t))])
    np.testing.assert_allclose(d_t, fd, atol=1e-7 * np.abs(fd).max())
    assert np.abs(d_t * t - fd).max() > 1e-3 * np.abs(fd).max()


def test_loss_is_the_forward_inner_product(oracle):
    """The loss that the finite differences differentiate is tied to the pinned
    forward: L = sum(dout * out) with out from the oracle's gated attention (whose
    own pins fix the bias sign, the temperature's place and the GQA map).  A
    mistake in the loss's private attention row -- a flipped bias, the
    temperature on the bias, a wrong kv head -- would keep the analytic and
    numerical gradients consistent with each other, but not with this."""
    q, k, v, cu, l, g, t, dout = _case([5, 9, 1, 12, 3], Hq=6, Hkv=2, dh=8, seed=11)
    # the forward takes float32 log-gates, gains and temperatures: use values
    # that float32 holds exactly, so both sides see the same numbers
    l, g, t = (np.asarray(a, np.float32).astype(np.float64) for a in (l, g * 1.5, t * 1.4))
    out, _ = oracle.gated_attention(q, k, v, cu, logsig=l, gain=g, temp=t)
    terms = dout.astype(np.float64) * out
    ref = float(terms.sum())
    got = oracle.attention_loss(q, k, v, cu, l, g, t, dout)
    assert abs(got - ref) <= 1e-12 * np.abs(terms).sum(), (got, ref)
