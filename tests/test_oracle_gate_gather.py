"""Pins for the oracle's gate scorer, compaction, RoPE and log-sigmoid (CPU only).

Gate (pages: "at layer L a small MLP scores each token from its post-attention
residual"): z = w2 . GELU(W1 h + b1) + b2 with the exact GELU.  Compaction
(pages: "layers above L process only the kept tokens and create no KV entry for
the dropped ones"): kept rows are copied; q and k are rotated at their original
positions; each kept document key carries l = log sigmoid(z).

Independent references used here: scipy's normal CDF, torch's float64 linear /
GELU / logsigmoid, numpy complex exponentials, and closed-form properties.
"""
import numpy as np
import pytest
import scipy.stats
import torch
import torch.nn.functional as F

from learned_token_pruning_gate_b200 import inputs as gen


def test_gate_closed_form_identity_slice(oracle):
    rng = np.random.default_rng(0)
    n, d, dg = 64, 32, 8
    h = rng.standard_normal((n, d)).astype(np.float32) * 3
    W1 = np.zeros((dg, d), np.float32)
    W1[np.arange(dg), np.arange(dg)] = 1.0
    w2 = np.zeros(dg, np.float32)
    w2[0] = 1.0
    z = oracle.gate_score(h, W1, np.zeros(dg), w2, 0.0)
    x = h[:, 0].astype(np.float64)
    np.testing.assert_allclose(z, x * scipy.stats.norm.cdf(x), rtol=1e-13, atol=1e-14)


def test_gate_matches_torch_float64(oracle):
    inp = gen.make_inputs(gen.scaled(gen.WORKLOADS["tiny_fp32"], 4), with_qkv=False)
    h, W1 = inp.f32("h"), inp.f32("W1")
    z = oracle.gate_score(h, W1, inp.b1.numpy(), inp.w2.numpy(), inp.b2)
    t = torch.from_numpy
    a = F.linear(t(h).double(), t(W1).double(), inp.b1.double())
    ref = F.gelu(a, approximate="none") @ inp.w2.double() + inp.b2
    np.testing.assert_allclose(z, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_gate_linear_in_output_layer(oracle):
    rng = np.random.default_rng(1)
    n, d, dg = 40, 48, 16
    h = rng.standard_normal((n, d)).astype(np.float32)
    W1 = (rng.standard_normal((dg, d)) * 0.3).astype(np.float32)
    b1 = (rng.standard_normal(dg) * 0.1).astype(np.float32)
    wa = rng.standard_normal(dg).astype(np.float32)
    wb = rng.standard_normal(dg).astype(np.float32)
    za = oracle.gate_score(h, W1, b1, wa, 0.25)
    zb = oracle.gate_score(h, W1, b1, wb, -0.5)
    zab = oracle.gate_score(h, W1, b1, (wa.astype(np.float64) + wb).astype(np.float32), -0.25)
    # wa + wb is exact in fp32 only up to rounding; compare with the rounded sum's effect
    np.testing.assert_allclose(zab, za + zb, rtol=1e-6, atol=1e-6)


def test_gate_row_subset(oracle):
    rng = np.random.default_rng(2)
    h = rng.standard_normal((100, 16)).astype(np.float32)
    W1 = rng.standard_normal((8, 16)).astype(np.float32)
    b1, w2 = rng.standard_normal(8).astype(np.float32), rng.standard_normal(8).astype(np.float32)
    full = oracle.gate_score(h, W1, b1, w2, 0.1)
    rows = np.array([99, 0, 57, 57])
    np.testing.assert_array_equal(oracle.gate_score(h, W1, b1, w2, 0.1, rows=rows), full[rows])


def _rope_complex(x, pos, theta):
    """RoPE as multiplication of (x_i + i x_{i+d/2}) by exp(i pos theta^(-2i/d))."""
    d = x.shape[-1]
    half = d // 2
    freq = np.power(np.float64(theta), -np.arange(half, dtype=np.float64) * 2.0 / d)
    zc = (x[..., :half].astype(np.float64) + 1j * x[..., half:].astype(np.float64))
    zc = zc * np.exp(1j * np.outer(pos, freq))[:, None, :]
    return np.concatenate([zc.real, zc.imag], axis=-1)


def test_gather_plain_rows_are_copies(oracle):
    rng = np.random.default_rng(3)
    src = rng.standard_normal((50, 3, 8)).astype(np.float32)
    kept = np.array([0, 3, 4, 20, 21, 49], np.int32)
    out = oracle.gather_rows(kept, [0, 20, 50], src)
    np.testing.assert_array_equal(out, src[kept].astype(np.float64))


@pytest.mark.parametrize("dh,theta", [(64, 1e6), (128, 1e6), (128, 1e4)])
def test_rope_matches_complex_rotation(oracle, dh, theta):
    rng = np.random.default_rng(dh)
    lens = [700, 131072 - 700]
    cu = np.array([0, 700, 131072], np.int32)
    kept = np.sort(rng.choice(131072, size=300, replace=False)).astype(np.int32)
    src = rng.standard_normal((131072, 2, dh)).astype(np.float32)
    out = oracle.gather_rows(kept, cu, src, rope_heads=2, head_dim=dh, theta=theta)
    pos = np.where(kept < 700, kept, kept - 700)
    ref = _rope_complex(src[kept], pos, theta)
    # fp64 angles near 1.3e5 rad carry ~1e-11 rad of rounding; allow a few times that
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-9)
    assert lens[0] + lens[1] == 131072


def test_rope_properties(oracle):
    rng = np.random.default_rng(5)
    dh = 64
    src = rng.standard_normal((1000, 1, dh)).astype(np.float32)
    kept = np.arange(1000, dtype=np.int32)
    out = oracle.gather_rows(kept, [0, 1000], src, rope_heads=1, head_dim=dh)
    # position 0 is the identity; pair norms are preserved
    np.testing.assert_array_equal(out[0], src[0].astype(np.float64))
    half = dh // 2
    n_in = src[..., :half].astype(np.float64) ** 2 + src[..., half:].astype(np.float64) ** 2
    n_out = out[..., :half] ** 2 + out[..., half:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)
    # relative-position property: <R(p)a, R(p')b> depends on p - p' only
    a = np.repeat(src[3:4], 1000, 0)
    b = np.repeat(src[8:9], 1000, 0)
    ra = oracle.gather_rows(kept, [0, 1000], a, rope_heads=1, head_dim=dh)[:, 0]
    rb = oracle.gather_rows(kept, [0, 1000], b, rope_heads=1, head_dim=dh)[:, 0]
    d1 = np.dot(ra[100], rb[40])
    d2 = np.dot(ra[560], rb[500])
    assert abs(d1 - d2) < 1e-9


def test_logsig_matches_torch_and_protects_question(oracle):
    z = gen.random_scores(600, seed=11, specials=False) * 20
    z[:4] = [0.0, 80.0, -80.0, 1e-30]
    cu = np.array([0, 250, 600], np.int32)
    s, e = np.array([0, 50], np.int32), np.array([200, 350], np.int32)
    kept = np.arange(600, dtype=np.int32)
    ls = oracle.logsig(kept, cu, s, e, z)
    ref = F.logsigmoid(torch.from_numpy(z).double()).numpy()
    pos = np.where(kept < 250, kept, kept - 250)
    b = (kept >= 250).astype(int)
    is_doc = (pos >= s[b]) & (pos < e[b])
    np.testing.assert_allclose(ls[is_doc], ref[is_doc], rtol=1e-14, atol=1e-300)
    assert np.all(ls[~is_doc] == 0.0)
    assert ls[0] == pytest.approx(-np.log(2.0), rel=1e-15)
    assert ls[2] == pytest.approx(-80.0, rel=1e-15)
