"""Pins of the fp64 oracle of the gated upper-layer stack (oracle/stack.py):
closed forms of its pieces, an independent reimplementation of the attention
step (the C oracle), RoPE invariants, and the identity the residual structure
gives when the output projections vanish."""
import math

import numpy as np
import pytest

import oracle
from learned_token_pruning_gate_b200 import inputs as gen
from oracle import stack as so


def test_rmsnorm_closed_form():
    w = np.linspace(0.5, 1.5, 8)
    for c in (-3.0, 0.25, 7.0):
        got = so.rmsnorm(np.full(8, c), w, eps=1e-6)
        np.testing.assert_allclose(got, w * c / math.sqrt(c * c + 1e-6), rtol=1e-14)


def test_silu_closed_form():
    for x in (-20.0, -1.5, 0.0, 0.3, 9.0):
        assert abs(so.silu(x) - x / (1.0 + math.exp(-x))) <= 1e-15 * max(1.0, abs(x))


def test_rope_invariants():
    rng = np.random.default_rng(0)
    d = 16
    q = rng.standard_normal((5, 2, d))
    k = rng.standard_normal((5, 2, d))
    pos = np.array([0, 3, 17, 250, 131071])
    r = so.rope(q, pos, 1e6)
    np.testing.assert_allclose(r[0], q[0], rtol=0, atol=1e-15)  # position 0: identity
    # each (i, i + d/2) pair keeps its length
    n = lambda a: a[..., : d // 2] ** 2 + a[..., d // 2:] ** 2  # noqa: E731
    np.testing.assert_allclose(n(r), n(q), rtol=1e-12)
    # scores depend only on the position difference
    for m, nn, t in [(3, 1, 5), (100, 40, 1000)]:
        a = (so.rope(q[:1], [m], 1e6) * so.rope(k[:1], [nn], 1e6)).sum(-1)
        b = (so.rope(q[:1], [m + t], 1e6) * so.rope(k[:1], [nn + t], 1e6)).sum(-1)
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-12)


def test_stack_attention_matches_c_oracle():
    cu, q, k, v, ls, gain, temp = gen.attention_inputs([7, 0, 30, 1], 4, 2, 16, 3, "fp32", True)
    ref, _ = oracle.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, ls.numpy(), gain.numpy(),
                                    temp.numpy())
    got = so.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, ls.numpy(), gain.numpy(),
                             temp.numpy())
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n_layers", [1, 3])
def test_stack_identity_without_output_projections(n_layers):
    """With Wo = 0 and Wd = 0 every layer adds nothing: x comes back unchanged, and
    each layer's cache holds RoPE(RMSNorm(K projection of RMSNorm(x0)))."""
    cu, pos, x0, ls, layers = gen.stack_inputs([40, 25], n_layers, 32, 4, 2, 8, 48, 9, "fp32")
    lay = [{k_: np.asarray(v_, np.float64) for k_, v_ in ly.items()} for ly in layers]
    for ly in lay:
        ly["wo"][:] = 0.0
        ly["wd"][:] = 0.0
    x, ck, cv = so.stack(x0.numpy(), pos, cu, ls.numpy(), lay, 4, 2, 8)
    np.testing.assert_array_equal(x, x0.numpy().astype(np.float64))
    for i, ly in enumerate(lay):
        a = so.rmsnorm(x0.numpy(), ly["w_ln1"])
        kp = (a @ ly["wqkv"].T)[:, 32:48].reshape(-1, 2, 8)
        np.testing.assert_allclose(ck[i], so.rope(so.rmsnorm(kp, ly["w_kn"]), pos, 1e6), rtol=1e-12)
        np.testing.assert_allclose(cv[i], (a @ ly["wqkv"].T)[:, 48:].reshape(-1, 2, 8), rtol=1e-12)


def _layer_step_by_step(so_mod):
    """One layer over one-row prompts, written out step by step.  A prompt of one
    kept row has a single key, whose softmax weight is exactly 1, so the
    attention output of query head h is the row's own v of kv head h // G,
    whatever the gate bias and temperature.  The rest of the layer then follows
    from its definition: the output projection added to the residual, RMSNorm
    (torch's float64 rms_norm) of that post-attention residual, the SwiGLU MLP
    SiLU(b Wg^T) * (b Wu^T) (torch's float64 silu) and the down projection added
    to the residual.  The weights are scaled up so that the MLP works in SiLU's
    curved region and the residual adds are far from negligible."""
    import torch
    import torch.nn.functional as F

    Hq, Hkv, d, dm, inter = 4, 2, 8, 32, 48
    cu, pos, x0, ls, layers = gen.stack_inputs([1] * 9, 1, dm, Hq, Hkv, d, inter, 17, "fp32")
    ly = {k_: np.asarray(v_, np.float64) for k_, v_ in layers[0].items()}
    for name in ("wqkv", "wo", "wg", "wu", "wd"):
        ly[name] = ly[name] * 25.0
    x0 = x0.numpy().astype(np.float64)
    x, ck, cv = so_mod.stack(x0, pos, cu, ls.numpy(), [ly], Hq, Hkv, d)

    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float64))  # noqa: E731
    a = F.rms_norm(t(x0), (dm,), t(ly["w_ln1"]), eps=1e-6).numpy()
    v = (a @ ly["wqkv"].T)[:, (Hq + Hkv) * d:].reshape(-1, Hkv, d)
    o = v[:, np.arange(Hq) // (Hq // Hkv)]  # one key: out = v of the head's kv head
    x1 = x0 + o.reshape(-1, Hq * d) @ ly["wo"].T
    b = F.rms_norm(t(x1), (dm,), t(ly["w_ln2"]), eps=1e-6).numpy()
    mid = F.silu(t(b @ ly["wg"].T)).numpy() * (b @ ly["wu"].T)
    x2 = x1 + mid @ ly["wd"].T
    assert np.abs(mid).max() > 0.5  # the MLP term is not negligible
    np.testing.assert_allclose(cv[0], v, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(x, x2, rtol=1e-12, atol=1e-12)


def test_stack_layer_step_by_step():
    _layer_step_by_step(so)


STACK_MUTATIONS = [
    # (name, [(original text, planted mistake)])
    ("ln2_on_pre_attention_x",
     [('a = rmsnorm(x, ly["w_ln1"], eps)', 'x_in = x\n        a = rmsnorm(x, ly["w_ln1"], eps)'),
      ('b = rmsnorm(x, ly["w_ln2"], eps)', 'b = rmsnorm(x_in, ly["w_ln2"], eps)')]),
    ("gate_up_swapped",
     [('silu(b @ np.asarray(ly["wg"], np.float64).T) * (b @ np.asarray(ly["wu"], np.float64).T)',
       'silu(b @ np.asarray(ly["wu"], np.float64).T) * (b @ np.asarray(ly["wg"], np.float64).T)')]),
    ("mlp_residual_dropped",
     [('x = x + hmid @ np.asarray(ly["wd"], np.float64).T',
       'x = hmid @ np.asarray(ly["wd"], np.float64).T')]),
    ("attention_residual_dropped",
     [('x = x + o.reshape(M, Hq * d) @ np.asarray(ly["wo"], np.float64).T',
       'x = o.reshape(M, Hq * d) @ np.asarray(ly["wo"], np.float64).T')]),
]


@pytest.mark.parametrize("name,edits", STACK_MUTATIONS, ids=[m[0] for m in STACK_MUTATIONS])
def test_stack_pin_catches_planted_mistake(tmp_path, name, edits):
    """Each planted mistake in a temporary copy of the stack oracle must fail the
    step-by-step pin (the committed file is never touched)."""
    import importlib.util
    import os

    src = open(os.path.join(os.path.dirname(so.__file__), "stack.py")).read()
    for old, new in edits:
        assert src.count(old) == 1, f"mutation {name}: text not found once in the stack oracle"
        src = src.replace(old, new)
    path = tmp_path / f"stack_{name}.py"
    path.write_text(src)
    spec = importlib.util.spec_from_file_location(f"stack_mut_{name}", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with pytest.raises(AssertionError):
        _layer_step_by_step(mod)
