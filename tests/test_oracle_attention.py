"""Pins for the oracle's token-gated causal GQA attention (CPU only).

Definition (pages: the kept tokens' gate scores become a bias on the attention
logits above the gate -- the Mixture-of-Experts router trick -- with a per-head
learned gain, and a per-head learned temperature compensates for each query
seeing fewer keys):

    logit_ij = q_i . k_j / (sqrt(d_h) tau_h) + g_h l_j,   j <= i within the prompt

Pins: reduction to ordinary causal softmax attention (torch SDPA, float64) when
g = 0 and tau = 1; closed forms when q = 0 or when every key is equal; the
temperature/scale equivalence; the single-key case; and the LSE closed form.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from learned_token_pruning_gate_b200 import inputs as gen


def _sdpa_reference(q, k, v, cu):
    """Plain causal GQA attention per prompt via torch's float64 SDPA."""
    outs = []
    G = q.shape[1] // k.shape[1]
    for b in range(len(cu) - 1):
        qs = torch.from_numpy(q[cu[b]:cu[b + 1]]).double().transpose(0, 1)
        ks = torch.from_numpy(k[cu[b]:cu[b + 1]]).double().repeat_interleave(G, 1).transpose(0, 1)
        vs = torch.from_numpy(v[cu[b]:cu[b + 1]]).double().repeat_interleave(G, 1).transpose(0, 1)
        o = F.scaled_dot_product_attention(qs[None], ks[None], vs[None], is_causal=True)[0]
        outs.append(o.transpose(0, 1).numpy())
    return np.concatenate(outs, 0)


@pytest.mark.parametrize("lens,Hq,Hkv,dh", [([37], 4, 2, 16), ([5, 64, 1, 130], 4, 1, 8),
                                             ([200], 2, 2, 64)])
def test_reduces_to_causal_attention(oracle, lens, Hq, Hkv, dh):
    cu, q, k, v, ls, _, _ = gen.attention_inputs(lens, Hq, Hkv, dh, seed=sum(lens), dtype="fp32")
    out, _ = oracle.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, logsig=ls.numpy(),
                                    gain=np.zeros(Hq), temp=np.ones(Hq))
    ref = _sdpa_reference(q.numpy(), k.numpy(), v.numpy(), cu)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_temperature_equals_query_scaling(oracle):
    lens, Hq, Hkv, dh = [90, 33], 4, 2, 32
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, seed=3, dtype="fp32")
    out, _ = oracle.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, logsig=None,
                                    gain=gain.numpy(), temp=temp.numpy())
    qs = (q.double() / temp.double()[None, :, None]).numpy()
    ref = _sdpa_reference(qs, k.numpy(), v.numpy(), cu)
    np.testing.assert_allclose(out, ref, rtol=1e-6, atol=1e-6)  # qs rounded to fp32 inside


def test_zero_query_closed_form(oracle):
    """q = 0: o_i = sum_j sigma_j^g v_j / sum_j sigma_j^g  (weights exp(g l_j))."""
    lens, Hq, Hkv, dh = [50, 20], 4, 2, 8
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, seed=4, dtype="fp32")
    q = torch.zeros_like(q)
    out, _ = oracle.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, logsig=ls.numpy(),
                                    gain=gain.numpy(), temp=temp.numpy())
    G = Hq // Hkv
    V = v.double().numpy()
    L = ls.double().numpy()
    for b in range(len(lens)):
        for i in range(cu[b], cu[b + 1]):
            for h in range(Hq):
                wgt = np.exp(gain[h].item() * L[cu[b]:i + 1])
                ref = (wgt[:, None] * V[cu[b]:i + 1, h // G]).sum(0) / wgt.sum()
                np.testing.assert_allclose(out[i, h], ref, rtol=1e-12, atol=1e-13)


def test_equal_keys_make_temperature_irrelevant_to_bias(oracle):
    """All keys equal => q.k_j is the same for every j, so only g l_j matters: tau must
    not divide the bias."""
    lens, Hq, Hkv, dh = [40], 2, 1, 16
    cu, q, k, v, ls, gain, _ = gen.attention_inputs(lens, Hq, Hkv, dh, seed=5, dtype="fp32")
    k = k[:1].expand_as(k).contiguous()
    gain = torch.tensor([0.7, 1.0])
    res = []
    for tau in ([1.0, 1.0], [0.5, 3.0]):
        out, _ = oracle.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, logsig=ls.numpy(),
                                        gain=gain.numpy(), temp=np.array(tau, np.float32))
        res.append(out)
    np.testing.assert_allclose(res[0], res[1], rtol=1e-12, atol=1e-13)
    wgt = np.exp(np.float64(np.float32(0.7)) * ls.double().numpy())
    i = 39
    ref = (wgt[:, None] * v.double().numpy()[:, 0]).sum(0) / wgt.sum()
    np.testing.assert_allclose(res[0][i, 0], ref, rtol=1e-12)


def test_first_row_sees_one_key_and_lse(oracle):
    lens, Hq, Hkv, dh = [10, 1, 7], 4, 2, 8
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, seed=6, dtype="fp32")
    out, lse = oracle.gated_attention(q.numpy(), k.numpy(), v.numpy(), cu, logsig=ls.numpy(),
                                      gain=gain.numpy(), temp=temp.numpy())
    for b in range(3):
        i = cu[b]
        for h in range(Hq):
            np.testing.assert_array_equal(out[i, h], v.numpy()[i, h // 2].astype(np.float64))
    # q = 0 and g = 0: every logit is 0, so lse_i = log(number of visible keys)
    out, lse = oracle.gated_attention(np.zeros_like(q.numpy()), k.numpy(), v.numpy(), cu)
    for b in range(3):
        for i in range(cu[b], cu[b + 1]):
            np.testing.assert_allclose(lse[i], np.log(i - cu[b] + 1), rtol=1e-14, atol=1e-15)


def test_row_subset_matches_full(oracle):
    lens, Hq, Hkv, dh = [64, 64], 4, 2, 16
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, seed=8, dtype="fp32")
    args = (q.numpy(), k.numpy(), v.numpy(), cu)
    kw = dict(logsig=ls.numpy(), gain=gain.numpy(), temp=temp.numpy())
    full, lse_full = oracle.gated_attention(*args, **kw)
    rows = np.array([127, 0, 64, 63])
    part, lse_part = oracle.gated_attention(*args, rows=rows, **kw)
    np.testing.assert_array_equal(part, full[rows])
    np.testing.assert_array_equal(lse_part, lse_full[rows])
