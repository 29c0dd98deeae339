"""GPU parity of the gated-attention backward (log-gates, gains, temperatures)
against the fp64 oracle gradient on the same inputs.

Error budget: the GPU takes D_i = dout_i . out_i from the forward's stored output
(bf16: each element rounded to 2^-9 relative) and the forward's fp32 LSE; every
other step is fp32.  The rounding of out moves D_i by up to 2^-9 sum|dout||out|,
which enters each log-gate gradient through sum_i P_ij delta(D_i); the bound is
taken as 2 % of the case's largest gradient for bf16 outputs and 0.1 % for fp32
outputs (whose D_i is exact to fp32 rounding).
"""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import dev, host_f32

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "fp32": 1e-3}  # of the case's largest |gradient|, per element


def _case(oracle, lens, Hq, Hkv, dh, dtype, algo, seed):
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, seed, dtype, True)
    M = int(cu[-1])
    dout = gen.attention_output_grad(M, Hq, dh, seed, dtype)
    qd, kd, vd, lsd, gd, td, dod = (dev(x) for x in (q, k, v, ls, gain, temp, dout))
    out, lse = tg.gated_attention(qd, kd, vd, cu, lsd, gd, td, want_lse=True)
    d_l, d_z, d_g, d_t = tg.gated_attention_backward(qd, kd, vd, cu, lsd, gd, td, out, lse, dod,
                                                     algo=algo)
    torch.cuda.synchronize()
    assert tg.device_status() == 0
    r_l, r_g, r_t = oracle.gated_attention_backward(
        host_f32(q), host_f32(k), host_f32(v), cu, ls.numpy().astype(np.float64),
        gain.numpy().astype(np.float64), temp.numpy().astype(np.float64), host_f32(dout))
    tol = TOL[dtype]
    for name, got, ref in [("d_logsig", d_l, r_l), ("d_gain", d_g, r_g), ("d_temp", d_t, r_t)]:
        got = got.cpu().numpy().astype(np.float64)
        scale = max(np.abs(ref).max(), 1e-30)
        err = np.abs(got - ref).max() / scale
        assert err <= tol, f"{name}: max error {err:.2e} of the largest gradient (tol {tol})"
    # dL/dz of the kept rows = dL/dl (1 - sigmoid(z)), sigmoid(z) = exp(l); 0 where l = 0
    r_z = r_l * (1.0 - np.exp(ls.numpy().astype(np.float64)))
    got_z = d_z.cpu().numpy().astype(np.float64)
    assert np.abs(got_z - r_z).max() <= tol * max(np.abs(r_l).max(), 1e-30)


@pytest.mark.parametrize("algo", [tg.ALGO_SIMT, tg.ALGO_AUTO])
@pytest.mark.parametrize("lens,Hq,Hkv,dh", [([300], 16, 8, 128), ([5, 0, 260, 1, 640], 4, 2, 64),
                                            ([129, 700], 12, 4, 128)])
def test_attention_backward_bf16(oracle, lens, Hq, Hkv, dh, algo):
    _case(oracle, lens, Hq, Hkv, dh, "bf16", algo, seed=sum(lens) + Hq)


@pytest.mark.parametrize("lens", [[320], [33, 100, 0, 257]])
def test_attention_backward_fp32(oracle, lens):
    _case(oracle, lens, 4, 2, 64, "fp32", tg.ALGO_AUTO, seed=sum(lens))


def test_attention_backward_full_size_16k(oracle):
    """The qwen_16k shape (one prompt kept to 2304 rows, 16/8 heads x 128)."""
    _case(oracle, [2304], 16, 8, 128, "bf16", tg.ALGO_AUTO, seed=11)
