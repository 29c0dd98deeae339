"""GPU parity of the gated-attention backward (log-gates, gains, temperatures)
against the fp64 oracle gradient on the same inputs.

Error budget: the GPU takes D_i = dout_i . out_i from the forward's stored output
(bf16: each element rounded to 2^-9 relative) and the forward's fp32 LSE; every
other step is fp32.  The rounding of out moves D_i by up to 2^-9 sum|dout||out|,
which enters each log-gate gradient through sum_i P_ij delta(D_i): an error that
does not shrink with the entry's own size, so each element is held to
|gpu - ref| <= atol + rtol |ref| with atol a fraction of the case's largest
gradient and rtol catching scale errors on every entry.  Per quantity (bf16):
  d_logsig  atol 1e-3 max, rtol 1e-2 (measured need at that rtol: <= 4.3e-4 max)
  d_gain    atol 3e-3 max, rtol 2e-2 (measured <= 9.3e-4 max)
  d_temp    atol 1e-2 max, rtol 2e-2 (measured <= 6.8e-3 max: a sum of dlogit
            times q.k over every pair, the largest cancellation)
and fp32 outputs (D_i exact to fp32 rounding, measured errors <= 1.2e-6 max):
atol 1e-5 max, rtol 1e-4, for all three.
"""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import assert_close, dev, host_f32

pytestmark = pytest.mark.gpu

# (atol as a fraction of the case's largest |gradient|, rtol) per quantity
TOL = {"bf16": {"d_logsig": (1e-3, 1e-2), "d_gain": (3e-3, 2e-2), "d_temp": (1e-2, 2e-2)},
       "fp32": {"d_logsig": (1e-5, 1e-4), "d_gain": (1e-5, 1e-4), "d_temp": (1e-5, 1e-4)}}


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
    for name, got, ref in [("d_logsig", d_l, r_l), ("d_gain", d_g, r_g), ("d_temp", d_t, r_t)]:
        atol, rtol = TOL[dtype][name]
        assert_close(name, got.cpu().numpy(), ref, atol * max(np.abs(ref).max(), 1e-30), rtol)
    # dL/dz of the kept rows = dL/dl (1 - sigmoid(z)), sigmoid(z) = exp(l); 0 where l = 0
    r_z = r_l * (1.0 - np.exp(ls.numpy().astype(np.float64)))
    atol, rtol = TOL[dtype]["d_logsig"]
    assert_close("d_z_kept", d_z.cpu().numpy(), r_z, atol * max(np.abs(r_l).max(), 1e-30), rtol)


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
