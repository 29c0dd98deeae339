"""The Python binding refuses mismatched operands before anything launches.

The kernels receive raw pointers and derive every size from the other
arguments (q's element size and row count for k and v, M and the head counts
for the outputs).  A k in another dtype than q, or an output smaller than the
call writes, would be read or written past its end on the device, so the
binding checks dtype, shape, device and contiguity of every tensor it is given
first.  These checks run on CPU tensors here: the error must name the
mismatch, not the missing CUDA device, which shows it comes before any launch.
"""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg

M, HQ, HKV, D = 12, 4, 2, 16
CU = np.array([0, 5, 12], np.int32)


def _attn(dtype=torch.bfloat16):
    q = torch.zeros(M, HQ, D, dtype=dtype)
    k = torch.zeros(M, HKV, D, dtype=dtype)
    v = torch.zeros(M, HKV, D, dtype=dtype)
    ls = torch.zeros(M)
    g, t = torch.zeros(HQ), torch.ones(HQ)
    return q, k, v, ls, g, t


def _raises(match, fn, *a, **kw):
    with pytest.raises(ValueError, match=match) as e:
        fn(*a, **kw)
    assert "CUDA tensors only" not in str(e.value)


def test_attention_rejects_mismatched_operands():
    q, k, v, ls, g, t = _attn()
    _raises("k: dtype", tg.gated_attention, q, k.float(), v, CU, ls, g, t)
    _raises("v: dtype", tg.gated_attention, q, k, v.float(), CU, ls, g, t)
    _raises("k: shape", tg.gated_attention, q, k[:-1], v, CU, ls, g, t)
    _raises("v: shape", tg.gated_attention, q, k, torch.zeros(M, HKV, D // 2,
                                                              dtype=q.dtype), CU, ls, g, t)
    _raises("logsig: shape", tg.gated_attention, q, k, v, CU, ls[:-1], g, t)
    _raises("gain: dtype", tg.gated_attention, q, k, v, CU, ls, g.double(), t)
    _raises("out: shape", tg.gated_attention, q, k, v, CU, ls, g, t, out=q[:-1])
    _raises("out: dtype", tg.gated_attention, q, k, v, CU, ls, g, t, out=q.float())
    _raises("lse: shape", tg.gated_attention, q, k, v, CU, ls, g, t,
            lse=torch.zeros(HQ, M - 1))
    _raises("k must be contiguous", tg.gated_attention, q, k.transpose(1, 2).contiguous()
            .transpose(1, 2), v, CU, ls, g, t)
    _raises("cu_kept_host ends", tg.gated_attention, q, k, v, np.array([0, 5, 11]), ls, g, t)
    _raises("workspace", tg.gated_attention, q, k, v, CU, ls, g, t,
            workspace=torch.zeros(64, dtype=torch.int32))
    _raises("multiple", tg.gated_attention, q, torch.zeros(M, 3, D, dtype=q.dtype),
            torch.zeros(M, 3, D, dtype=q.dtype), CU, ls, g, t)


def test_backward_rejects_mismatched_operands():
    q, k, v, ls, g, t = _attn()
    out, lse, dout = torch.zeros_like(q), torch.zeros(HQ, M), torch.zeros_like(q)
    bwd = tg.gated_attention_backward
    _raises("k: dtype", bwd, q, k.float(), v, CU, ls, g, t, out, lse, dout)
    _raises("dout: shape", bwd, q, k, v, CU, ls, g, t, out, lse, dout[:-1])
    _raises("out: dtype", bwd, q, k, v, CU, ls, g, t, out.float(), lse, dout)
    _raises("lse: shape", bwd, q, k, v, CU, ls, g, t, out, lse.T.contiguous(), dout)
    _raises("log-gates", bwd, q, k, v, CU, None, g, t, out, lse, dout)


def test_delta_scan_rejects_mismatched_operands():
    q = torch.zeros(M, 2, 64, dtype=torch.float32)
    la, be = torch.zeros(M, 2), torch.zeros(M, 2)
    _raises("k: dtype", tg.gated_delta_scan, q, q.bfloat16(), q, CU, la, be)
    _raises("v: dtype", tg.gated_delta_scan, q, q, q.bfloat16(), CU, la, be)
    _raises("out: shape", tg.gated_delta_scan, q, q, q, CU, la, be, out=q[:-1])
    _raises("out: dtype", tg.gated_delta_scan, q, q, q, CU, la, be, out=q.bfloat16())
    _raises("state: shape", tg.gated_delta_scan, q, q, q, CU, la, be,
            state=torch.zeros(2, 2, 64, 32))
    _raises("state: dtype", tg.gated_delta_scan, q, q, q, CU, la, be,
            state=torch.zeros(2, 2, 64, 64, dtype=torch.float64))
    _raises("cu_kept_host ends", tg.gated_delta_scan, q, q, q, np.array([0, 5]), la, be)


def test_gate_select_gather_and_stack_reject_mismatches():
    h = torch.zeros(CU[-1], 64, dtype=torch.bfloat16)
    W1 = torch.zeros(32, 64, dtype=torch.bfloat16)
    b1, w2 = torch.zeros(32), torch.zeros(32)
    _raises("b1: shape", tg.gate_score, h, W1, b1[:-1], w2, 0.0)
    _raises("out: dtype", tg.gate_score, h, W1, b1, w2, 0.0, out=torch.zeros(CU[-1],
                                                                             dtype=torch.float64))
    _raises("out: shape", tg.gate_score, h, W1, b1, w2, 0.0, out=torch.zeros(CU[-1] - 1))
    s, e, K = [0, 0], [3, 5], [1, 2]
    z = torch.zeros(int(CU[-1]))
    _raises("z: shape", tg.topk_select, z[:-1], CU, s, e, K)
    _raises("kept_idx: shape", tg.topk_select, z, CU, s, e, K,
            kept_idx=torch.zeros(3, dtype=torch.int32))
    kept = torch.zeros(8, dtype=torch.int32)
    _raises("tensors\\[1\\]: shape", tg.compact_gather, kept, CU, s, e, K, [h, h[:-1]])
    _raises("outs\\[0\\]: shape", tg.compact_gather, kept, CU, s, e, K, [h],
            outs=[torch.zeros(7, 64, dtype=h.dtype)])
    _raises("z: dtype", tg.compact_gather, kept, CU, s, e, K, [h], z=z.double())
    x = torch.zeros(5, 64)
    _raises("weight: shape", tg.rmsnorm, x, torch.zeros(32))
    _raises("out: shape", tg.swiglu, torch.zeros(5, 64), out=torch.zeros(5, 31))
