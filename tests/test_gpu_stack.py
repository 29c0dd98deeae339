"""GPU parity of the gated upper-layer stack (RMSNorm, QKV split with per-head
norm, RoPE and KV emission, SwiGLU, and the whole stack) against the fp64
oracle (oracle/stack.py) on the same bf16 inputs.

Error budget: each step stores bf16 (rounding <= 2^-9 relative, one unit in the
last place 2^-8 to 2^-7); the single steps are checked to two bf16 units.  The
whole stack rounds the residual and eight intermediates per layer, and the
cuBLAS GEMMs accumulate in fp32; the outputs and the caches are checked per
element to 2e-2 of their rms value plus 2e-2 of the element (the budget of ~16
independent 2^-9 roundings of the typical magnitude, with margin)."""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from learned_token_pruning_gate_b200.pipeline import GatedStack
from oracle import stack as so
from tests.parity_utils import assert_close, dev, host_f32

pytestmark = pytest.mark.gpu
ULP2 = 2.0 ** -7


def _kept_idx(cu_kept, pos, pos_span):
    """Global row ids of the kept rows: prompt b spans pos_span * M_b tokens."""
    lens = np.diff(cu_kept)
    starts = np.concatenate([[0], np.cumsum(pos_span * lens)])[:-1]
    prompt = np.repeat(np.arange(len(lens)), lens)
    cu_seq = np.concatenate([[0], np.cumsum(pos_span * lens)]).astype(np.int32)
    return (starts[prompt] + pos).astype(np.int32), cu_seq


def test_rmsnorm_and_swiglu():
    rng = np.random.default_rng(1)
    x = torch.from_numpy(rng.standard_normal((257, 384), dtype=np.float32) * 3).bfloat16()
    w = torch.from_numpy(1 + 0.1 * rng.standard_normal(384, dtype=np.float32)).bfloat16()
    got = tg.rmsnorm(dev(x), dev(w), 1e-6)
    ref = so.rmsnorm(host_f32(x), host_f32(w), 1e-6)
    assert_close("rmsnorm", host_f32(got), ref, 1e-6, ULP2)
    gu = torch.from_numpy(rng.standard_normal((130, 2 * 200), dtype=np.float32) * 4).bfloat16()
    got = tg.swiglu(dev(gu))
    g, u = host_f32(gu)[:, :200], host_f32(gu)[:, 200:]
    assert_close("swiglu", host_f32(got), so.silu(g) * u, 1e-5, ULP2)


@pytest.mark.parametrize("lens,Hq,Hkv,dh", [([300, 0, 129], 4, 2, 64), ([512], 16, 8, 128)])
def test_qkv_rope_emit(lens, Hq, Hkv, dh):
    cu, pos, x0, ls, layers = gen.stack_inputs(lens, 1, 256, Hq, Hkv, dh, 64, 5, "bf16")
    kept, cu_seq = _kept_idx(cu, pos, 4)
    M = int(cu[-1])
    rng = np.random.default_rng(2)
    qkv = torch.from_numpy(rng.standard_normal((M, (Hq + 2 * Hkv) * dh), dtype=np.float32)).bfloat16()
    ly = layers[0]
    q, k, v = tg.qkv_rope_emit(dev(qkv), cu_seq, cu, dev(torch.from_numpy(kept)), Hq, Hkv, dh,
                               dev(ly["w_qn"]), dev(ly["w_kn"]), 1e-6, 1e6)
    a = host_f32(qkv)
    rq = so.rope(so.rmsnorm(a[:, :Hq * dh].reshape(M, Hq, dh), host_f32(ly["w_qn"])), pos, 1e6)
    rk = so.rope(so.rmsnorm(a[:, Hq * dh:(Hq + Hkv) * dh].reshape(M, Hkv, dh), host_f32(ly["w_kn"])),
                 pos, 1e6)
    assert_close("q", host_f32(q), rq, ULP2, ULP2)
    assert_close("k", host_f32(k), rk, ULP2, ULP2)
    assert torch.equal(v.cpu().view(torch.int16),
                       qkv[:, (Hq + Hkv) * dh:].reshape(M, Hkv, dh).contiguous().view(torch.int16))


@pytest.mark.parametrize("lens,n_layers,dm,Hq,Hkv,dh,inter", [
    ([300, 0, 129], 2, 256, 4, 2, 64, 512),      # small Qwen-like
    ([512], 1, 2048, 16, 8, 128, 6144),         # Qwen3-1.7B-shaped layer
])
def test_stack_matches_oracle(lens, n_layers, dm, Hq, Hkv, dh, inter):
    cu, pos, x0, ls, layers = gen.stack_inputs(lens, n_layers, dm, Hq, Hkv, dh, inter, 7, "bf16")
    kept, cu_seq = _kept_idx(cu, pos, 4)
    dlayers = [{k: dev(v) for k, v in ly.items()} for ly in layers]
    st = GatedStack(dlayers, Hq, Hkv, dh, cu_seq, cu, dev(torch.from_numpy(kept)), dev(ls))
    x, ck, cv = st.run(dev(x0).clone())
    torch.cuda.synchronize()
    assert tg.device_status() == 0
    lay = [{k: host_f32(v).astype(np.float64) for k, v in ly.items()} for ly in layers]
    rx, rk, rv = so.stack(host_f32(x0), pos, cu, ls.numpy(), lay, Hq, Hkv, dh)
    # per element |gpu - ref| <= 2e-2 rms + 2e-2 |ref|: bf16 storage of every
    # intermediate (x, the projections, q/k/v) and bf16 GEMM inputs put errors of
    # a few bf16 units of the typical magnitude on every element, independent of
    # the element's own size (measured need at rtol 2e-2: <= 1.3e-2 rms)
    for name, got, ref in [("x", x, rx), ("cache_k", ck, rk), ("cache_v", cv, rv)]:
        ref = np.asarray(ref, np.float64)
        g = host_f32(got).astype(np.float64).reshape(ref.shape)
        rms = np.sqrt(np.mean(ref * ref))
        assert_close(name, g, ref, 2e-2 * rms, 2e-2)
