"""GPU parity of the gated-delta-rule scan over the kept rows (tg_gated_delta_scan)
against the fp64 oracle (oracle/delta.py) on the same inputs.

Error budget: the kernel keeps the state in fp32 and upcasts the inputs exactly.
One step rounds ~3 d-term dot products and the update (relative 2^-24 per term);
the update map S -> alpha S (I - beta k k^T) has norm <= 1, so rounding errors do
not grow with the prompt length beyond their sum.  fp32 outputs and every state
are checked to 1e-4 absolute + 1e-3 relative; bf16 outputs, rounded once to bf16
(2^-9 relative), to 2e-3 absolute + 2^-7 relative (two bf16 units)."""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from oracle import delta as do
from tests.parity_utils import assert_close, dev, host_f32

pytestmark = pytest.mark.gpu

# Both forms compute the same function: the recurrence row by row
# (tg_gated_delta_scan) and the chunked scan (tg_gated_delta_scan_chunked).
ALGOS = ["recurrent", "chunked"]


@pytest.fixture(params=ALGOS)
def algo(request):
    return request.param


def _run(lens, H, d, dtype, seed, algo, decay=0.1):
    cu, q, k, v, la, beta = gen.delta_inputs(lens, H, d, seed, dtype, decay)
    o, state = tg.gated_delta_scan(dev(q), dev(k), dev(v), cu, dev(la), dev(beta), algo=algo)
    torch.cuda.synchronize()
    assert tg.device_status() == 0
    ro, rs = do.scan(host_f32(q), host_f32(k), host_f32(v), host_f32(la), host_f32(beta), cu)
    return host_f32(o), host_f32(state), ro, rs


@pytest.mark.parametrize("lens,H,d,dtype", [
    ([37, 0, 90, 1], 3, 64, "fp32"),
    ([300, 129], 4, 128, "fp32"),
    ([300, 129], 4, 128, "bf16"),
    ([1, 2, 255], 2, 64, "bf16"),
])
def test_delta_scan_matches_oracle(lens, H, d, dtype, algo):
    o, s, ro, rs = _run(lens, H, d, dtype, seed=11, algo=algo)
    if dtype == "fp32":
        assert_close("out", o, ro, 1e-4, 1e-3)
    else:
        assert_close("out", o, ro, 2e-3, 2.0 ** -7)
    assert_close("state", s, rs, 1e-4, 1e-3)


def test_delta_scan_strong_decay_and_no_write(algo):
    """alpha -> 0 (log_alpha = -inf): each output depends on its own row only;
    beta = 0: nothing is written, outputs and states are zero."""
    cu, q, k, v, la, beta = gen.delta_inputs([64, 33], 2, 128, 5, "fp32")
    la_inf = torch.full_like(la, -float("inf"))
    o, s = tg.gated_delta_scan(dev(q), dev(k), dev(v), cu, dev(la_inf), dev(beta), algo=algo)
    ro, rs = do.scan(host_f32(q), host_f32(k), host_f32(v), host_f32(la_inf), host_f32(beta), cu)
    assert_close("out", host_f32(o), ro, 1e-5, 1e-4)
    assert_close("state", host_f32(s), rs, 1e-5, 1e-4)
    o0, s0 = tg.gated_delta_scan(dev(q), dev(k), dev(v), cu, dev(la), dev(torch.zeros_like(beta)),
                                 algo=algo)
    torch.cuda.synchronize()
    assert not host_f32(o0).any() and not host_f32(s0).any()


def test_delta_scan_is_an_exact_memory_for_orthonormal_keys(algo):
    """alpha = beta = 1, keys e_t: querying key s returns v_s / sqrt(d) from row s on."""
    d, T, s = 64, 40, 7
    k = torch.zeros(T, 1, d)
    k[torch.arange(T), 0, torch.arange(T)] = 1.0
    v = torch.randn(T, 1, d, generator=torch.Generator().manual_seed(3))
    q = torch.zeros(T, 1, d)
    q[:, 0, s] = 1.0
    o, state = tg.gated_delta_scan(dev(q), dev(k), dev(v), [0, T], dev(torch.zeros(T, 1)),
                                   dev(torch.ones(T, 1)), eps=0.0, algo=algo)
    want = np.where(np.arange(T)[:, None] >= s, host_f32(v)[s, 0] / np.sqrt(d), 0.0)
    assert_close("out", host_f32(o)[:, 0], want, 1e-6, 1e-6)
    assert_close("state", host_f32(state)[0, 0], host_f32(v)[:, 0].T @ host_f32(k)[:, 0], 1e-6, 1e-6)


def test_delta_scan_full_size(algo):
    """The kept rows of the 16k workload (2304 rows, 16 heads of 128), bf16; every
    output and state against the oracle."""
    o, s, ro, rs = _run([2304], 16, 128, "bf16", seed=21, algo=algo, decay=0.05)
    assert_close("out", o, ro, 2e-3, 2.0 ** -7)
    assert_close("state", s, rs, 1e-4, 1e-3)


def test_delta_scan_empty_prompts_give_zero_state(algo):
    cu = [0, 0, 0]
    e = torch.empty(0, 2, 64, device="cuda")
    st = torch.full((2, 2, 64, 64), 7.0, device="cuda")
    tg.gated_delta_scan(e, e, e, cu, torch.empty(0, 2, device="cuda"), torch.empty(0, 2, device="cuda"),
                        state=st, algo=algo)
    torch.cuda.synchronize()
    assert not host_f32(st).any()


def test_delta_scan_rejects_unsupported_head_dim(algo):
    x = torch.zeros(4, 1, 96, device="cuda")
    with pytest.raises(tg.TokenGateError, match="TG_ERR_UNSUPPORTED"):
        tg.gated_delta_scan(x, x, x, [0, 4], torch.zeros(4, 1, device="cuda"),
                            torch.zeros(4, 1, device="cuda"), algo=algo)


def test_delta_scan_maximum_batch(algo):
    """TG_MAX_BATCH prompts of ragged lengths (0 to 40 rows): every prompt's state
    starts from zero and ends where the oracle says."""
    rng = np.random.default_rng(4)
    lens = [int(x) for x in rng.integers(0, 41, tg.MAX_BATCH)]
    o, s, ro, rs = _run(lens, 2, 64, "fp32", seed=12, algo=algo, decay=0.3)
    assert_close("out", o, ro, 1e-4, 1e-3)
    assert_close("state", s, rs, 1e-4, 1e-3)


def test_delta_scan_over_the_gated_layers_kept_rows(algo):
    """The layer consumes what the gated layer produces: the compacted q, k, v of a
    gated prefill (kept rows only, RoPE applied) as its inputs."""
    w = gen.scaled(gen.WORKLOADS["qwen_16k"], 8, name="delta_chain")
    inp = gen.make_inputs(w)
    r = tg.gated_prefill(*(dev(x) for x in (inp.h, inp.q, inp.k, inp.v, inp.W1, inp.b1, inp.w2)),
                         inp.b2, dev(inp.gain), dev(inp.temp), inp.cu_seqlens, inp.doc_begin,
                         inp.doc_end, inp.budget, rope_theta=w.rope_theta)
    ck = r["cu_kept_host"]
    M = int(ck[-1])
    H = r["k"].shape[1]
    rng = np.random.default_rng(5)
    la = torch.from_numpy(-rng.uniform(0.0, 0.1, (M, H)).astype(np.float32))
    beta = torch.from_numpy(rng.uniform(0.0, 1.0, (M, H)).astype(np.float32))
    q = r["q"][:, :H].contiguous()  # one query head per state head
    o, s = tg.gated_delta_scan(q, r["k"], r["v"], ck, dev(la), dev(beta), algo=algo)
    torch.cuda.synchronize()
    ro, rs = do.scan(host_f32(q), host_f32(r["k"]), host_f32(r["v"]), la.numpy(), beta.numpy(), ck)
    assert_close("out", host_f32(o), ro, 2e-3, 2.0 ** -7)
    assert_close("state", host_f32(s), rs, 1e-4, 1e-3)


def test_chunked_scan_chunk_boundaries_and_long_prompts():
    """Prompts that end exactly on, one before and one after a 64-row chunk
    boundary, a long prompt of many chunks with strong and weak decay mixed, and
    rows with alpha = 0 inside a chunk (the decay ratios across them are 0)."""
    lens = [64, 63, 65, 128, 1, 1000]
    cu, q, k, v, la, beta = gen.delta_inputs(lens, 3, 128, 41, "fp32", 0.2)
    la = la.clone()
    la[70, 1] = -float("inf")
    la[500:505, 2] = -float("inf")
    la[900:] *= 0.01
    o, s = tg.gated_delta_scan(dev(q), dev(k), dev(v), cu, dev(la), dev(beta), algo="chunked")
    torch.cuda.synchronize()
    assert tg.device_status() == 0
    ro, rs = do.scan(host_f32(q), host_f32(k), host_f32(v), host_f32(la), host_f32(beta), cu)
    assert_close("out", host_f32(o), ro, 1e-4, 1e-3)
    assert_close("state", host_f32(s), rs, 1e-4, 1e-3)


def test_chunked_scan_workspace_reuse_and_size_check():
    """A workspace reused by a second call with other inputs gives that call's
    results; one byte too small is refused before anything launches."""
    cu, q, k, v, la, beta = gen.delta_inputs([200, 77], 2, 64, 8, "fp32", 0.1)
    need = tg.delta_scan_workspace_bytes(cu, 2, 64)
    ws = torch.full((need,), 255, dtype=torch.uint8, device="cuda")
    tg.gated_delta_scan(dev(q), dev(k), dev(v), cu, dev(la), dev(beta), workspace=ws)
    q2 = q.flip(0).contiguous()
    o, s = tg.gated_delta_scan(dev(q2), dev(k), dev(v), cu, dev(la), dev(beta), workspace=ws)
    torch.cuda.synchronize()
    ro, rs = do.scan(host_f32(q2), host_f32(k), host_f32(v), host_f32(la), host_f32(beta), cu)
    assert_close("out", host_f32(o), ro, 1e-4, 1e-3)
    assert_close("state", host_f32(s), rs, 1e-4, 1e-3)
    with pytest.raises(tg.TokenGateError, match="TG_ERR_WORKSPACE"):
        tg.gated_delta_scan(dev(q), dev(k), dev(v), cu, dev(la), dev(beta), workspace=ws[:need - 1])
