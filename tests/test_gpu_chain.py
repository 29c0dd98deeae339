"""GPU parity of the whole gated layer (score -> select -> compact -> attend)
against the oracle's own chain on the same raw inputs, plus edge cases."""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import (ATTN_BF16, ATTN_FP32, GATE_ATOL, assert_close, dev, host_f32,
                                kept_set_agrees, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tg.library()
    yield
    assert tg.device_status() == 0, "a kernel reported a timed-out wait"


def _run_gpu(inp, algo=tg.ALGO_AUTO):
    w = inp.w
    return tg.gated_prefill(dev(inp.h), dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.W1),
                            dev(inp.b1), dev(inp.w2), inp.b2, dev(inp.gain), dev(inp.temp),
                            inp.cu_seqlens, inp.doc_begin, inp.doc_end, inp.budget,
                            rope_theta=w.rope_theta, algo=algo, want_lse=True)


def _oracle_chain(oracle, inp, rows=None):
    w = inp.w
    z = oracle.gate_score(inp.f32("h"), inp.f32("W1"), inp.b1.numpy(), inp.w2.numpy(), inp.b2)
    z32 = z.astype(np.float32)
    kept, cu_kept = oracle.topk_select(z32, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                       inp.budget)
    q = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("q"), w.n_q_heads, w.head_dim,
                           w.rope_theta)
    k = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("k"), w.n_kv_heads, w.head_dim,
                           w.rope_theta)
    v = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("v"))
    ls = oracle.logsig(kept, inp.cu_seqlens, inp.doc_begin, inp.doc_end, z32)
    out, lse = oracle.gated_attention(q, k, v, cu_kept, ls, inp.gain.numpy(), inp.temp.numpy(),
                                      rows=rows)
    return dict(z=z, kept=kept, cu_kept=cu_kept, out=out, lse=lse)


@pytest.mark.parametrize("name,algo", [("tiny_fp32", tg.ALGO_AUTO), ("tiny_fp32", tg.ALGO_SIMT),
                                       ("qwen_16k", tg.ALGO_AUTO)])
def test_chain_matches_oracle(oracle, name, algo):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w)
    g = _run_gpu(inp, algo)
    M = int(g["cu_kept_host"][-1])
    rows = None if w.total_tokens <= 4096 else sample_rows(M, g["cu_kept_host"], 24, seed=1)
    ref = _oracle_chain(oracle, inp, rows)
    assert_close("z", g["z"].cpu().numpy(), ref["z"], GATE_ATOL, 0.0)
    ok, ndiff = kept_set_agrees(g["kept_idx"].cpu().numpy(), ref["kept"], ref["z"], inp.cu_seqlens,
                                inp.doc_begin, inp.doc_end, inp.budget)
    assert ok, f"kept sets differ beyond the 1e-3 band ({ndiff} tokens)"
    for rows_b in inp.needle_rows:  # the planted needle always survives
        assert set(rows_b.tolist()) <= set(g["kept_idx"].cpu().numpy().tolist())
    if ndiff == 0:
        got = host_f32(g["out"])
        if rows is not None:
            got = got[rows]
        tol = ATTN_FP32 if w.dtype == "fp32" else ATTN_BF16
        # bf16 chain: the oracle attends over fp64 RoPE'd q/k while the GPU stores them
        # in bf16 first, so the bf16 bar applies; fp32 chain: the fp32 bar.
        assert_close("out", got, ref["out"], *tol)


@pytest.mark.parametrize("name", ["qwen_128k", "ragged_4"])
def test_chain_full_size_properties(oracle, name):
    """Full-size chain: sampled gate scores against the oracle, and the selection
    properties checked on the GPU's own scores (top-K is exact for given scores)."""
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w)
    g = _run_gpu(inp)
    z = g["z"].cpu().numpy()
    kept = g["kept_idx"].cpu().numpy()
    cu_kept = g["cu_kept"].cpu().numpy()
    np.testing.assert_array_equal(cu_kept, np.concatenate([[0], np.cumsum(w.kept_lengths())]))
    rng = np.random.default_rng(0)
    rows = rng.integers(0, w.total_tokens, 256)
    ref = oracle.gate_score(inp.f32("h"), inp.f32("W1"), inp.b1.numpy(), inp.w2.numpy(), inp.b2,
                            rows=rows)
    assert_close("z", z[rows], ref, GATE_ATOL, 0.0)
    for b in range(w.batch):
        s = inp.cu_seqlens[b] + inp.doc_begin[b]
        e = inp.cu_seqlens[b] + inp.doc_end[b]
        kb = kept[cu_kept[b]:cu_kept[b + 1]]
        assert np.all(np.diff(kb) > 0)
        doc_kept = kb[(kb >= s) & (kb < e)]
        assert len(doc_kept) == min(w.budgets[b], e - s)
        dropped = np.setdiff1d(np.arange(s, e), doc_kept)
        if len(dropped) and len(doc_kept):
            assert z[doc_kept].min() >= z[dropped].max()
        assert set(range(inp.cu_seqlens[b + 1] - w.question[b], inp.cu_seqlens[b + 1])) <= set(
            kb.tolist())
        assert set(inp.needle_rows[b].tolist()) <= set(kb.tolist())
    assert np.isfinite(host_f32(g["out"])).all()


def test_chain_edge_cases(oracle):
    """Empty prompts, K = 0, K >= n_doc, a prompt that is all question, one token."""
    w = gen.Workload("edges", (0, 1, 300, 257, 64, 130), (0, 1, 300, 7, 0, 2),
                     (5, 1, 10, 0, 1000, 64), 128, 32, 4, 2, 64, "bf16", 2, 21)
    inp = gen.make_inputs(w)
    g = _run_gpu(inp)
    ref = _oracle_chain(oracle, inp)
    assert_close("z", g["z"].cpu().numpy(), ref["z"], GATE_ATOL, 0.0)
    ok, ndiff = kept_set_agrees(g["kept_idx"].cpu().numpy(), ref["kept"], ref["z"], inp.cu_seqlens,
                                inp.doc_begin, inp.doc_end, inp.budget)
    assert ok
    if ndiff == 0:
        assert_close("out", host_f32(g["out"]), ref["out"], *ATTN_BF16)


def test_chain_maximum_batch(oracle):
    """TG_MAX_BATCH prompts through the whole chain (small model shape)."""
    rng = np.random.default_rng(91)
    B = tg.MAX_BATCH
    seq = rng.integers(1, 400, size=B)
    seq[::23] = 1
    qn = np.minimum(seq, rng.integers(0, 40, size=B))
    bud = rng.integers(0, 200, size=B)
    w = gen.Workload("max_batch", tuple(int(x) for x in seq), tuple(int(x) for x in qn),
                     tuple(int(x) for x in bud), 128, 32, 4, 2, 64, "bf16", 0, 92)
    inp = gen.make_inputs(w)
    g = _run_gpu(inp)
    ref = _oracle_chain(oracle, inp)
    assert_close("z", g["z"].cpu().numpy(), ref["z"], GATE_ATOL, 0.0)
    ok, ndiff = kept_set_agrees(g["kept_idx"].cpu().numpy(), ref["kept"], ref["z"], inp.cu_seqlens,
                                inp.doc_begin, inp.doc_end, inp.budget)
    assert ok
    if ndiff == 0:
        assert_close("out", host_f32(g["out"]), ref["out"], *ATTN_BF16)
