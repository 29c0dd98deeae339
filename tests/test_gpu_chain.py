"""GPU parity of the whole gated layer (score -> select -> compact -> attend)
against the oracle's own chain on the same raw inputs, plus edge cases."""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import (ATTN_BF16, ATTN_FP32, GATE_ATOL, LOGSIG_TOL, LSE_ATOL,
                                assert_close, assert_rope_close, dev, host_f32, kept_set_agrees,
                                sample_rows)

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
    """The oracle's own chain from the raw inputs (its scores, its selection)."""
    w = inp.w
    z = oracle.gate_score(inp.f32("h"), inp.f32("W1"), inp.b1.numpy(), inp.w2.numpy(), inp.b2)
    z32 = z.astype(np.float32)
    kept, cu_kept = oracle.topk_select(z32, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                       inp.budget)
    return dict(z=z, kept=kept, cu_kept=cu_kept)


def _check_chain(oracle, inp, g, rows=None, gate_rows=None):
    """Every stage of the GPU chain against the oracle:
      - gate scores within 1e-3 (all rows, or the sampled gate_rows);
      - the selection bit-exact against the oracle's top-K on the GPU's scores,
        and, when the oracle scored every row, within the 1e-3 band of its own;
      - the planted needle kept wherever the budget can hold it;
      - the compaction of the GPU's kept rows: residual and v bit-exact, q and
        k within one storage ulp of the oracle's fp64 RoPE, log-gates 1e-6;
      - the attention on the GPU's compacted rows at the stage bar (output
        and LSE), and the output of the oracle's own fp64 compaction and
        attention of the GPU's kept set at the dtype's bar."""
    w = inp.w
    z = g["z"].cpu().numpy()
    kept = g["kept_idx"].cpu().numpy()
    cu_kept = g["cu_kept"].cpu().numpy()
    if gate_rows is None:
        ref = _oracle_chain(oracle, inp)
        assert_close("z", z, ref["z"], GATE_ATOL, 0.0)
        ok, ndiff = kept_set_agrees(kept, ref["kept"], ref["z"], inp.cu_seqlens, inp.doc_begin,
                                    inp.doc_end, inp.budget)
        assert ok, f"kept sets differ beyond the 1e-3 band ({ndiff} tokens)"
    else:
        zr = oracle.gate_score(inp.f32("h"), inp.f32("W1"), inp.b1.numpy(), inp.w2.numpy(),
                               inp.b2, rows=gate_rows)
        assert_close("z", z[gate_rows], zr, GATE_ATOL, 0.0)
    ref_kept, ref_cu = oracle.topk_select(z, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                          inp.budget)
    np.testing.assert_array_equal(kept, ref_kept)
    np.testing.assert_array_equal(cu_kept, ref_cu)
    for b, rows_b in enumerate(inp.needle_rows):  # the planted needle survives
        if inp.budget[b] >= len(rows_b):
            assert set(rows_b.tolist()) <= set(kept.tolist())
    # compaction
    kt = torch.from_numpy(kept.astype(np.int64))
    for name in ("h", "v"):
        np.testing.assert_array_equal(g[name].cpu().view(torch.int16 if w.dtype == "bf16"
                                                         else torch.int32).numpy(),
                                      getattr(inp, name)[kt].view(
                                          torch.int16 if w.dtype == "bf16" else torch.int32
                                      ).numpy())
    ref_q = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("q"), w.n_q_heads, w.head_dim,
                               w.rope_theta)
    ref_k = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("k"), w.n_kv_heads, w.head_dim,
                               w.rope_theta)
    v64 = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("v"))
    if w.dtype == "bf16":
        assert_rope_close("q'", host_f32(g["q"]), ref_q)
        assert_rope_close("k'", host_f32(g["k"]), ref_k)
    else:
        assert_close("q'", host_f32(g["q"]), ref_q, 1e-5, 1e-5)
        assert_close("k'", host_f32(g["k"]), ref_k, 1e-5, 1e-5)
    ls = oracle.logsig(kept, inp.cu_seqlens, inp.doc_begin, inp.doc_end, z)
    assert_close("logsig", g["logsig"].cpu().numpy(), ls, *LOGSIG_TOL)
    # attention on the GPU's compacted rows (the stage's own inputs)
    tol = ATTN_FP32 if w.dtype == "fp32" else ATTN_BF16
    got = host_f32(g["out"])
    lse = g["lse"].cpu().numpy().T  # [M, Hq]
    if rows is not None:
        got, lse = got[rows], lse[rows]
    out_s, lse_s = oracle.gated_attention(host_f32(g["q"]), host_f32(g["k"]), host_f32(g["v"]),
                                          cu_kept, g["logsig"].cpu().numpy(), inp.gain.numpy(),
                                          inp.temp.numpy(), rows=rows)
    assert_close("out (stage)", got, out_s, *tol)
    assert_close("lse (stage)", lse, lse_s, LSE_ATOL, 1e-5)
    # end to end: the oracle's fp64 compaction and attention of the same kept set
    out_e, _ = oracle.gated_attention(ref_q, ref_k, v64, cu_kept, ls, inp.gain.numpy(),
                                      inp.temp.numpy(), rows=rows)
    assert_close("out (end to end)", got, out_e, *tol)


@pytest.mark.parametrize("name,algo", [("tiny_fp32", tg.ALGO_AUTO), ("tiny_fp32", tg.ALGO_SIMT),
                                       ("qwen_16k", tg.ALGO_AUTO)])
def test_chain_matches_oracle(oracle, name, algo):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w)
    g = _run_gpu(inp, algo)
    M = int(g["cu_kept_host"][-1])
    rows = None if w.total_tokens <= 4096 else sample_rows(M, g["cu_kept_host"], 24, seed=1)
    _check_chain(oracle, inp, g, rows)


@pytest.mark.parametrize("name", ["qwen_32k_k1024", "qwen_32k_k4096", "qwen_32k_k8192",
                                  "qwen_128k", "ragged_4"])
def test_chain_full_size_sampled(oracle, name):
    """Full-size chain on sampled rows: gate scores on sampled tokens, the
    selection bit-exact on the GPU's scores plus its properties, and the
    attention of sampled query rows over the GPU's kept set."""
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w)
    g = _run_gpu(inp)
    z = g["z"].cpu().numpy()
    kept = g["kept_idx"].cpu().numpy()
    cu_kept = g["cu_kept"].cpu().numpy()
    np.testing.assert_array_equal(cu_kept, np.concatenate([[0], np.cumsum(w.kept_lengths())]))
    rng = np.random.default_rng(0)
    gate_rows = np.unique(np.concatenate([rng.integers(0, w.total_tokens, 256),
                                          np.concatenate(inp.needle_rows)[:64]]))
    M = int(cu_kept[-1])
    rows = sample_rows(M, cu_kept, 24, seed=M)
    _check_chain(oracle, inp, g, rows, gate_rows)
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
    assert np.isfinite(host_f32(g["out"])).all()


def test_chain_edge_cases(oracle):
    """Empty prompts, K = 0, K >= n_doc, a prompt that is all question, one token."""
    w = gen.Workload("edges", (0, 1, 300, 257, 64, 130), (0, 1, 300, 7, 0, 2),
                     (5, 1, 10, 0, 1000, 64), 128, 32, 4, 2, 64, "bf16", 2, 21)
    inp = gen.make_inputs(w)
    _check_chain(oracle, inp, _run_gpu(inp))


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
    _check_chain(oracle, inp, _run_gpu(inp))
