"""GPU parity: gate score (tcgen05 and CUDA-core kernels) and top-K selection,
through the C ABI, against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import GATE_ATOL, assert_close, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tg.library()
    yield
    assert tg.device_status() == 0, "a kernel reported a timed-out wait"


# ---- gate ------------------------------------------------------------------

def _rand_gate(n, d, dg, dtype, seed, needle=False):
    rng = np.random.Generator(np.random.Philox(seed))
    h = rng.standard_normal((n, d), dtype=np.float32)
    W1 = rng.standard_normal((dg, d), dtype=np.float32) * 0.02
    if needle:
        h[n // 3] *= 6.0
    b1 = rng.standard_normal(dg, dtype=np.float32) * 0.02
    w2 = rng.standard_normal(dg, dtype=np.float32) * 0.02
    t = torch.float32 if dtype == "fp32" else torch.bfloat16
    return (torch.from_numpy(h).to(t), torch.from_numpy(W1).to(t), torch.from_numpy(b1),
            torch.from_numpy(w2), 0.013)


@pytest.mark.parametrize("n,d,dg,dtype,algo", [
    (1024, 256, 64, "fp32", tg.ALGO_AUTO),       # the tiny fp32 layer
    (1000, 2048, 256, "bf16", tg.ALGO_TCGEN05),  # Qwen-shaped, ragged last tile
    (1000, 2048, 256, "bf16", tg.ALGO_SIMT),
    (129, 128, 32, "bf16", tg.ALGO_TCGEN05),     # two tiles, one row in the second
    (1, 64, 32, "bf16", tg.ALGO_TCGEN05),
    (300, 320, 96, "bf16", tg.ALGO_TCGEN05),
    (5000, 512, 224, "bf16", tg.ALGO_TCGEN05),   # more tiles than SMs reuse the TMEM ring
    (77, 100, 20, "fp32", tg.ALGO_SIMT),
])
def test_gate_parity(oracle, n, d, dg, dtype, algo):
    h, W1, b1, w2, b2 = _rand_gate(n, d, dg, dtype, seed=n * 7 + d, needle=True)
    z = tg.gate_score(dev(h), dev(W1), dev(b1), dev(w2), b2, algo=algo)
    ref = oracle.gate_score(h.float().numpy(), W1.float().numpy(), b1.numpy(), w2.numpy(), b2)
    assert_close("z", z.cpu().numpy(), ref, GATE_ATOL, 0.0)
    if dtype == "fp32":  # fp32 products: far inside the bar
        assert_close("z(fp32)", z.cpu().numpy(), ref, 2e-5, 0.0)


@pytest.mark.parametrize("name", ["qwen_16k", "qwen_32k_k1024", "qwen_32k_k4096",
                                  "qwen_32k_k8192", "qwen_128k", "ragged_4"])
def test_gate_full_size_sampled(oracle, name):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w, with_qkv=False)
    z = tg.gate_score(dev(inp.h), dev(inp.W1), dev(inp.b1), dev(inp.w2), inp.b2).cpu().numpy()
    N = w.total_tokens
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([
        rng.integers(0, N, 384), np.arange(N - 130, N), np.arange(0, 130),
        np.concatenate(inp.needle_rows)[:64]]))
    ref = oracle.gate_score(inp.f32("h"), inp.f32("W1"), inp.b1.numpy(), inp.w2.numpy(), inp.b2,
                            rows=rows)
    assert_close("z", z[rows], ref, GATE_ATOL, 0.0)
    assert np.isfinite(z).all()


# ---- top-K -------------------------------------------------------------------

def _topk_both(oracle, z, cu, s, e, k):
    kept, cu_kept, host = tg.topk_select(torch.from_numpy(z).cuda(), cu, s, e, k)
    ref_kept, ref_cu = oracle.topk_select(z, cu, s, e, k)
    np.testing.assert_array_equal(host, ref_cu)
    np.testing.assert_array_equal(cu_kept.cpu().numpy(), ref_cu)
    np.testing.assert_array_equal(kept.cpu().numpy(), ref_kept)


@pytest.mark.parametrize("n", [1, 2, 31, 100, 1000, 4097, 16384, 131072])
@pytest.mark.parametrize("kfrac", [0.0, 0.001, 0.25, 0.999, 1.0, 2.0])
def test_topk_bit_exact_single(oracle, n, kfrac):
    z = gen.random_scores(n, seed=n)
    q = min(256, n // 4)
    n_doc = n - q
    K = int(round(kfrac * n_doc))
    _topk_both(oracle, z, [0, n], [0], [n_doc], [K])


@pytest.mark.parametrize("seed", range(6))
def test_topk_bit_exact_varlen(oracle, seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 12))
    lens = rng.integers(0, 20000, size=B)
    lens[rng.random(B) < 0.2] = 0
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    s = np.array([rng.integers(0, L + 1) for L in lens], np.int32)
    e = np.array([rng.integers(ss, L + 1) for ss, L in zip(s, lens)], np.int32)
    k = np.array([rng.integers(0, max(ee - ss, 1) + 3) for ss, ee in zip(s, e)], np.int32)
    z = gen.random_scores(int(cu[-1]), seed=100 + seed)
    _topk_both(oracle, z, cu, s, e, k)


def test_topk_ties_everywhere(oracle):
    n = 50000
    z = np.full(n, 0.5, np.float32)
    z[::7] = 0.25
    z[::1000] = np.nan
    z[5::9] = -0.0
    z[6::9] = 0.0
    for K in (1, 6000, 30000, 49000):
        _topk_both(oracle, z, [0, n], [100], [n - 100], [K])


def test_topk_question_in_the_middle_and_front(oracle):
    z = gen.random_scores(30000, seed=3)
    cu = [0, 10000, 30000]
    _topk_both(oracle, z, cu, [500, 0], [9000, 19000], [700, 12345])


@pytest.mark.parametrize("name,seed", [("qwen_128k", 3), ("ragged_4", 4), ("qwen_32k_k1024", 2),
                                       ("qwen_32k_k4096", 2), ("qwen_32k_k8192", 2)])
def test_topk_full_size(oracle, name, seed):
    w = gen.WORKLOADS[name]
    cu = np.concatenate([[0], np.cumsum(w.seqlens)]).astype(np.int32)
    e = np.array([n - q for n, q in zip(w.seqlens, w.question)], np.int32)
    z = gen.random_scores(int(cu[-1]), seed=seed, specials=False)
    _topk_both(oracle, z, cu, np.zeros(w.batch, np.int32), e, np.array(w.budgets, np.int32))


# ---- random-K selection (caller-drawn keys) and budget sweeps ---------------------

def _varlen(seed, lens):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    s, e = [], []
    for n in lens:
        a = int(rng.integers(0, max(n // 4, 1))) if n else 0
        b = int(rng.integers(max(a, n - n // 4), n + 1)) if n else 0
        s.append(a)
        e.append(b)
    return cu, np.array(s, np.int32), np.array(e, np.int32)


@pytest.mark.parametrize("lens,bits", [([1], 32), ([1000], 32), ([4097], 3), ([16384], 32),
                                       ([131072], 32), ([5, 0, 300, 1, 2049], 32),
                                       ([700, 900], 1)])
def test_random_select_bit_exact(oracle, lens, bits):
    cu, s, e = _varlen(len(lens) + bits, lens)
    keys = gen.random_keys(int(cu[-1]), seed=sum(lens) + bits, bits=bits)
    rng = np.random.default_rng(bits)
    for kfrac in (0.0, 0.1, 0.5, 1.0, 2.0):
        k = np.array([int(kfrac * (b - a)) for a, b in zip(s, e)], np.int32)
        kk, ck, _ = tg.random_select(torch.from_numpy(keys.view(np.int32)).cuda(), cu, s, e, k)
        ref, ref_cu = oracle.select_by_keys(keys, cu, s, e, k)
        assert ck.cpu().numpy().tolist() == ref_cu.tolist()
        np.testing.assert_array_equal(kk.cpu().numpy(), ref)


@pytest.mark.parametrize("lens", [[16384], [5, 0, 300, 1, 2049, 8192], [131072]])
def test_topk_budget_sweep_bit_exact(oracle, lens):
    """One launch, up to eight budgets from the same scores: each budget's
    kept rows equal the oracle's top-K with that budget."""
    cu, s, e = _varlen(7, lens)
    z = gen.random_scores(int(cu[-1]), seed=len(lens))
    n_doc = e - s
    fracs = [0.0, 0.01, 0.125, 0.3, 0.5, 0.9, 1.0, 1.5]
    budgets = [[int(f * nd) for nd in n_doc] for f in fracs]
    outs = tg.topk_select_multi(torch.from_numpy(z).cuda(), cu, s, e, budgets)
    assert len(outs) == len(budgets)
    for (kk, ck, host), k in zip(outs, budgets):
        ref, ref_cu = oracle.topk_select(z, cu, s, e, k)
        assert ck.cpu().numpy().tolist() == ref_cu.tolist() == host.tolist()
        np.testing.assert_array_equal(kk.cpu().numpy(), ref)


def test_topk_maximum_batch(oracle):
    """TG_MAX_BATCH prompts in one launch, empty and one-token prompts among them."""
    rng = np.random.default_rng(77)
    B = tg.MAX_BATCH
    lens = rng.integers(0, 700, size=B)
    lens[::17] = 0
    lens[5::19] = 1
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = np.minimum(lens, rng.integers(0, 64, size=B))
    s = np.zeros(B, np.int32)
    e = (lens - q).astype(np.int32)
    k = rng.integers(0, 300, size=B).astype(np.int32)
    z = gen.random_scores(int(cu[-1]), seed=78)
    _topk_both(oracle, z, cu, s, e, k)


def test_topk_longest_prompt(oracle):
    """The longest prompt the cluster holds: 8 CTAs x 45056 keys; one more is refused."""
    n = 8 * 45056
    z = gen.random_scores(n, seed=79)
    _topk_both(oracle, z, [0, n], [0], [n - 512], [n // 8])
    z2 = torch.from_numpy(gen.random_scores(n + 1, seed=80)).cuda()
    with pytest.raises(tg.TokenGateError, match="TG_ERR_UNSUPPORTED.*exceeds"):
        tg.topk_select(z2, [0, n + 1], [0], [n], [1000])


# ---- the selection's first radix pass counted by the gate ---------------------

def _fused(inp, ws, algo=tg.ALGO_AUTO, z=None):
    z = tg.gate_score(dev(inp.h), dev(inp.W1), dev(inp.b1), dev(inp.w2), inp.b2, out=z,
                      algo=algo, topk_ws=ws, cu_seqlens=inp.cu_seqlens, doc_begin=inp.doc_begin,
                      doc_end=inp.doc_end)
    return z


def _select_ws(oracle, inp, z, ws):
    kept, cu_kept, host = tg.topk_select(z, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                         inp.budget, workspace=ws)
    ref_kept, ref_cu = oracle.topk_select(z.cpu().numpy(), inp.cu_seqlens, inp.doc_begin,
                                          inp.doc_end, inp.budget)
    np.testing.assert_array_equal(kept.cpu().numpy(), ref_kept)
    np.testing.assert_array_equal(cu_kept.cpu().numpy(), ref_cu)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0, "the selection must leave the workspace zeroed"


@pytest.mark.parametrize("name", ["tiny_fp32", "qwen_16k", "qwen_32k_k4096", "qwen_128k",
                                  "ragged_4"])
def test_fused_gate_selection_bit_exact(oracle, name):
    """Gate with the first-pass histograms, then the selection from them: the
    kept rows equal the oracle's top-K of the same scores, bit for bit, and the
    scores equal the plain gate's exactly (the histogram changes no score)."""
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w, with_qkv=False)
    ws = tg.topk_workspace(w.batch)
    z = _fused(inp, ws)
    z_plain = tg.gate_score(dev(inp.h), dev(inp.W1), dev(inp.b1), dev(inp.w2), inp.b2)
    assert torch.equal(z, z_plain)
    _select_ws(oracle, inp, z, ws)


def test_fused_histogram_counts_every_document_token(oracle):
    """The gate's histogram of each prompt is exactly the count of its document
    tokens' scores by the top 11 bits of the order key (read before any
    selection consumes it), and the tag names the scores."""
    w = gen.Workload("hist", (300, 0, 1000, 64, 2049), (20, 0, 1000, 3, 49), (5, 1, 10, 0, 100),
                     256, 64, 4, 2, 64, "bf16", 4, 31)
    inp = gen.make_inputs(w, with_qkv=False)
    ws = tg.topk_workspace(w.batch)
    z = _fused(inp, ws)
    torch.cuda.synchronize()
    words = ws.view(torch.int32).cpu().numpy().view(np.uint32).reshape(w.batch, 2112)
    u = z.cpu().numpy().view(np.uint32).copy()
    u[u == 0x80000000] = 0  # -0.0 counts as +0.0
    key = np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)
    key[np.isnan(z.cpu().numpy())] = 0
    for b in range(w.batch):
        s = inp.cu_seqlens[b] + inp.doc_begin[b]
        e = inp.cu_seqlens[b] + inp.doc_end[b]
        ref = np.bincount(key[s:e] >> 21, minlength=2048)
        np.testing.assert_array_equal(words[b, :2048], ref)
        assert words[b, 2048] == 0x7A6E5B1F and words[b, 2049] == w.total_tokens
        assert (int(words[b, 2051]) << 32 | int(words[b, 2050])) == z.data_ptr()
    # the selection consumes them and leaves the workspace zeroed
    _select_ws(oracle, inp, z, ws)


def test_fused_selection_falls_back_when_the_histogram_does_not_fit(oracle):
    """The selection counts the first pass itself when the workspace does not
    hold a histogram of these scores: never counted (zero), counted twice (two
    gate calls, twice the tokens), or counted from scores at another address.
    The kept rows are exact in every case and the workspace ends zeroed."""
    w = gen.WORKLOADS["qwen_16k"]
    inp = gen.make_inputs(w, with_qkv=False)
    ws = tg.topk_workspace(w.batch)
    z = _fused(inp, ws)
    torch.cuda.synchronize()
    ws.zero_()                                   # never counted
    _select_ws(oracle, inp, z, ws)
    _fused(inp, ws, z=z)
    _fused(inp, ws, z=z)                         # counted twice
    _select_ws(oracle, inp, z, ws)
    other = torch.empty_like(z)
    _fused(inp, ws, z=other)                     # the tag names `other`
    _select_ws(oracle, inp, z.clone(), ws)


def test_fused_selection_edge_batches(oracle):
    """Empty prompts, K = 0, K >= n_doc, an all-question prompt, a document in
    the middle, one-token prompts, and TG_MAX_BATCH prompts, through the
    CUDA-core gate (fp32) and the tensor-core gate (bf16)."""
    rng = np.random.default_rng(5)
    B = tg.MAX_BATCH
    seq = rng.integers(1, 600, size=B)
    seq[::17] = 1
    seq[5] = 0
    qn = np.minimum(seq, rng.integers(0, 40, size=B))
    bud = rng.integers(0, 300, size=B)
    bud[::11] = 0
    for dt, algo in (("bf16", tg.ALGO_AUTO), ("fp32", tg.ALGO_SIMT)):
        w = gen.Workload("edges", tuple(int(x) for x in seq), tuple(int(x) for x in qn),
                         tuple(int(x) for x in bud), 128, 32, 4, 2, 64, dt, 1, 17)
        inp = gen.make_inputs(w, with_qkv=False)
        ws = tg.topk_workspace(w.batch)
        _select_ws(oracle, inp, _fused(inp, ws, algo), ws)
    # a document span in the middle of its prompt (question before and after)
    w = gen.Workload("mid", (5000, 3000), (0, 0), (700, 2999), 128, 32, 4, 2, 64, "bf16", 1, 18)
    inp = gen.make_inputs(w, with_qkv=False)
    inp.doc_begin[:] = [1000, 1]
    inp.doc_end[:] = [4000, 3000]
    ws = tg.topk_workspace(w.batch)
    _select_ws(oracle, inp, _fused(inp, ws), ws)


@pytest.mark.parametrize("name", ["qwen_16k", "ragged_4"])
def test_fused_budget_sweep_shares_the_gate_histogram(oracle, name):
    """A budget sweep on the gate's first-pass histogram: every budget's kept
    rows equal the oracle's top-K of the same scores with that budget, and the
    workspace is zero once the last budget has read it (budgets of 0, 1, the
    whole document and in between, per prompt)."""
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w, with_qkv=False)
    n_doc = np.asarray(inp.doc_end) - np.asarray(inp.doc_begin)
    sweep = [[0] * w.batch, [1] * w.batch, [int(x) for x in n_doc], [int(x) + 5 for x in n_doc]]
    sweep += [[max(1, int(f * nd)) for nd in n_doc] for f in (0.03, 0.125, 0.5, 0.9)]
    ws = tg.topk_workspace(w.batch)
    z = _fused(inp, ws)
    outs = tg.topk_select_multi(z, inp.cu_seqlens, inp.doc_begin, inp.doc_end, sweep,
                                workspace=ws)
    zh = z.cpu().numpy()
    for (kept, cu_kept, host), bud in zip(outs, sweep):
        ref_kept, ref_cu = oracle.topk_select(zh, inp.cu_seqlens, inp.doc_begin, inp.doc_end,
                                              np.asarray(bud, np.int32))
        np.testing.assert_array_equal(kept.cpu().numpy(), ref_kept)
        np.testing.assert_array_equal(cu_kept.cpu().numpy(), ref_cu)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0
