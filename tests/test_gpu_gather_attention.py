"""GPU parity: compaction (+RoPE, log-sigmoid) and token-gated attention
(tcgen05 and CUDA-core kernels), through the C ABI, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import (ATTN_BF16, ATTN_FP32, LOGSIG_TOL, LSE_ATOL, assert_close,
                                assert_rope_close, dev, host_f32, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tg.library()
    yield
    assert tg.device_status() == 0, "a kernel reported a timed-out wait"


# ---- compaction --------------------------------------------------------------

def _gather_case(oracle, w, seed):
    inp = gen.make_inputs(w)
    z = gen.random_scores(w.total_tokens, seed=seed, specials=False)
    kept, cu_kept = oracle.topk_select(z, inp.cu_seqlens, inp.doc_begin, inp.doc_end, inp.budget)
    kd = torch.from_numpy(kept).cuda()
    kt = torch.from_numpy(kept.astype(np.int64))
    Hq, Hkv, dh = w.n_q_heads, w.n_kv_heads, w.head_dim
    (hc, qc, kc, vc), ls = tg.compact_gather(
        kd, inp.cu_seqlens, inp.doc_begin, inp.doc_end, inp.budget,
        [dev(inp.h), dev(inp.q), dev(inp.k), dev(inp.v)], rope_heads=[0, Hq, Hkv, 0],
        head_dim=dh, rope_theta=w.rope_theta, z=torch.from_numpy(z).cuda())
    # untouched rows are bit-exact copies
    np.testing.assert_array_equal(hc.cpu().view(torch.int16).numpy(),
                                  inp.h[kt].view(torch.int16).numpy())
    np.testing.assert_array_equal(vc.cpu().view(torch.int16).numpy(),
                                  inp.v[kt].view(torch.int16).numpy())
    ref_q = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("q"), Hq, dh, w.rope_theta)
    ref_k = oracle.gather_rows(kept, inp.cu_seqlens, inp.f32("k"), Hkv, dh, w.rope_theta)
    if w.dtype == "bf16":
        assert_rope_close("q'", host_f32(qc), ref_q)
        assert_rope_close("k'", host_f32(kc), ref_k)
    else:
        assert_close("q'", host_f32(qc), ref_q, 1e-5, 1e-5)
        assert_close("k'", host_f32(kc), ref_k, 1e-5, 1e-5)
    ref_ls = oracle.logsig(kept, inp.cu_seqlens, inp.doc_begin, inp.doc_end, z)
    assert_close("logsig", ls.cpu().numpy(), ref_ls, *LOGSIG_TOL)


@pytest.mark.parametrize("name", ["tiny_fp32", "qwen_16k", "qwen_32k_k1024", "qwen_32k_k4096",
                                  "qwen_32k_k8192", "qwen_128k", "ragged_4"])
def test_gather_parity(oracle, name):
    _gather_case(oracle, gen.WORKLOADS[name], seed=11)


def test_gather_varlen_small_and_empty(oracle):
    w = gen.Workload("edge", (5, 0, 300, 1, 129), (1, 0, 50, 1, 0), (2, 3, 0, 1, 1000), 128, 32,
                     4, 2, 64, "bf16", 1, 9)
    _gather_case(oracle, w, seed=5)


@pytest.mark.parametrize("dtype,d_model", [("bf16", 32768), ("fp32", 16384)])
def test_gather_rows_wider_than_a_stage(oracle, dtype, d_model):
    # a kept row of more than 48 KB over its four tensors does not fit one stage of
    # the bulk-copy ring: the warp-per-(row, tensor) kernel moves it
    w = gen.Workload("wide", (300, 0, 77), (20, 0, 5), (40, 1, 100), d_model, 32, 4, 2, 64, dtype,
                     1, 13)
    _gather_case(oracle, w, seed=3)


# ---- attention -----------------------------------------------------------------

def _attn_case(oracle, lens, Hq, Hkv, dh, dtype, algo, bias=True, seed=0, rows=None,
               workspace="auto"):
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, seed, dtype, bias)
    out, lse = tg.gated_attention(dev(q), dev(k), dev(v), cu, dev(ls), dev(gain), dev(temp),
                                  algo=algo, want_lse=True, workspace=workspace)
    ref, ref_lse = oracle.gated_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                          cu, None if ls is None else ls.numpy(), gain.numpy(),
                                          temp.numpy(), rows=rows)
    got = host_f32(out)
    got_lse = lse.cpu().numpy().T
    if rows is not None:
        got, got_lse = got[rows], got_lse[rows]
    tol = ATTN_BF16 if dtype == "bf16" else ATTN_FP32
    assert_close("attn", got, ref, *tol)
    assert_close("lse", got_lse, ref_lse, LSE_ATOL, 1e-5)


@pytest.mark.parametrize("lens", [[1], [127], [128], [129], [300], [1000], [5, 0, 260, 1, 640]])
@pytest.mark.parametrize("algo", [tg.ALGO_TCGEN05, tg.ALGO_SIMT])
def test_attention_bf16_d128(oracle, lens, algo):
    _attn_case(oracle, lens, 16, 8, 128, "bf16", algo, seed=len(lens) + sum(lens))


@pytest.mark.parametrize("lens", [[1000], [2304], [5, 0, 260, 1, 640]])
def test_attention_without_workspace(oracle, lens):
    """No workspace: every query tile stays on one SM (no key-range split)."""
    _attn_case(oracle, lens, 16, 8, 128, "bf16", tg.ALGO_TCGEN05, seed=sum(lens) + 3,
               workspace=None)


@pytest.mark.parametrize("lens,Hq,Hkv,dh", [([1000], 16, 8, 64), ([1280], 12, 4, 128),
                                            ([700, 90, 1500], 12, 4, 128), ([900], 4, 2, 64)])
def test_attention_split_matches_unsplit_and_repeats(lens, Hq, Hkv, dh):
    """Small batches split long query tiles over several SMs; the merged result
    must agree with the unsplit kernel and be identical on repeated calls (the
    merge order is fixed, and each call re-arms the workspace counters)."""
    cu = np.concatenate([[0], np.cumsum(lens)])
    need = tg.attention_workspace_bytes(cu, Hq, Hkv, dh)
    assert need > 0, "this shape is expected to split"
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, 17, "bf16", True)
    args = [dev(x) for x in (q, k, v)] + [cu, dev(ls), dev(gain), dev(temp)]
    ws = torch.full((need,), 0xAB, dtype=torch.uint8, device="cuda")  # counters must be re-armed
    o1, l1 = tg.gated_attention(*args, algo=tg.ALGO_TCGEN05, want_lse=True, workspace=ws)
    o2, l2 = tg.gated_attention(*args, algo=tg.ALGO_TCGEN05, want_lse=True, workspace=ws)
    o0, l0 = tg.gated_attention(*args, algo=tg.ALGO_TCGEN05, want_lse=True, workspace=None)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)
    assert_close("split vs unsplit", host_f32(o1), host_f32(o0), 2 ** -7, 2 ** -7)
    assert_close("split vs unsplit lse", l1.cpu().numpy(), l0.cpu().numpy(), 1e-4, 1e-6)


@pytest.mark.parametrize("lens,bias", [([700], True), ([700], False), ([64, 200, 3], True)])
@pytest.mark.parametrize("algo", [tg.ALGO_TCGEN05, tg.ALGO_SIMT])
def test_attention_bf16_d64_and_nobias(oracle, lens, bias, algo):
    _attn_case(oracle, lens, 4, 2, 64, "bf16", algo, bias=bias, seed=sum(lens))
    _attn_case(oracle, lens, 4, 4, 128, "bf16", algo, bias=bias, seed=sum(lens) + 1)


@pytest.mark.parametrize("lens", [[320], [1], [33, 100, 0, 257]])
def test_attention_fp32(oracle, lens):
    _attn_case(oracle, lens, 4, 2, 64, "fp32", tg.ALGO_AUTO, seed=sum(lens))


def test_attention_gain_zero_temp_one_is_plain_causal(oracle):
    """Checked against torch's own SDPA on the GPU as a second, independent reference."""
    lens, Hq, Hkv, dh = [1000], 16, 8, 128
    cu, q, k, v, ls, _, _ = gen.attention_inputs(lens, Hq, Hkv, dh, 5, "bf16")
    gain, temp = torch.zeros(Hq), torch.ones(Hq)
    out, _ = tg.gated_attention(dev(q), dev(k), dev(v), cu, dev(ls), dev(gain), dev(temp),
                                algo=tg.ALGO_TCGEN05)
    qf, kf, vf = (dev(x).float().transpose(0, 1) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        qf[None], kf.repeat_interleave(2, 0)[None], vf.repeat_interleave(2, 0)[None],
        is_causal=True)[0].transpose(0, 1)
    assert_close("sdpa", host_f32(out), ref.cpu().numpy(), *ATTN_BF16)


@pytest.mark.parametrize("name", ["qwen_16k", "qwen_32k_k1024", "qwen_32k_k4096",
                                  "qwen_32k_k8192", "qwen_128k", "ragged_4"])
def test_attention_full_size_sampled(oracle, name):
    w = gen.WORKLOADS[name]
    lens = w.kept_lengths()
    M = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)])
    rows = sample_rows(M, cu, n_random=24, seed=M)
    _attn_case(oracle, lens, w.n_q_heads, w.n_kv_heads, w.head_dim, "bf16", tg.ALGO_TCGEN05,
               seed=w.seed, rows=rows)


@pytest.mark.parametrize("name", ["qwen_32k_k8192"])
def test_ungated_full_n_attention_sampled(oracle, name):
    """The ungated comparison of the 32k configuration: plain causal GQA
    attention over all N tokens (no log-gates, gain 0, temperature 1), checked
    on about a thousand query rows spread over the whole length."""
    w = gen.WORKLOADS[name]
    N = w.total_tokens
    cu, q, k, v, _, _, _ = gen.attention_inputs([N], w.n_q_heads, w.n_kv_heads, w.head_dim,
                                                w.seed + 5, "bf16", False)
    Hq = w.n_q_heads
    gain, temp = torch.zeros(Hq), torch.ones(Hq)
    out, lse = tg.gated_attention(dev(q), dev(k), dev(v), cu, None, dev(gain), dev(temp),
                                  want_lse=True)
    rows = sample_rows(N, cu, n_random=1000, seed=N)
    ref, ref_lse = oracle.gated_attention(q.float().numpy(), k.float().numpy(),
                                          v.float().numpy(), cu, None, gain.numpy(),
                                          temp.numpy(), rows=rows)
    assert_close("ungated out", host_f32(out)[rows], ref, *ATTN_BF16)
    assert_close("ungated lse", lse.cpu().numpy().T[rows], ref_lse, LSE_ATOL, 0.0)


def test_attention_repeated_calls_identical():
    """Back-to-back calls: every pipeline barrier returns to the same state, so
    repeated launches give bit-identical results and no wait times out."""
    lens = [300, 1000, 129]
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, 16, 8, 128, 23, "bf16", True)
    args = [dev(x) for x in (q, k, v)] + [cu, dev(ls), dev(gain), dev(temp)]
    outs = [tg.gated_attention(*args, algo=tg.ALGO_TCGEN05, workspace=None)[0] for _ in range(8)]
    torch.cuda.synchronize()
    assert tg.device_status() == 0
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
