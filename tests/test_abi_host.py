"""C-ABI checks that need no GPU: the library loads, exports every function the
header declares, and rejects invalid arguments with the documented status
before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import build as tgbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tokengate.h")

OK, INVALID, SHAPE, DTYPE, ALIGN, UNSUP, CUDA = 0, 1, 2, 3, 4, 5, 6
WORKSPACE = 8
FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced by a rejected call
FAKE_ODD = ctypes.c_void_p(0x10008)  # 8-byte aligned only


@pytest.fixture(scope="module")
def L():
    tgbuild.build()
    return tg.library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tg_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    declared = _declared_functions()
    assert declared, "no declarations parsed"
    assert set(declared) == set(tg.EXPORTED_SYMBOLS)
    for name in declared:
        assert hasattr(L, name), name


def test_only_abi_symbols_are_exported(L):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", tg.LIB_PATH], capture_output=True,
                         text=True).stdout
    syms = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {s for s in syms if s.startswith("tg_")} == set(tg.EXPORTED_SYMBOLS)


def test_status_strings_and_version(L):
    assert L.tg_status_string(0) == b"TG_OK"
    assert L.tg_status_string(5) == b"TG_ERR_UNSUPPORTED"
    assert b"sm_100a" in L.tg_version()


def _arr(a):
    a = np.ascontiguousarray(a, np.int32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def test_kept_offsets_matches_definition(L):
    cu, cu_p = _arr([0, 100, 100, 350])
    s, s_p = _arr([10, 0, 0])
    e, e_p = _arr([90, 0, 250])
    k, k_p = _arr([30, 5, 1000])
    out = np.zeros(4, np.int32)
    rc = L.tg_kept_offsets(3, cu_p, s_p, e_p, k_p, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    assert rc == OK
    # M_b = min(K, n_doc) + (N_b - n_doc)
    assert out.tolist() == [0, 30 + 20, 50 + 0, 50 + 250]


@pytest.mark.parametrize("cu,s,e,k,code", [
    ([0, 10], [0], [11], [1], INVALID),   # span past the end
    ([0, 10], [5], [4], [1], INVALID),    # reversed span
    ([0, 10], [0], [5], [-1], INVALID),   # negative budget
    ([1, 10], [0], [5], [1], INVALID),    # cu_seqlens[0] != 0
    ([0, 10, 5], [0, 0], [5, 0], [1, 1], INVALID),  # decreasing offsets
])
def test_prompt_validation(L, cu, s, e, k, code):
    _, cu_p = _arr(cu)
    _, s_p = _arr(s)
    _, e_p = _arr(e)
    _, k_p = _arr(k)
    out = np.zeros(len(s) + 1, np.int32)
    assert L.tg_kept_offsets(len(s), cu_p, s_p, e_p, k_p,
                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))) == code
    assert L.tg_topk_select(FAKE, len(s), cu_p, s_p, e_p, k_p, FAKE, FAKE, None) == code
    assert b"" != L.tg_last_error_message()


def test_topk_limits(L):
    B = 129
    _, cu_p = _arr(np.arange(B + 1) * 4)
    _, s_p = _arr(np.zeros(B))
    _, e_p = _arr(np.full(B, 2))
    _, k_p = _arr(np.ones(B))
    assert L.tg_topk_select(FAKE, B, cu_p, s_p, e_p, k_p, FAKE, FAKE, None) == UNSUP
    _, cu_p = _arr([0, 400000])
    _, s_p = _arr([0])
    _, e_p = _arr([399000])
    _, k_p = _arr([10])
    assert L.tg_topk_select(FAKE, 1, cu_p, s_p, e_p, k_p, FAKE, FAKE, None) == UNSUP


def test_gate_validation(L):
    g = L.tg_gate_score
    assert g(FAKE, 7, 16, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 0, None) == DTYPE
    assert g(FAKE, 0, -1, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 0, None) == INVALID
    assert g(FAKE_ODD, 0, 16, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 0, None) == ALIGN
    assert g(FAKE, 0, 16, 60, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 0, None) == ALIGN  # 120-byte rows
    assert g(FAKE, 1, 16, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 2, None) == UNSUP  # tcgen05 + fp32
    assert g(FAKE, 0, 16, 96, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 2, None) == UNSUP  # d % 64
    assert g(FAKE, 0, 16, 64, FAKE, FAKE, 48, FAKE, 0.0, FAKE, 2, None) == UNSUP  # dg % 32
    assert g(FAKE, 0, 16, 64, FAKE, FAKE, 512, FAKE, 0.0, FAKE, 2, None) == UNSUP  # dg > 256
    assert g(FAKE, 0, 16, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 9, None) == INVALID
    assert g(None, 0, 16, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 0, None) == INVALID
    assert g(None, 0, 0, 64, None, None, 32, None, 0.0, None, 0, None) == OK  # empty: no-op


def test_gather_validation(L):
    _, cu_p = _arr([0, 10])
    _, s_p = _arr([0])
    _, e_p = _arr([8])
    _, k_p = _arr([4])
    t = (tg.GatherTensor * 1)()
    t[0].src, t[0].dst, t[0].row_elems, t[0].rope_heads = 0x10000, 0x20000, 64, 1
    f = L.tg_compact_gather
    assert f(FAKE, 5, 1, cu_p, s_p, e_p, k_p, 0, t, 1, 64, 1e6, FAKE, FAKE, None) == SHAPE  # M=6
    assert f(FAKE, 6, 1, cu_p, s_p, e_p, k_p, 0, t, 1, 96, 1e6, FAKE, FAKE, None) == SHAPE  # 96>64
    assert f(FAKE, 6, 1, cu_p, s_p, e_p, k_p, 0, t, 1, 40, 1e6, FAKE, FAKE, None) == UNSUP
    assert f(FAKE, 6, 1, cu_p, s_p, e_p, k_p, 0, t, 1, 64, 0.5, FAKE, FAKE, None) == INVALID
    t[0].row_elems = 60  # 120-byte rows
    t[0].rope_heads = 0
    assert f(FAKE, 6, 1, cu_p, s_p, e_p, k_p, 0, t, 1, 0, 1e6, FAKE, FAKE, None) == ALIGN
    assert f(FAKE, 6, 1, cu_p, s_p, e_p, k_p, 0, t, 9, 0, 1e6, FAKE, FAKE, None) == INVALID


def test_attention_validation(L):
    _, ck = _arr([0, 100])
    a = L.tg_gated_attention
    n = None  # workspace pointer
    assert a(FAKE, FAKE, FAKE, 0, 1, ck, 16, 6, 128, None, FAKE, FAKE, FAKE, None, n, 0, 0,
             None) == SHAPE
    assert a(FAKE, FAKE, FAKE, 0, 1, ck, 16, 8, 96, None, FAKE, FAKE, FAKE, None, n, 0, 0,
             None) == UNSUP
    assert a(FAKE, FAKE, FAKE, 1, 1, ck, 16, 8, 128, None, FAKE, FAKE, FAKE, None, n, 0, 2,
             None) == UNSUP
    assert a(FAKE_ODD, FAKE, FAKE, 0, 1, ck, 16, 8, 128, None, FAKE, FAKE, FAKE, None, n, 0, 0,
             None) == ALIGN
    assert a(FAKE, FAKE, FAKE, 0, 1, ck, 16, 8, 128, None, FAKE, FAKE, FAKE, None, FAKE_ODD,
             1 << 20, 0, None) == ALIGN
    _, bad = _arr([0, 100, 50])
    assert a(FAKE, FAKE, FAKE, 0, 2, bad, 16, 8, 128, None, FAKE, FAKE, FAKE, None, n, 0, 0,
             None) == INVALID


def _ws_bytes(L, cu, hq=16, hkv=8, dh=128, dtype=0, algo=0):
    _, ck = _arr(cu)
    out = ctypes.c_size_t(123)
    st = L.tg_attention_workspace_bytes(dtype, len(cu) - 1, ck, hq, hkv, dh, algo,
                                        ctypes.byref(out))
    return st, out.value


def test_attention_workspace_plan(L):
    """The split plan is host logic: small batches that cannot fill the GPU ask
    for workspace; long prompts, fp32 and the CUDA-core kernel ask for none.
    (Without a GPU the planner assumes 148 SMs.)"""
    import torch

    if torch.cuda.is_available():
        pytest.skip("plan sizes below assume 148 SMs")
    st, b = _ws_bytes(L, [0, 1280], hq=12, hkv=4)  # one prompt kept down to 1280 rows
    assert st == 0 and b > 0
    # with even GQA groups the same batch runs on CTA pairs, which never split
    assert _ws_bytes(L, [0, 1280]) == (0, 0)
    # every partial slot holds 2 heads x 128 rows x (head_dim + 1) floats, plus counters
    assert b % 4 == 0 and b >= 2 * 128 * 129 * 4
    st, b = _ws_bytes(L, [0, 8448])  # 66 query tiles x 8 head pairs: no split
    assert (st, b) == (0, 0)
    assert _ws_bytes(L, [0, 2304], dtype=1) == (0, 0)  # fp32: CUDA-core kernel
    assert _ws_bytes(L, [0, 2304], algo=1) == (0, 0)
    assert _ws_bytes(L, [0, 0]) == (0, 0)  # nothing kept
    assert _ws_bytes(L, [0, 2304], hkv=6)[0] == SHAPE
    assert _ws_bytes(L, [0, 2304], dh=96)[0] == UNSUP
    _, ck = _arr([0, 10])
    assert L.tg_attention_workspace_bytes(0, 1, ck, 16, 8, 128, 0, None) == INVALID
    # a workspace smaller than the plan needs is refused before anything launches
    st, need = _ws_bytes(L, [0, 1280], hq=12, hkv=4)
    _, ck = _arr([0, 1280])
    a = L.tg_gated_attention
    assert a(FAKE, FAKE, FAKE, 0, 1, ck, 12, 4, 128, None, FAKE, FAKE, FAKE, None, FAKE,
             need - 16, 0, None) == WORKSPACE
    assert b"needed" in L.tg_last_error_message()


def test_attention_kernel_choice():
    """The per-call plan on 148 SMs: CTA pairs when a small batch cannot fill the
    GPU, key-range split when that balances better, one SM per unit otherwise."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("choices below assume 148 SMs")
    assert tg.attention_kernel([0, 2304], 16, 8, 128) == "attn_pair_kernel"
    assert tg.attention_kernel([0, 1280], 16, 8, 128) == "attn_pair_kernel"
    assert tg.attention_kernel([0, 1280], 12, 4, 128) == "attn_tc_kernel (key-range split)"
    assert tg.attention_kernel([0, 1280], 12, 4, 128, with_workspace=False) == "attn_tc_kernel"
    assert tg.attention_kernel([0, 8448], 16, 8, 128) == "attn_tc_kernel"
    assert tg.attention_kernel([0, 2304], 12, 4, 128, with_workspace=False) == "attn_tc_kernel"
    assert tg.attention_kernel([0, 2304], 16, 8, 64, with_workspace=False) == "attn_tc_kernel"
    assert tg.attention_kernel([0, 2304], 16, 8, 128, dtype="fp32") == "attn_simt_kernel"


def test_no_gpu_means_cuda_error_not_crash(L):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    bits = ctypes.c_uint32(0)
    assert L.tg_device_status(None, ctypes.byref(bits)) == CUDA


def test_budget_sweep_and_random_select_validation(L):
    cu, cu_p = _arr([0, 10])
    s, s_p = _arr([2])
    e, e_p = _arr([8])
    ks, ks_p = _arr([3, 4])
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE)
    f = L.tg_topk_select_multi
    assert f(FAKE, 1, cu_p, s_p, e_p, 0, ks_p, ptrs, None, None) == INVALID   # no budget
    assert f(FAKE, 1, cu_p, s_p, e_p, 9, ks_p, ptrs, None, None) == INVALID   # > TG_MAX_BUDGETS
    assert f(FAKE, 1, cu_p, s_p, e_p, 2, None, ptrs, None, None) == INVALID
    nulls = (ctypes.c_void_p * 2)(FAKE, None)
    assert f(FAKE, 1, cu_p, s_p, e_p, 2, ks_p, nulls, None, None) == INVALID  # budget 1 output
    bad, bad_p = _arr([3, -1])
    assert f(FAKE, 1, cu_p, s_p, e_p, 2, bad_p, ptrs, None, None) == INVALID  # negative budget
    assert f(None, 1, cu_p, s_p, e_p, 2, ks_p, ptrs, None, None) == INVALID   # scores
    r = L.tg_random_select
    k1, k1_p = _arr([3])
    assert r(None, 1, cu_p, s_p, e_p, k1_p, FAKE, FAKE, None) == INVALID      # keys
    assert r(FAKE, 1, cu_p, s_p, e_p, k1_p, None, FAKE, None) == INVALID      # output
    big, big_p = _arr([0, 400000])
    s0, s0_p = _arr([0])
    assert r(FAKE, 1, big_p, s0_p, s0_p, k1_p, FAKE, FAKE, None) == UNSUP     # too long


def test_attention_backward_validation(L):
    """The backward rejects bad arguments before launching anything."""
    _, ck = _arr([0, 300])
    need = ctypes.c_size_t(0)
    assert L.tg_attention_backward_workspace_bytes(1, ck, 16, ctypes.byref(need)) == OK
    # D for 300 rows x 16 heads plus the per-head accumulators, 256-byte rounded
    assert need.value >= 300 * 16 * 4 + 2 * 16 * 4 and need.value % 256 == 0
    assert L.tg_attention_backward_workspace_bytes(1, ck, 0, ctypes.byref(need)) == SHAPE
    assert L.tg_attention_backward_workspace_bytes(1, ck, 16, None) == INVALID
    L.tg_attention_backward_workspace_bytes(1, ck, 16, ctypes.byref(need))
    b = L.tg_gated_attention_backward

    def call(dtype=0, hq=16, hkv=8, dh=128, logsig=FAKE, lse=FAKE, ws=FAKE, ws_bytes=None,
             algo=0, q=FAKE):
        return b(q, FAKE, FAKE, dtype, 1, ck, hq, hkv, dh, logsig, FAKE, FAKE, FAKE, lse, FAKE,
                 FAKE, FAKE, FAKE, FAKE, ws, need.value if ws_bytes is None else ws_bytes, algo,
                 None)

    assert call(dtype=7) == DTYPE
    assert call(hkv=6) == SHAPE
    assert call(dh=96) == UNSUP
    assert call(algo=9) == INVALID
    assert call(logsig=None) == INVALID  # no bias, no gate gradient
    assert call(lse=None) == INVALID
    assert call(ws=None) == INVALID
    assert call(q=FAKE_ODD) == ALIGN
    assert call(ws_bytes=need.value - 16) == WORKSPACE
    assert b"needed" in L.tg_last_error_message()
    assert call(dtype=1, algo=2) == UNSUP  # tcgen05 needs bf16
    # nothing kept: nothing to do, nothing launched
    _, ck0 = _arr([0, 0])
    assert b(None, None, None, 0, 1, ck0, 16, 8, 128, None, None, None, None, None, None, None,
             None, None, None, None, 0, 0, None) == OK


def test_delta_scan_validation(L):
    """The gated delta scan rejects bad arguments before launching anything."""
    _, ck = _arr([0, 40, 90])
    f = L.tg_gated_delta_scan

    def call(dtype=0, batch=2, cu=ck, heads=4, d=128, eps=1e-6, q=FAKE, la=FAKE, state=FAKE):
        return f(q, FAKE, FAKE, dtype, la, FAKE, batch, cu, heads, d, eps, FAKE, state, None)

    assert call(dtype=5) == DTYPE
    assert call(heads=0) == SHAPE
    assert call(d=96) == UNSUP
    assert call(eps=-1.0) == INVALID
    assert call(eps=float("nan")) == INVALID
    assert call(q=None) == INVALID
    assert call(la=None) == INVALID
    assert call(q=FAKE_ODD) == ALIGN
    assert call(state=FAKE_ODD) == ALIGN
    assert call(batch=tg.MAX_BATCH + 1, cu=_arr(list(range(tg.MAX_BATCH + 2)))[1]) == UNSUP
    assert call(cu=_arr([0, 50, 40])[1]) == INVALID  # a prompt with a negative count
    assert call(cu=_arr([3, 50, 90])[1]) == INVALID
    # nothing kept and no state wanted: nothing to do
    _, ck0 = _arr([0, 0])
    assert f(None, None, None, 0, None, None, 1, ck0, 4, 64, 1e-6, None, None, None) == OK
    assert f(None, None, None, 0, None, None, 0, ck0, 4, 64, 1e-6, None, None, None) == OK


def test_delta_scan_launch_size_bound(L):
    """batch x heads x state slices beyond one launch's blocks is rejected."""
    cu, ck = _arr([0] * (tg.MAX_BATCH + 1))
    heads = (2 ** 31) // (tg.MAX_BATCH * 4) + 1
    assert L.tg_gated_delta_scan(None, None, None, 0, None, None, tg.MAX_BATCH, ck, heads, 128, 1e-6,
                                 None, FAKE, None) == UNSUP


def test_delta_scan_wrapper_rejects_mismatched_shapes():
    """The Python binding checks shapes before anything reaches the library."""
    import torch

    x = torch.zeros(6, 2, 64)
    a = torch.zeros(6, 2)
    with pytest.raises(ValueError, match="share one"):
        tg.gated_delta_scan(x, torch.zeros(6, 2, 32), x, [0, 6], a, a)
    with pytest.raises(ValueError, match=r"\[M, H\]"):
        tg.gated_delta_scan(x, x, x, [0, 6], torch.zeros(6, 3), a)
    with pytest.raises(ValueError, match="float32"):
        tg.gated_delta_scan(x, x, x, [0, 6], a.double(), a)
    with pytest.raises(ValueError, match="CUDA"):
        tg.gated_delta_scan(x, x, x, [0, 6], a, a)


def test_topk_workspace_size_and_fused_gate_validation(L):
    """The top-K workspace holds one 8448-byte block per prompt (2048 histogram
    bins and a tag); the fused gate and the workspace selection refuse a
    missing or short workspace and a batch that does not cover n_tokens,
    before anything launches."""
    assert L.tg_topk_workspace_bytes(1, 16384) == 8448
    assert L.tg_topk_workspace_bytes(4, 147456) == 4 * 8448
    assert L.tg_topk_workspace_bytes(0, 0) == 0
    assert L.tg_topk_workspace_bytes(129, 0) == 0
    _, cu_p = _arr([0, 100, 356])
    _, s_p = _arr([0, 0])
    _, e_p = _arr([90, 250])
    _, k_p = _arr([10, 20])
    gh = L.tg_gate_score_hist
    args = (FAKE, 0, 356, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 2, cu_p, s_p, e_p)
    assert gh(*args, None, 2 * 8448, 0, None) == INVALID        # no workspace
    assert gh(*args, FAKE, 2 * 8448 - 1, 0, None) == WORKSPACE  # one byte short
    assert gh(*args, FAKE_ODD, 2 * 8448, 0, None) == ALIGN
    bad = (FAKE, 0, 355, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 2, cu_p, s_p, e_p)
    assert gh(*bad, FAKE, 2 * 8448, 0, None) == SHAPE           # cu_seqlens ends at 356
    _, e_bad = _arr([101, 250])
    assert gh(FAKE, 0, 356, 64, FAKE, FAKE, 32, FAKE, 0.0, FAKE, 2, cu_p, s_p, e_bad, FAKE,
              2 * 8448, 0, None) == INVALID                     # span past its prompt
    ws = L.tg_topk_select_ws
    assert ws(FAKE, 2, cu_p, s_p, e_p, k_p, FAKE, FAKE, None, 2 * 8448, None) == INVALID
    assert ws(FAKE, 2, cu_p, s_p, e_p, k_p, FAKE, FAKE, FAKE, 8448, None) == WORKSPACE
