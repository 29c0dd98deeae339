"""tg_gated_attention_noalloc: the gated attention for callers that cannot
allocate device memory (for example a server whose allocator owns the whole
GPU, or code that must not allocate around CUDA-graph capture).  It takes the
scratch of the key-range split from an array built into the library instead of
a caller workspace.  Its results must match tg_gated_attention with a
workspace, call after call.  Some cases below split (their plan needs scratch,
so the built-in array and the reset of its counters are exercised); one needs
more than the array's 32 MiB and must run the unsplit plan instead.  This file
is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import learned_token_pruning_gate_b200 as tg
from learned_token_pruning_gate_b200 import inputs as gen
from tests.parity_utils import ATTN_BF16, LSE_ATOL, assert_close, dev, host_f32


def _noalloc(q, k, v, cu, ls, gain, temp, out, lse):
    cu_h = np.ascontiguousarray(cu, np.int32)
    L = tg.library()
    st = L.tg_gated_attention_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        0, len(cu_h) - 1, cu_h.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), q.shape[1],
        k.shape[1], q.shape[2], ctypes.c_void_p(ls.data_ptr()), ctypes.c_void_p(gain.data_ptr()),
        ctypes.c_void_p(temp.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), tg.ALGO_AUTO,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, (L.tg_status_string(st), L.tg_last_error_message())


SCRATCH_BYTES = 32 << 20
CASES = [([1000], 16, 8), ([2304], 16, 8), ([5, 0, 260, 1, 640], 16, 8), ([8448], 16, 8),
         ([1280], 12, 4), ([2304], 12, 4), ([15000], 4, 2)]


def test_cases_cover_split_and_oversize_plans():
    """Host-only: the planner sizes these cases the same way on any machine with
    148 SMs (a B200; the host planner assumes 148 without a device)."""
    need = [tg.attention_workspace_bytes(np.array([0, *np.cumsum(l)], np.int32), hq, hkv, 128)
            for l, hq, hkv in CASES]
    assert any(0 < n <= SCRATCH_BYTES for n in need), need
    assert any(n > SCRATCH_BYTES for n in need), need


@pytest.mark.gpu
@pytest.mark.parametrize("lens,Hq,Hkv", CASES)
def test_noalloc_matches_workspace_call_twice(lens, Hq, Hkv):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dh = 128
    cu, q, k, v, ls, gain, temp = gen.attention_inputs(lens, Hq, Hkv, dh, 31 + len(lens), "bf16",
                                                       True)
    q, k, v, ls, gain, temp = (dev(x) for x in (q, k, v, ls, gain, temp))
    ref, ref_lse = tg.gated_attention(q, k, v, cu, ls, gain, temp, want_lse=True,
                                      workspace="auto")
    for _ in range(2):  # the built-in scratch keeps the previous call's contents
        out = torch.full_like(q, float("nan"))
        lse = torch.full((Hq, q.shape[0]), float("nan"), dtype=torch.float32, device=q.device)
        _noalloc(q, k, v, cu, ls, gain, temp, out, lse)
        torch.cuda.synchronize()
        assert_close("noalloc out", host_f32(out), host_f32(ref), *ATTN_BF16)
        assert_close("noalloc lse", lse.cpu().numpy(), ref_lse.cpu().numpy(), LSE_ATOL, 1e-5)
    assert tg.device_status() == 0
