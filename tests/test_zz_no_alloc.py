"""tg_gated_attention_noalloc: the gated attention for callers that cannot
allocate device memory (for example a server whose allocator owns the whole
GPU, or code that must not allocate around CUDA-graph capture).  It takes the
scratch of the key-range split from an array built into the library instead of
a caller workspace.  Its results must match tg_gated_attention with a
workspace, call after call.  This file is collected last on purpose."""
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


@pytest.mark.gpu
@pytest.mark.parametrize("lens,Hq,Hkv", [([1000], 16, 8), ([2304], 16, 8), ([5, 0, 260, 1, 640], 16, 8),
                                         ([8448], 16, 8), ([1280], 12, 4), ([2304], 12, 4)])
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
