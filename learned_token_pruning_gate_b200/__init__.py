"""TokenGate gated-prefill hot path for B200 (sm_100a).

Thin Python binding over ``libtokengate.so`` (C ABI in ``include/tokengate.h``).
This module only marshals arguments: torch tensors supply device memory and the
current CUDA stream, every step runs in the library's kernels.  There is no
fallback: if the library is missing or a call fails, an exception is raised.

The four calls follow the method's forward pass (TokenGate abstract page;
news write-ups, "how it works"):

    gate_score -> topk_select -> compact_gather -> gated_attention

``gated_prefill`` chains them for one prompt batch.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

__all__ = [
    "TG_BF16", "TG_FP32", "ALGO_AUTO", "ALGO_SIMT", "ALGO_TCGEN05", "TokenGateError",
    "library", "kept_offsets", "gate_score", "topk_select", "compact_gather", "gated_attention",
    "gated_prefill", "device_status", "EXPORTED_SYMBOLS", "attention_workspace_bytes",
    "attention_kernel", "topk_select_multi", "random_select", "gated_attention_backward",
    "attention_backward_workspace_bytes", "rmsnorm", "qkv_rope_emit", "swiglu", "gated_delta_scan",
    "topk_workspace_bytes", "topk_workspace", "delta_scan_workspace_bytes",
]

TG_BF16, TG_FP32 = 0, 1
ALGO_AUTO, ALGO_SIMT, ALGO_TCGEN05 = 0, 1, 2
MAX_BATCH = 128
MAX_GATHER_TENSORS = 8

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtokengate.so")

EXPORTED_SYMBOLS = (
    "tg_status_string", "tg_last_error_message", "tg_version", "tg_device_status",
    "tg_kept_offsets", "tg_gate_score", "tg_topk_select", "tg_compact_gather",
    "tg_gated_attention", "tg_attention_workspace_bytes", "tg_attention_kernel",
    "tg_gated_attention_noalloc", "tg_topk_select_multi", "tg_random_select",
    "tg_gated_attention_backward", "tg_attention_backward_workspace_bytes", "tg_rmsnorm",
    "tg_qkv_rope_emit", "tg_swiglu", "tg_gated_delta_scan", "tg_last_device_error",
    "tg_topk_workspace_bytes", "tg_gate_score_hist", "tg_topk_select_ws",
    "tg_gated_delta_scan_chunked", "tg_delta_scan_workspace_bytes", "tg_topk_select_multi_ws",
)
MAX_BUDGETS = 8
ATTN_KERNELS = {0: "attn_simt_kernel", 1: "attn_tc_kernel", 2: "attn_tc_kernel (key-range split)",
                3: "attn_pair_kernel"}


class TokenGateError(RuntimeError):
    """A libtokengate call returned an error status."""

    def __init__(self, fn, status, message):
        super().__init__(f"{fn}: {status}: {message}")
        self.status = status


class GatherTensor(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p),
                ("row_elems", ctypes.c_int32), ("rope_heads", ctypes.c_int32)]


_lib = None
_vp, _i32, _i64, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
_i32p = ctypes.POINTER(ctypes.c_int32)


def library():
    """Load libtokengate.so (built by ``python -m learned_token_pruning_gate_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m learned_token_pruning_gate_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.tg_status_string.restype = ctypes.c_char_p
    L.tg_status_string.argtypes = [ctypes.c_int]
    L.tg_last_error_message.restype = ctypes.c_char_p
    L.tg_version.restype = ctypes.c_char_p
    L.tg_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
    L.tg_last_device_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_int32)]
    L.tg_kept_offsets.argtypes = [_i32, _i32p, _i32p, _i32p, _i32p, _i32p]
    L.tg_gate_score.argtypes = [_vp, ctypes.c_int, _i64, _i32, _vp, _vp, _i32, _vp, _f32, _vp,
                                _i32, _vp]
    L.tg_topk_select.argtypes = [_vp, _i32, _i32p, _i32p, _i32p, _i32p, _vp, _vp, _vp]
    L.tg_topk_workspace_bytes.argtypes = [_i32, _i64]
    L.tg_gate_score_hist.argtypes = [_vp, ctypes.c_int, _i64, _i32, _vp, _vp, _i32, _vp, _f32,
                                     _vp, _i32, _i32p, _i32p, _i32p, _vp, ctypes.c_size_t, _i32,
                                     _vp]
    L.tg_topk_select_ws.argtypes = [_vp, _i32, _i32p, _i32p, _i32p, _i32p, _vp, _vp, _vp,
                                    ctypes.c_size_t, _vp]
    L.tg_topk_select_multi.argtypes = [_vp, _i32, _i32p, _i32p, _i32p, _i32, _i32p,
                                       ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp]
    L.tg_topk_select_multi_ws.argtypes = [_vp, _i32, _i32p, _i32p, _i32p, _i32, _i32p,
                                          ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp,
                                          ctypes.c_size_t, _vp]
    L.tg_random_select.argtypes = [_vp, _i32, _i32p, _i32p, _i32p, _i32p, _vp, _vp, _vp]
    L.tg_compact_gather.argtypes = [_vp, _i64, _i32, _i32p, _i32p, _i32p, _i32p, ctypes.c_int,
                                    ctypes.POINTER(GatherTensor), _i32, _i32, ctypes.c_double,
                                    _vp, _vp, _vp]
    L.tg_gated_attention.argtypes = [_vp, _vp, _vp, ctypes.c_int, _i32, _i32p, _i32, _i32, _i32,
                                     _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _i32, _vp]
    L.tg_attention_workspace_bytes.argtypes = [ctypes.c_int, _i32, _i32p, _i32, _i32, _i32, _i32,
                                               ctypes.POINTER(ctypes.c_size_t)]
    L.tg_attention_kernel.argtypes = [ctypes.c_int, _i32, _i32p, _i32, _i32, _i32, _i32, _i32,
                                      ctypes.POINTER(ctypes.c_int32)]
    L.tg_gated_attention_noalloc.argtypes = [_vp, _vp, _vp, ctypes.c_int, _i32, _i32p, _i32, _i32,
                                             _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
    L.tg_gated_attention_backward.argtypes = [_vp, _vp, _vp, ctypes.c_int, _i32, _i32p, _i32, _i32,
                                              _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                              _vp, _vp, ctypes.c_size_t, _i32, _vp]
    L.tg_attention_backward_workspace_bytes.argtypes = [_i32, _i32p, _i32,
                                                        ctypes.POINTER(ctypes.c_size_t)]
    L.tg_rmsnorm.argtypes = [_vp, _vp, _vp, ctypes.c_int, _i64, _i32, _f32, _vp]
    L.tg_qkv_rope_emit.argtypes = [_vp, ctypes.c_int, _i32, _i32p, _i32p, _vp, _i32, _i32, _i32,
                                   _vp, _vp, _f32, ctypes.c_double, _vp, _vp, _vp, _vp]
    L.tg_swiglu.argtypes = [_vp, _vp, ctypes.c_int, _i64, _i32, _vp]
    L.tg_gated_delta_scan.argtypes = [_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _i32, _i32p, _i32, _i32,
                                      _f32, _vp, _vp, _vp]
    L.tg_gated_delta_scan_chunked.argtypes = [_vp, _vp, _vp, ctypes.c_int, _vp, _vp, _i32, _i32p,
                                              _i32, _i32, _f32, _vp, _vp, _vp, ctypes.c_size_t,
                                              _vp]
    L.tg_delta_scan_workspace_bytes.argtypes = [_i32, _i32p, _i32, _i32,
                                                ctypes.POINTER(ctypes.c_size_t)]
    for name in EXPORTED_SYMBOLS:
        if name not in ("tg_status_string", "tg_last_error_message", "tg_version",
                        "tg_topk_workspace_bytes"):
            getattr(L, name).restype = ctypes.c_int
    L.tg_topk_workspace_bytes.restype = ctypes.c_size_t
    _lib = L
    return L


def _check(fn, status):
    if status != 0:
        L = library()
        raise TokenGateError(fn, L.tg_status_string(status).decode(),
                             L.tg_last_error_message().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _host_i32(a):
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.int32))
    return arr, arr.ctypes.data_as(_i32p)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return TG_BF16
    if t.dtype == torch.float32:
        return TG_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libtokengate operates on CUDA tensors only")


def _expect(name, t, shape, dtype, device):
    """A caller-passed tensor must match what the call reads or writes exactly:
    the kernels take raw pointers and trust the sizes derived from the other
    arguments, so a smaller buffer would be read or written past its end."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def device_status(stream=None):
    """Synchronise and return (and clear) the device status bits (0 = no failure)."""
    bits = ctypes.c_uint32(0)
    st = stream if stream is not None else _stream()
    rc = library().tg_device_status(st, ctypes.byref(bits))
    if rc not in (0, 7):
        _check("tg_device_status", rc)
    return bits.value


def kept_offsets(cu_seqlens, doc_begin, doc_end, budget) -> np.ndarray:
    """Host-side kept-row offsets cu_kept [B+1] (validates the prompt batch)."""
    cu, cu_p = _host_i32(cu_seqlens)
    s, s_p = _host_i32(doc_begin)
    e, e_p = _host_i32(doc_end)
    k, k_p = _host_i32(budget)
    out = np.zeros(len(s) + 1, np.int32)
    _check("tg_kept_offsets", library().tg_kept_offsets(len(s), cu_p, s_p, e_p, k_p,
                                                        out.ctypes.data_as(_i32p)))
    return out


def topk_workspace_bytes(batch, total_tokens=0):
    """Bytes of the top-K workspace (first-pass histograms) for `batch` prompts."""
    return int(library().tg_topk_workspace_bytes(int(batch), int(total_tokens)))


def topk_workspace(batch, device=None):
    """A zeroed top-K workspace for `batch` prompts (uint8 device tensor)."""
    return torch.zeros(topk_workspace_bytes(batch), dtype=torch.uint8, device=device or "cuda")


def gate_score(h, W1, b1, w2, b2, out=None, algo=ALGO_AUTO, topk_ws=None, cu_seqlens=None,
               doc_begin=None, doc_end=None):
    """z = w2 . GELU(W1 h + b1) + b2 for every row of h [n, d].

    With ``topk_ws`` (a zeroed top-K workspace) and the prompt spans, the gate
    also counts the selection's first radix pass into it (tg_gate_score_hist),
    for a following ``topk_select(..., workspace=topk_ws)``."""
    n, d = h.shape
    dg = W1.shape[0]
    if W1.shape[1] != d or W1.dtype != h.dtype:
        raise ValueError("W1 must be [d_hidden, d_model] with h's dtype")
    _expect("h", h, (n, d), h.dtype, h.device)
    _expect("W1", W1, (dg, d), h.dtype, h.device)
    _expect("b1", b1, (dg,), torch.float32, h.device)
    _expect("w2", w2, (dg,), torch.float32, h.device)
    _expect("out", out, (n,), torch.float32, h.device)
    _need_cuda(h, W1, b1, w2)
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=h.device)
    if topk_ws is None:
        _check("tg_gate_score", library().tg_gate_score(
            _ptr(h), _dtype_code(h), n, d, _ptr(W1), _ptr(b1), dg, _ptr(w2), float(b2),
            _ptr(out), algo, _stream(h.device)))
        return out
    if topk_ws.dtype != torch.uint8 or not topk_ws.is_contiguous() or topk_ws.device != h.device:
        raise ValueError("topk_ws must be a contiguous uint8 tensor on h's device")
    cu, cu_p = _host_i32(cu_seqlens)
    s, s_p = _host_i32(doc_begin)
    e, e_p = _host_i32(doc_end)
    _check("tg_gate_score_hist", library().tg_gate_score_hist(
        _ptr(h), _dtype_code(h), n, d, _ptr(W1), _ptr(b1), dg, _ptr(w2), float(b2), _ptr(out),
        len(s), cu_p, s_p, e_p, _ptr(topk_ws), topk_ws.numel(), algo, _stream(h.device)))
    return out


def topk_select(z, cu_seqlens, doc_begin, doc_end, budget, kept_idx=None, cu_kept=None,
                workspace=None):
    """Per-prompt top-K of the document span (question kept).

    ``workspace``: a top-K workspace, possibly holding the gate's first-pass
    histograms of these scores (tg_topk_select_ws); left zeroed.
    Returns (kept_idx [M] int32 device, cu_kept [B+1] int32 device, cu_kept_host).
    """
    cu, cu_p = _host_i32(cu_seqlens)
    s, s_p = _host_i32(doc_begin)
    e, e_p = _host_i32(doc_end)
    k, k_p = _host_i32(budget)
    host = kept_offsets(cu, s, e, k)
    M = int(host[-1])
    _expect("z", z, (int(cu[-1]),), torch.float32, z.device)
    _expect("kept_idx", kept_idx, (M,), torch.int32, z.device)
    _expect("cu_kept", cu_kept, (len(s) + 1,), torch.int32, z.device)
    if workspace is not None and (workspace.dtype != torch.uint8 or
                                  not workspace.is_contiguous() or workspace.device != z.device):
        raise ValueError("workspace must be a contiguous uint8 tensor on z's device")
    _need_cuda(z)
    if kept_idx is None:
        kept_idx = torch.empty(max(M, 1), dtype=torch.int32, device=z.device)[:M]
    if cu_kept is None:
        cu_kept = torch.empty(len(s) + 1, dtype=torch.int32, device=z.device)
    if workspace is None:
        _check("tg_topk_select", library().tg_topk_select(
            _ptr(z), len(s), cu_p, s_p, e_p, k_p, _ptr(kept_idx), _ptr(cu_kept),
            _stream(z.device)))
    else:
        _check("tg_topk_select_ws", library().tg_topk_select_ws(
            _ptr(z), len(s), cu_p, s_p, e_p, k_p, _ptr(kept_idx), _ptr(cu_kept), _ptr(workspace),
            workspace.numel(), _stream(z.device)))
    return kept_idx, cu_kept, host


def topk_select_multi(z, cu_seqlens, doc_begin, doc_end, budgets, workspace=None):
    """Top-K for a budget sweep from one score vector: budgets is a list of
    per-prompt budget lists (at most MAX_BUDGETS).  One launch.  With
    ``workspace`` (a top-K workspace the gate counted these scores into, see
    gate_score) every budget takes its first radix pass from that one histogram.

    Returns a list of (kept_idx [M_q] device, cu_kept [B+1] device, cu_kept_host).
    """
    _need_cuda(z)
    cu, cu_p = _host_i32(cu_seqlens)
    s, s_p = _host_i32(doc_begin)
    e, e_p = _host_i32(doc_end)
    _expect("z", z, (int(cu[-1]),), torch.float32, z.device)
    ks = np.ascontiguousarray(np.asarray(budgets, dtype=np.int32).reshape(len(budgets), len(s)))
    outs, kept_ptrs, cu_ptrs = [], (_vp * len(ks))(), (_vp * len(ks))()
    for q, k in enumerate(ks):
        host = kept_offsets(cu, s, e, k)
        M = int(host[-1])
        kept = torch.empty(max(M, 1), dtype=torch.int32, device=z.device)[:M]
        cuk = torch.empty(len(s) + 1, dtype=torch.int32, device=z.device)
        kept_ptrs[q], cu_ptrs[q] = kept.data_ptr() if M else None, cuk.data_ptr()
        outs.append((kept, cuk, host))
    if workspace is None:
        _check("tg_topk_select_multi", library().tg_topk_select_multi(
            _ptr(z), len(s), cu_p, s_p, e_p, len(ks), ks.ctypes.data_as(_i32p), kept_ptrs,
            cu_ptrs, _stream(z.device)))
        return outs
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or \
            workspace.device != z.device:
        raise ValueError("workspace must be a contiguous uint8 tensor on z's device")
    _check("tg_topk_select_multi_ws", library().tg_topk_select_multi_ws(
        _ptr(z), len(s), cu_p, s_p, e_p, len(ks), ks.ctypes.data_as(_i32p), kept_ptrs, cu_ptrs,
        _ptr(workspace), workspace.numel(), _stream(z.device)))
    return outs


def random_select(keys, cu_seqlens, doc_begin, doc_end, budget):
    """Random-K selection from caller-drawn uint32 keys (a device tensor of
    torch.int32 holding the key bits, one per token): the K document tokens with
    the largest keys, question kept.  Returns (kept_idx, cu_kept, cu_kept_host)."""
    _need_cuda(keys)
    cu, cu_p = _host_i32(cu_seqlens)
    s, s_p = _host_i32(doc_begin)
    e, e_p = _host_i32(doc_end)
    k, k_p = _host_i32(budget)
    host = kept_offsets(cu, s, e, k)
    M = int(host[-1])
    _expect("keys", keys, (int(cu[-1]),), torch.int32, keys.device)
    kept_idx = torch.empty(max(M, 1), dtype=torch.int32, device=keys.device)[:M]
    cu_kept = torch.empty(len(s) + 1, dtype=torch.int32, device=keys.device)
    _check("tg_random_select", library().tg_random_select(
        _ptr(keys), len(s), cu_p, s_p, e_p, k_p, _ptr(kept_idx), _ptr(cu_kept),
        _stream(keys.device)))
    return kept_idx, cu_kept, host


def compact_gather(kept_idx, cu_seqlens, doc_begin, doc_end, budget, tensors, rope_heads=None,
                   head_dim=0, rope_theta=1e6, z=None, logsig_out=None, outs=None):
    """Gather kept rows of each tensor in ``tensors`` (RoPE where rope_heads[i] > 0).

    Returns (list of compacted tensors, logsig [M] fp32 or None).
    """
    if len(tensors) > MAX_GATHER_TENSORS:
        raise ValueError("too many tensors")
    cu, cu_p = _host_i32(cu_seqlens)
    s, s_p = _host_i32(doc_begin)
    e, e_p = _host_i32(doc_end)
    k, k_p = _host_i32(budget)
    M = kept_idx.shape[0]
    dtypes = {t.dtype for t in tensors}
    if len(dtypes) > 1:
        raise ValueError("all gathered tensors must share one dtype")
    dcode = _dtype_code(tensors[0]) if tensors else TG_BF16
    rope_heads = rope_heads or [0] * len(tensors)
    dev0 = tensors[0].device if tensors else kept_idx.device
    _expect("kept_idx", kept_idx, (M,), torch.int32, dev0)
    N = int(cu[-1])
    for i, t in enumerate(tensors):
        _expect(f"tensors[{i}]", t, (N,) + tuple(t.shape[1:]), tensors[0].dtype, dev0)
    if z is not None:
        _expect("z", z, (N,), torch.float32, dev0)
    if outs is None:
        outs = [torch.empty((M,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
                for t in tensors]
    if len(outs) != len(tensors):
        raise ValueError("one output per gathered tensor")
    for i, (t, o) in enumerate(zip(tensors, outs)):
        _expect(f"outs[{i}]", o, (M,) + tuple(t.shape[1:]), t.dtype, dev0)
    if logsig_out is not None:
        _expect("logsig_out", logsig_out, (M,), torch.float32, dev0)
    _need_cuda(kept_idx, z, *tensors)
    arr = (GatherTensor * max(len(tensors), 1))()
    for i, (src, dst) in enumerate(zip(tensors, outs)):
        if not src.is_contiguous() or not dst.is_contiguous():
            raise ValueError("gather tensors must be contiguous")
        arr[i].src = src.data_ptr()
        arr[i].dst = dst.data_ptr()
        arr[i].row_elems = src[0].numel() if src.shape[0] > 0 else int(np.prod(src.shape[1:]))
        arr[i].rope_heads = int(rope_heads[i])
    if z is not None and logsig_out is None:
        logsig_out = torch.empty(M, dtype=torch.float32, device=z.device)
    dev = (tensors[0].device if tensors else z.device)
    _check("tg_compact_gather", library().tg_compact_gather(
        _ptr(kept_idx), M, len(s), cu_p, s_p, e_p, k_p, dcode, arr, len(tensors), head_dim,
        float(rope_theta), _ptr(z), _ptr(logsig_out), _stream(dev)))
    return outs, logsig_out


def _attention_operands(q, k, v, logsig, gain, temp):
    """q [M, Hq, d], k and v [M, Hkv, d] of one dtype on one device, contiguous;
    logsig [M], gain and temp [Hq] fp32.  The kernels read k and v with q's
    element size and row count, so any mismatch would read past their end."""
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k and v must be [rows, heads, head_dim]")
    M, Hq, dh = q.shape
    Hkv = k.shape[1]
    if Hkv <= 0 or Hq % Hkv != 0:
        raise ValueError(f"{Hq} query heads are not a multiple of {Hkv} kv heads")
    _expect("q", q, (M, Hq, dh), q.dtype, q.device)
    _expect("k", k, (M, Hkv, dh), q.dtype, q.device)
    _expect("v", v, (M, Hkv, dh), q.dtype, q.device)
    _expect("logsig", logsig, (M,), torch.float32, q.device)
    _expect("gain", gain, (Hq,), torch.float32, q.device)
    _expect("temp", temp, (Hq,), torch.float32, q.device)


def attention_workspace_bytes(cu_kept_host, n_q_heads, n_kv_heads, head_dim, dtype="bf16",
                              algo=ALGO_AUTO):
    """Workspace bytes tg_gated_attention may use for this batch on the current device."""
    cu, cu_p = _host_i32(cu_kept_host)
    code = 0 if dtype in ("bf16", torch.bfloat16) else 1
    out = ctypes.c_size_t(0)
    _check("tg_attention_workspace_bytes", library().tg_attention_workspace_bytes(
        code, len(cu) - 1, cu_p, n_q_heads, n_kv_heads, head_dim, algo, ctypes.byref(out)))
    return int(out.value)


def attention_kernel(cu_kept_host, n_q_heads, n_kv_heads, head_dim, dtype="bf16",
                     algo=ALGO_AUTO, with_workspace=True):
    """Name of the attention kernel tg_gated_attention launches for this batch."""
    cu, cu_p = _host_i32(cu_kept_host)
    code = 0 if dtype in ("bf16", torch.bfloat16) else 1
    out = ctypes.c_int32(-1)
    _check("tg_attention_kernel", library().tg_attention_kernel(
        code, len(cu) - 1, cu_p, n_q_heads, n_kv_heads, head_dim, algo, int(with_workspace),
        ctypes.byref(out)))
    return ATTN_KERNELS[out.value]


def gated_attention(q, k, v, cu_kept_host, logsig=None, gain=None, temp=None, out=None,
                    lse=None, algo=ALGO_AUTO, want_lse=False, workspace="auto"):
    """Token-gated causal GQA attention over packed kept rows.

    q [M, Hq, d], k/v [M, Hkv, d]; cu_kept_host [B+1] host offsets.
    workspace: "auto" (allocate what the call can use), None (no split), or a
    uint8 device tensor.  Returns (out [M, Hq, d], lse [Hq, M] or None).
    """
    _attention_operands(q, k, v, logsig, gain, temp)
    M, Hq, dh = q.shape
    Hkv = k.shape[1]
    cu, cu_p = _host_i32(cu_kept_host)
    if int(cu[-1]) != M:
        raise ValueError(f"cu_kept_host ends at {int(cu[-1])}, q has {M} rows")
    _expect("out", out, (M, Hq, dh), q.dtype, q.device)
    _expect("lse", lse, (Hq, M), torch.float32, q.device)
    if workspace is not None and not isinstance(workspace, str):
        if workspace.dtype != torch.uint8 or not workspace.is_contiguous() or \
                workspace.device != q.device:
            raise ValueError("workspace must be a contiguous uint8 tensor on q's device")
    _need_cuda(q, k, v, logsig, gain, temp)
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((Hq, M), dtype=torch.float32, device=q.device)
    if isinstance(workspace, str):
        nbytes = attention_workspace_bytes(cu, Hq, Hkv, dh, q.dtype, algo)
        workspace = (torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None)
    ws_bytes = 0 if workspace is None else workspace.numel()
    _check("tg_gated_attention", library().tg_gated_attention(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), len(cu) - 1, cu_p, Hq, Hkv, dh, _ptr(logsig),
        _ptr(gain), _ptr(temp), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, algo,
        _stream(q.device)))
    return out, lse


def attention_backward_workspace_bytes(cu_kept_host, n_q_heads):
    """Device scratch bytes gated_attention_backward needs for this batch."""
    cu, cu_p = _host_i32(cu_kept_host)
    out = ctypes.c_size_t(0)
    _check("tg_attention_backward_workspace_bytes", library().tg_attention_backward_workspace_bytes(
        len(cu) - 1, cu_p, n_q_heads, ctypes.byref(out)))
    return int(out.value)


def gated_attention_backward(q, k, v, cu_kept_host, logsig, gain, temp, out, lse, dout,
                             algo=ALGO_AUTO, workspace=None):
    """Gradient of a loss through gated_attention with respect to the log-gates
    (and the kept rows' gate scores), the gains and the temperatures.

    dout = dL/dout [M, Hq, d]; out, lse = the forward's outputs (lse [Hq, M]).
    Returns (d_logsig [M], d_z_kept [M], d_gain [Hq], d_temp [Hq]), fp32 device.
    """
    _attention_operands(q, k, v, logsig, gain, temp)
    M, Hq, dh = q.shape
    Hkv = k.shape[1]
    if logsig is None or lse is None:
        raise ValueError("the backward needs the log-gates and the forward's lse")
    _expect("out", out, (M, Hq, dh), q.dtype, q.device)
    _expect("dout", dout, (M, Hq, dh), q.dtype, q.device)
    _expect("lse", lse, (Hq, M), torch.float32, q.device)
    cu, cu_p = _host_i32(cu_kept_host)
    if int(cu[-1]) != M:
        raise ValueError(f"cu_kept_host ends at {int(cu[-1])}, q has {M} rows")
    if workspace is not None and (workspace.dtype != torch.uint8 or
                                  not workspace.is_contiguous() or workspace.device != q.device):
        raise ValueError("workspace must be a contiguous uint8 tensor on q's device")
    _need_cuda(q, k, v, logsig, gain, temp, out, lse, dout)
    if workspace is None:
        workspace = torch.empty(attention_backward_workspace_bytes(cu, Hq), dtype=torch.uint8,
                                device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    d_l, d_z = torch.empty(M, **f32), torch.empty(M, **f32)
    d_g, d_t = torch.empty(Hq, **f32), torch.empty(Hq, **f32)
    _check("tg_gated_attention_backward", library().tg_gated_attention_backward(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), len(cu) - 1, cu_p, Hq, Hkv, dh, _ptr(logsig),
        _ptr(gain), _ptr(temp), _ptr(out), _ptr(lse), _ptr(dout), _ptr(d_l), _ptr(d_z), _ptr(d_g),
        _ptr(d_t), _ptr(workspace), workspace.numel(), algo, _stream(q.device)))
    return d_l, d_z, d_g, d_t


def rmsnorm(x, weight, eps=1e-6, out=None):
    """x / sqrt(mean(x^2) + eps) * weight over the last axis of x [rows, dim]."""
    rows, dim = x.shape
    _expect("x", x, (rows, dim), x.dtype, x.device)
    _expect("weight", weight, (dim,), x.dtype, x.device)
    _expect("out", out, (rows, dim), x.dtype, x.device)
    _need_cuda(x, weight)
    if out is None:
        out = torch.empty_like(x)
    _check("tg_rmsnorm", library().tg_rmsnorm(_ptr(x), _ptr(weight), _ptr(out), _dtype_code(x),
                                              rows, dim, eps, _stream(x.device)))
    return out


def qkv_rope_emit(qkv, cu_seqlens, cu_kept_host, kept_idx, n_q_heads, n_kv_heads, head_dim,
                  q_norm_w, k_norm_w, eps=1e-6, rope_theta=1e6, q_out=None, k_out=None,
                  v_out=None):
    """Split a fused QKV projection [M, (Hq + 2 Hkv) d] into q (per-head RMSNorm,
    RoPE), k (same; the layer's KV-cache slot) and v.  Returns (q, k, v)."""
    M = qkv.shape[0]
    cu, cu_p = _host_i32(cu_seqlens)
    ck, ck_p = _host_i32(cu_kept_host)
    if int(ck[-1]) != M:
        raise ValueError(f"cu_kept_host ends at {int(ck[-1])}, qkv has {M} rows")
    _expect("qkv", qkv, (M, (n_q_heads + 2 * n_kv_heads) * head_dim), qkv.dtype, qkv.device)
    _expect("kept_idx", kept_idx, (M,), torch.int32, qkv.device)
    _expect("q_norm_w", q_norm_w, (head_dim,), qkv.dtype, qkv.device)
    _expect("k_norm_w", k_norm_w, (head_dim,), qkv.dtype, qkv.device)
    _expect("q_out", q_out, (M, n_q_heads, head_dim), qkv.dtype, qkv.device)
    _expect("k_out", k_out, (M, n_kv_heads, head_dim), qkv.dtype, qkv.device)
    _expect("v_out", v_out, (M, n_kv_heads, head_dim), qkv.dtype, qkv.device)
    _need_cuda(qkv, kept_idx, q_norm_w, k_norm_w)
    mk = lambda h: torch.empty((M, h, head_dim), dtype=qkv.dtype, device=qkv.device)  # noqa: E731
    q_out = mk(n_q_heads) if q_out is None else q_out
    k_out = mk(n_kv_heads) if k_out is None else k_out
    v_out = mk(n_kv_heads) if v_out is None else v_out
    _check("tg_qkv_rope_emit", library().tg_qkv_rope_emit(
        _ptr(qkv), _dtype_code(qkv), len(cu) - 1, cu_p, ck_p, _ptr(kept_idx), n_q_heads, n_kv_heads,
        head_dim, _ptr(q_norm_w), _ptr(k_norm_w), eps, float(rope_theta), _ptr(q_out), _ptr(k_out),
        _ptr(v_out), _stream(qkv.device)))
    return q_out, k_out, v_out


def swiglu(gate_up, out=None):
    """SiLU(gate) * up of a fused [rows, 2 inter] projection."""
    rows, two = gate_up.shape
    if two % 2:
        raise ValueError("gate_up must hold the gate and up halves side by side")
    _expect("gate_up", gate_up, (rows, two), gate_up.dtype, gate_up.device)
    _expect("out", out, (rows, two // 2), gate_up.dtype, gate_up.device)
    _need_cuda(gate_up)
    if out is None:
        out = torch.empty((rows, two // 2), dtype=gate_up.dtype, device=gate_up.device)
    _check("tg_swiglu", library().tg_swiglu(_ptr(gate_up), _ptr(out), _dtype_code(gate_up), rows,
                                            two // 2, _stream(gate_up.device)))
    return out


def delta_scan_workspace_bytes(cu_kept_host, n_heads, head_dim):
    """Device scratch bytes the chunked delta-rule scan needs for this batch."""
    ck, ck_p = _host_i32(cu_kept_host)
    out = ctypes.c_size_t(0)
    _check("tg_delta_scan_workspace_bytes", library().tg_delta_scan_workspace_bytes(
        len(ck) - 1, ck_p, int(n_heads), int(head_dim), ctypes.byref(out)))
    return int(out.value)


def gated_delta_scan(q, k, v, cu_kept_host, log_alpha, beta, eps=1e-6, out=None, state=None,
                     want_state=True, algo="chunked", workspace=None):
    """Gated delta rule over each prompt's kept rows (a Gated DeltaNet layer above the
    gate): q, k, v [M, H, d] (d 64 or 128), log_alpha, beta [M, H] fp32.  Returns
    (o [M, H, d], state [B, H, d, d] fp32 or None).

    algo: "chunked" (tg_gated_delta_scan_chunked: parallel within chunks of 64
    rows; ``workspace`` a uint8 device tensor of delta_scan_workspace_bytes, or
    None to allocate one) or "recurrent" (tg_gated_delta_scan: row by row)."""
    if algo not in ("chunked", "recurrent"):
        raise ValueError(f"algo {algo!r}: 'chunked' or 'recurrent'")
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError(f"q, k, v must share one [M, H, d] shape: {tuple(q.shape)}, "
                         f"{tuple(k.shape)}, {tuple(v.shape)}")
    M, H, d = q.shape
    if tuple(log_alpha.shape) != (M, H) or tuple(beta.shape) != (M, H):
        raise ValueError(f"log_alpha and beta must be [M, H] = {(M, H)}")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise ValueError("log_alpha and beta must be float32")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(name, t, (M, H, d), q.dtype, q.device)
    _expect("log_alpha", log_alpha, (M, H), torch.float32, q.device)
    _expect("beta", beta, (M, H), torch.float32, q.device)
    ck, ck_p = _host_i32(cu_kept_host)
    if int(ck[-1]) != M:
        raise ValueError(f"cu_kept_host ends at {int(ck[-1])}, q has {M} rows")
    B = len(ck) - 1
    _expect("out", out, (M, H, d), q.dtype, q.device)
    _expect("state", state, (B, H, d, d), torch.float32, q.device)
    _need_cuda(q, k, v, log_alpha, beta)
    if out is None:
        out = torch.empty_like(v)
    if state is None and want_state:
        state = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if algo == "recurrent":
        _check("tg_gated_delta_scan", library().tg_gated_delta_scan(
            _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta), B, ck_p, H, d,
            float(eps), _ptr(out), _ptr(state) if state is not None else None,
            _stream(q.device)))
        return out, state
    if workspace is None:
        nbytes = delta_scan_workspace_bytes(ck, H, d)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
    elif workspace.dtype != torch.uint8 or not workspace.is_contiguous() or \
            workspace.device != q.device:
        raise ValueError("workspace must be a contiguous uint8 tensor on q's device")
    _check("tg_gated_delta_scan_chunked", library().tg_gated_delta_scan_chunked(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta), B, ck_p, H, d,
        float(eps), _ptr(out), _ptr(state) if state is not None else None, _ptr(workspace),
        workspace.numel(), _stream(q.device)))
    return out, state


def gated_prefill(h, q, k, v, W1, b1, w2, b2, gain, temp, cu_seqlens, doc_begin, doc_end,
                  budget, rope_theta=1e6, algo=ALGO_AUTO, want_lse=False):
    """One gated layer: score (with the selection's first radix pass), select,
    compact, attend.  Returns a dict of device tensors."""
    B = len(np.asarray(doc_begin))
    ws = topk_workspace(B, device=h.device) if B > 0 else None
    z = gate_score(h, W1, b1, w2, b2, algo=algo, topk_ws=ws, cu_seqlens=cu_seqlens,
                   doc_begin=doc_begin, doc_end=doc_end)
    kept_idx, cu_kept, cu_kept_host = topk_select(z, cu_seqlens, doc_begin, doc_end, budget,
                                                  workspace=ws)
    Hq, dh = q.shape[1], q.shape[2]
    (h_c, q_c, k_c, v_c), logsig = compact_gather(
        kept_idx, cu_seqlens, doc_begin, doc_end, budget, [h, q, k, v],
        rope_heads=[0, Hq, k.shape[1], 0], head_dim=dh, rope_theta=rope_theta, z=z)
    o, lse = gated_attention(q_c, k_c, v_c, cu_kept_host, logsig, gain, temp, algo=algo,
                             want_lse=want_lse)
    return dict(z=z, kept_idx=kept_idx, cu_kept=cu_kept, cu_kept_host=cu_kept_host, h=h_c, q=q_c,
                k=k_c, v=v_c, logsig=logsig, out=o, lse=lse)
