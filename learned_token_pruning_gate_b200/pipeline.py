"""A gated layer with preallocated device buffers.

``GatedLayer`` owns the device outputs of one prompt batch's gated prefill
(scores, kept indices, compacted residual/q/k/v, bias term, attention output)
and holds every C-ABI argument pre-marshalled, so ``run()`` is exactly four
library calls on one stream with no allocation and no host synchronisation --
the form that CUDA-graph capture and per-kernel timing need.  The gate counts
the selection's first radix pass into the layer's top-K workspace
(tg_gate_score_hist), and the selection starts from it (tg_topk_select_ws).
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import (ALGO_AUTO, GatherTensor, _check, _dtype_code, _host_i32,
               attention_workspace_bytes, gated_attention, kept_offsets, library, qkv_rope_emit,
               rmsnorm, swiglu, topk_workspace_bytes)


class GatedLayer:
    def __init__(self, h, q, k, v, W1, b1, w2, b2, gain, temp, cu_seqlens, doc_begin, doc_end,
                 budget, rope_theta=1e6, algo=ALGO_AUTO, want_lse=False):
        self.L = library()
        self.h, self.q, self.k, self.v = h, q, k, v
        self.W1, self.b1, self.w2, self.b2 = W1, b1, w2, float(b2)
        self.gain, self.temp = gain, temp
        self.algo = algo
        dev = h.device
        self.N, self.d = h.shape
        self.dg = W1.shape[0]
        self.Hq, self.dh = q.shape[1], q.shape[2]
        self.Hkv = k.shape[1]
        self.theta = float(rope_theta)
        self.cu, self.cu_p = _host_i32(cu_seqlens)
        self.s, self.s_p = _host_i32(doc_begin)
        self.e, self.e_p = _host_i32(doc_end)
        self.kb, self.k_p = _host_i32(budget)
        self.B = len(self.s)
        self.cu_kept_host, self.ck_p = _host_i32(kept_offsets(self.cu, self.s, self.e, self.kb))
        self.M = int(self.cu_kept_host[-1])
        f32 = dict(dtype=torch.float32, device=dev)
        self.z = torch.empty(self.N, **f32)
        self.kept_idx = torch.empty(max(self.M, 1), dtype=torch.int32, device=dev)
        self.cu_kept = torch.empty(self.B + 1, dtype=torch.int32, device=dev)
        self.h_c = torch.empty((self.M, self.d), dtype=h.dtype, device=dev)
        self.q_c = torch.empty((self.M, self.Hq, self.dh), dtype=q.dtype, device=dev)
        self.k_c = torch.empty((self.M, self.Hkv, self.dh), dtype=k.dtype, device=dev)
        self.v_c = torch.empty((self.M, self.Hkv, self.dh), dtype=v.dtype, device=dev)
        self.logsig = torch.empty(max(self.M, 1), **f32)
        self.out = torch.empty_like(self.q_c)
        self.lse = torch.empty((self.Hq, self.M), **f32) if want_lse else None
        ws = attention_workspace_bytes(self.cu_kept_host, self.Hq, self.Hkv, self.dh, q.dtype, algo)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev) if ws else None
        self.ws_bytes = ws
        # the top-K workspace: the gate counts the selection's first radix pass
        # into it, the selection reads it and leaves it zeroed (zero to start)
        self.topk_ws_bytes = topk_workspace_bytes(self.B) if self.B > 0 else 0
        self.topk_ws = torch.zeros(max(self.topk_ws_bytes, 1), dtype=torch.uint8, device=dev)
        self.dcode = _dtype_code(h)
        self.tensors = (GatherTensor * 4)()
        for i, (src, dst, heads) in enumerate([(h, self.h_c, 0), (q, self.q_c, self.Hq),
                                               (k, self.k_c, self.Hkv), (v, self.v_c, 0)]):
            self.tensors[i].src = src.data_ptr()
            self.tensors[i].dst = dst.data_ptr()
            self.tensors[i].row_elems = int(np.prod(src.shape[1:]))
            self.tensors[i].rope_heads = heads
        vp = ctypes.c_void_p
        self._p = {n: vp(t.data_ptr()) for n, t in dict(
            h=h, q=q, k=k, v=v, W1=W1, b1=b1, w2=w2, gain=gain, temp=temp, z=self.z,
            kept=self.kept_idx, cu_kept=self.cu_kept, q_c=self.q_c, k_c=self.k_c, v_c=self.v_c,
            logsig=self.logsig, out=self.out, topk_ws=self.topk_ws).items()}
        self._p["ws"] = vp(self.workspace.data_ptr()) if self.workspace is not None else None
        self._p["lse"] = vp(self.lse.data_ptr()) if self.lse is not None else None

    # each step is one C-ABI call; `stream` is a raw cudaStream_t handle
    def gate(self, stream):
        p = self._p
        if self.topk_ws_bytes == 0:
            _check("tg_gate_score", self.L.tg_gate_score(
                p["h"], self.dcode, self.N, self.d, p["W1"], p["b1"], self.dg, p["w2"], self.b2,
                p["z"], self.algo, stream))
            return
        _check("tg_gate_score_hist", self.L.tg_gate_score_hist(
            p["h"], self.dcode, self.N, self.d, p["W1"], p["b1"], self.dg, p["w2"], self.b2,
            p["z"], self.B, self.cu_p, self.s_p, self.e_p, p["topk_ws"], self.topk_ws_bytes,
            self.algo, stream))

    def topk(self, stream):
        p = self._p
        if self.topk_ws_bytes == 0:
            _check("tg_topk_select", self.L.tg_topk_select(
                p["z"], self.B, self.cu_p, self.s_p, self.e_p, self.k_p, p["kept"],
                p["cu_kept"], stream))
            return
        _check("tg_topk_select_ws", self.L.tg_topk_select_ws(
            p["z"], self.B, self.cu_p, self.s_p, self.e_p, self.k_p, p["kept"], p["cu_kept"],
            p["topk_ws"], self.topk_ws_bytes, stream))

    def gather(self, stream):
        p = self._p
        _check("tg_compact_gather", self.L.tg_compact_gather(
            p["kept"], self.M, self.B, self.cu_p, self.s_p, self.e_p, self.k_p, self.dcode,
            self.tensors, 4, self.dh, self.theta, p["z"], p["logsig"], stream))

    def attention(self, stream):
        p = self._p
        _check("tg_gated_attention", self.L.tg_gated_attention(
            p["q_c"], p["k_c"], p["v_c"], self.dcode, self.B, self.ck_p, self.Hq, self.Hkv,
            self.dh, p["logsig"], p["gain"], p["temp"], p["out"], p["lse"], p["ws"], self.ws_bytes,
            self.algo, stream))

    STAGES = ("gate", "topk", "gather", "attention")

    def run(self, stream=None):
        st = ctypes.c_void_p(stream if stream is not None
                             else torch.cuda.current_stream().cuda_stream)
        self.gate(st)
        self.topk(st)
        self.gather(st)
        self.attention(st)

    def capture(self):
        """Capture run() into a CUDA graph on a side stream; returns the graph."""
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.run(s.cuda_stream)  # warm: sets kernel attributes outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            self.run(s.cuda_stream)
        torch.cuda.synchronize()
        return g

    # algorithmic work of one step (for roofline fractions)
    def work(self):
        esz = self.h.element_size()
        row_bytes = esz * (self.d + (self.Hq + 2 * self.Hkv) * self.dh)
        lens = np.diff(self.cu_kept_host).astype(np.float64)
        attn_flops = float(np.sum(2.0 * self.dh * self.Hq * lens * (lens + 1)))
        return dict(
            gate_flops=2.0 * self.N * self.d * self.dg,
            gate_bytes=float(self.N * self.d * esz + self.dg * self.d * esz + 4 * self.N),
            topk_bytes=float(4 * self.N + 4 * self.M),
            gather_bytes=float(2 * self.M * row_bytes + 4 * self.M * 3),
            attn_flops=attn_flops,
            attn_bytes=float(self.M * row_bytes - self.M * self.d * esz
                             + self.M * self.Hq * self.dh * esz + 4 * self.M),
        )


class GatedStack:
    """Upper layers above the gate over the kept rows: every layer reuses the kept
    set and the log-gates, with its own gain and temperature, and emits its k and
    v (post-RoPE) into a compacted KV cache [layers, M, Hkv, d].  Qwen3-shaped
    layers (RMSNorm, fused QKV, per-head q/k RMSNorm, RoPE at the original
    positions, gated attention, output projection, RMSNorm, SwiGLU MLP); the
    projections are cuBLAS GEMMs (torch.mm), every other step a libtokengate call.

    layers: list of dicts of device tensors w_ln1, wqkv, w_qn, w_kn, wo, w_ln2, wg,
    wu, wd (dtype of the activations), gain, temp (fp32).
    """

    def __init__(self, layers, n_q_heads, n_kv_heads, head_dim, cu_seqlens, cu_kept_host, kept_idx,
                 logsig, rope_theta=1e6, eps=1e-6):
        self.layers = layers
        self.Hq, self.Hkv, self.dh = n_q_heads, n_kv_heads, head_dim
        self.cu = np.asarray(cu_seqlens, np.int32)
        self.ck = np.asarray(cu_kept_host, np.int32)
        self.kept_idx, self.logsig = kept_idx, logsig
        self.theta, self.eps = rope_theta, eps
        self.M = int(self.ck[-1])
        # fused [gate; up] weight per layer: one GEMM for both
        self.wgu = [torch.cat([ly["wg"], ly["wu"]], 0) for ly in layers]
        dev, dt = layers[0]["wqkv"].device, layers[0]["wqkv"].dtype
        L, M = len(layers), self.M
        self.cache_k = torch.empty((L, M, n_kv_heads, head_dim), dtype=dt, device=dev)
        self.cache_v = torch.empty((L, M, n_kv_heads, head_dim), dtype=dt, device=dev)
        self.q = torch.empty((M, n_q_heads, head_dim), dtype=dt, device=dev)
        self.o = torch.empty((M, n_q_heads, head_dim), dtype=dt, device=dev)
        nbytes = attention_workspace_bytes(self.ck, n_q_heads, n_kv_heads, head_dim, dt)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None

    def run(self, x):
        """x [M, d_model] (overwritten with the stack's output); returns (x, cache_k, cache_v)."""
        M, Hq = self.M, self.Hq
        for i, ly in enumerate(self.layers):
            a = rmsnorm(x, ly["w_ln1"], self.eps)
            qkv = torch.mm(a, ly["wqkv"].t())
            qkv_rope_emit(qkv, self.cu, self.ck, self.kept_idx, Hq, self.Hkv, self.dh, ly["w_qn"],
                             ly["w_kn"], self.eps, self.theta, q_out=self.q,
                             k_out=self.cache_k[i], v_out=self.cache_v[i])
            gated_attention(self.q, self.cache_k[i], self.cache_v[i], self.ck, self.logsig,
                               ly["gain"], ly["temp"], out=self.o, workspace=self.ws)
            x.addmm_(self.o.view(M, Hq * self.dh), ly["wo"].t())
            b = rmsnorm(x, ly["w_ln2"], self.eps)
            x.addmm_(swiglu(torch.mm(b, self.wgu[i].t())), ly["wd"].t())
        return x, self.cache_k, self.cache_v
