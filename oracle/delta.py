"""Plain fp64 oracle of a gated-delta-rule layer over the kept rows (test
infrastructure; only the tests, ``__graft_entry__.smoke()`` and the bench's CPU
baseline use it).

TokenGate also prunes the Gated DeltaNet layers of a hybrid backbone (Qwen3.5-2B
mixes them with full-attention layers): tokens dropped at the gate never enter
the layers above it, linear-attention layers included ([KO] "성능 결과", its
comparison table; [FR] body; [ABS]).  The pages do not write the layer out.  The
reading taken here is the published gated delta rule (Yang, Kautz and
Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta Rule", 2024),
run over each prompt's kept rows in their original order, with the state
starting at zero and no gate bias (the pages add the bias to attention logits,
and this layer has none):

    q^_t = q_t / sqrt(|q_t|^2 + eps) / sqrt(d_k),   k^_t = k_t / sqrt(|k_t|^2 + eps)
    S_t  = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k^_t) k^_t^T     (S: d_v x d_k)
    o_t  = S_t q^_t

per head, with alpha_t = exp(log_alpha_t) in (0, 1] and beta_t in [0, 1].  The
final S of each prompt and head is the layer's state for decoding (the analogue
of the compacted KV cache an attention layer emits).

``scan`` is the recurrence step by step.  ``scan_closed_form`` is an
independent statement of the same function used to pin it: unrolling the
recurrence gives S_t = sum_{s<=t} (g_t / g_s) u_s k^_s^T with g_t = prod_{r<=t}
alpha_r and u_t = beta_t (v_t - sum_{s<t} (g_t / g_s) (k^_s . k^_t) u_s), a unit
lower-triangular system (I + A) U = diag(beta) V solved with a library solver.
``scan_chunked`` states the same function chunk by chunk (the form a parallel kernel
takes: the state before a chunk enters every row's equation of that chunk).
"""
from __future__ import annotations

import numpy as np


def _normalise(x, eps):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def scan(q, k, v, log_alpha, beta, cu_kept, eps=1e-6):
    """q, k [M, H, d_k], v [M, H, d_v], log_alpha, beta [M, H]; cu_kept [B+1].

    Returns (o [M, H, d_v], state [B, H, d_v, d_k]) in fp64."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    la = np.asarray(log_alpha, np.float64)
    be = np.asarray(beta, np.float64)
    M, H, dk = q.shape
    dv = v.shape[2]
    qn = _normalise(q, eps) / np.sqrt(dk)
    kn = _normalise(k, eps)
    o = np.zeros((M, H, dv))
    B = len(cu_kept) - 1
    state = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk))
            for t in range(int(cu_kept[b]), int(cu_kept[b + 1])):
                a = np.exp(la[t, h])
                kt = kn[t, h]
                S = a * S + be[t, h] * np.outer(v[t, h] - a * (S @ kt), kt)
                o[t, h] = S @ qn[t, h]
            state[b, h] = S
    return o, state


def scan_closed_form(q, k, v, log_alpha, beta, cu_kept, eps=1e-6):
    """The same outputs from the unrolled form (triangular solve per prompt and head)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    la = np.asarray(log_alpha, np.float64)
    be = np.asarray(beta, np.float64)
    M, H, dk = q.shape
    dv = v.shape[2]
    qn = _normalise(q, eps) / np.sqrt(dk)
    kn = _normalise(k, eps)
    o = np.zeros((M, H, dv))
    B = len(cu_kept) - 1
    state = np.zeros((B, H, dv, dk))
    for b in range(B):
        r0, r1 = int(cu_kept[b]), int(cu_kept[b + 1])
        n = r1 - r0
        if n == 0:
            continue
        for h in range(H):
            K = kn[r0:r1, h]
            Q = qn[r0:r1, h]
            V = v[r0:r1, h]
            lg = np.cumsum(la[r0:r1, h])  # log g_t
            on_or_below = np.tril(np.ones((n, n), dtype=bool))
            # g_t / g_s for s <= t (0 above the diagonal, never exp of a positive sum)
            decay = np.exp(np.where(on_or_below, lg[:, None] - lg[None, :], -np.inf))
            A = be[r0:r1, h][:, None] * decay * (K @ K.T) * np.tril(np.ones((n, n)), -1)
            U = np.linalg.solve(np.eye(n) + A, be[r0:r1, h][:, None] * V)
            o[r0:r1, h] = (decay * (Q @ K.T)) @ U
            state[b, h] = (np.exp(lg[-1] - lg)[:, None] * U).T @ K
    return o, state


def scan_chunked(q, k, v, log_alpha, beta, cu_kept, chunk=16, eps=1e-6):
    """The same outputs computed chunk by chunk, the form a parallel kernel takes:
    with S_0 the state before a chunk and g_t = prod of alpha from the chunk's start,
    u_t = beta_t (v_t - g_t S_0 k^_t - sum_{s<t} (g_t/g_s) (k^_s . k^_t) u_s) (a unit
    lower-triangular solve), o_t = g_t S_0 q^_t + sum_{s<=t} (g_t/g_s) (k^_s . q^_t) u_s,
    and the state after the chunk g_C S_0 + sum_s (g_C/g_s) u_s k^_s^T."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    la = np.asarray(log_alpha, np.float64)
    be = np.asarray(beta, np.float64)
    M, H, dk = q.shape
    dv = v.shape[2]
    qn = _normalise(q, eps) / np.sqrt(dk)
    kn = _normalise(k, eps)
    o = np.zeros((M, H, dv))
    B = len(cu_kept) - 1
    state = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dv, dk))
            for c0 in range(int(cu_kept[b]), int(cu_kept[b + 1]), chunk):
                c1 = min(c0 + chunk, int(cu_kept[b + 1]))
                n = c1 - c0
                K, Q, V, bt = kn[c0:c1, h], qn[c0:c1, h], v[c0:c1, h], be[c0:c1, h]
                lg = np.cumsum(la[c0:c1, h])
                g = np.exp(lg)
                on_or_below = np.tril(np.ones((n, n), dtype=bool))
                decay = np.exp(np.where(on_or_below, lg[:, None] - lg[None, :], -np.inf))
                A = bt[:, None] * decay * (K @ K.T) * np.tril(np.ones((n, n)), -1)
                U = np.linalg.solve(np.eye(n) + A, bt[:, None] * (V - g[:, None] * (K @ S.T)))
                o[c0:c1, h] = g[:, None] * (Q @ S.T) + (decay * (Q @ K.T)) @ U
                S = g[-1] * S + (np.exp(lg[-1] - lg)[:, None] * U).T @ K
            state[b, h] = S
    return o, state
