"""Plain fp64 oracle of a stack of gated upper layers (test infrastructure; only
the tests, ``__graft_entry__.smoke()`` and the bench's CPU baseline use it).

TokenGate keeps one set of tokens for every layer above the gate: the layers
above L "process only the kept tokens" and create no KV entry for the others
([KO] "작동 방식", [IT] "Come funziona"), and each of their attention layers adds
the gate's bias with its own learned gain and temperature ([PT] "TokenGate
'ensina' o modelo a folhear o texto"; [ABS]).  The upper layers here are
Qwen3-shaped decoder layers with random weights (the pages' backbone is
Qwen3-1.7B; its checkpoints are not used):

    a   = RMSNorm(x) * w_ln1
    q, k, v = split(a Wqkv^T);  q, k = RMSNorm_head(q) * w_qn, RMSNorm_head(k) * w_kn
    q, k = RoPE(q, pos), RoPE(k, pos)   (rotate-half pairs, angle pos * theta^(-2i/d))
    cache_k[l], cache_v[l] = k, v       (the compacted KV cache the stack emits)
    o   = gated attention(q, k, v; l_j, g_l, tau_l)   (causal within each prompt)
    x  += o Wo^T
    b   = RMSNorm(x) * w_ln2
    x  += (SiLU(b Wg^T) * (b Wu^T)) Wd^T

Every step is the plain definition in fp64 with numpy (matrix products are
library calls); nothing is blocked or fused.  Positions are the kept rows'
original positions inside their prompt.
"""
from __future__ import annotations

import numpy as np


def rmsnorm(x, w, eps=1e-6):
    """x / sqrt(mean(x^2) + eps) * w over the last axis."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def silu(x):
    x = np.asarray(x, np.float64)
    return x / (1.0 + np.exp(-x))


def rope(x, pos, theta):
    """Rotate-half RoPE of x [M, H, d] at positions pos [M]."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half) / d)
    ang = np.asarray(pos, np.float64)[:, None] * inv[None, :]  # [M, half]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x0, x1 = x[..., :half], x[..., half:]
    return np.concatenate([x0 * c - x1 * s, x1 * c + x0 * s], axis=-1)


def gated_attention(q, k, v, cu_kept, logsig, gain, temp):
    """softmax_j(q_i.k_j / (sqrt(d) tau_h) + g_h l_j) v_j over keys j <= i of the
    same prompt; q [M, Hq, d], k/v [M, Hkv, d]."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    M, Hq, d = q.shape
    group = Hq // k.shape[1]
    out = np.zeros_like(q)
    ls = np.asarray(logsig, np.float64)
    for b in range(len(cu_kept) - 1):
        s, e = int(cu_kept[b]), int(cu_kept[b + 1])
        if e == s:
            continue
        mask = np.tril(np.ones((e - s, e - s), bool))
        for h in range(Hq):
            kh, vh = k[s:e, h // group], v[s:e, h // group]
            lg = q[s:e, h] @ kh.T / (np.sqrt(d) * float(temp[h])) + float(gain[h]) * ls[None, s:e]
            lg = np.where(mask, lg, -np.inf)
            lg -= lg.max(axis=1, keepdims=True)
            p = np.exp(lg)
            p /= p.sum(axis=1, keepdims=True)
            out[s:e, h] = p @ vh
    return out


def stack(x0, pos, cu_kept, logsig, layers, n_q_heads, n_kv_heads, head_dim, theta=1e6, eps=1e-6):
    """Run the upper layers over the kept rows.

    layers: list of dicts with w_ln1 [dm], wqkv [(Hq+2Hkv) d, dm], w_qn [d], w_kn [d],
    wo [dm, Hq d], w_ln2 [dm], wg [I, dm], wu [I, dm], wd [dm, I], gain [Hq], temp [Hq].
    Returns (x [M, dm], cache_k [L, M, Hkv, d], cache_v [L, M, Hkv, d]) in fp64.
    """
    x = np.array(x0, np.float64)
    M = x.shape[0]
    Hq, Hkv, d = n_q_heads, n_kv_heads, head_dim
    ck, cv = [], []
    for ly in layers:
        a = rmsnorm(x, ly["w_ln1"], eps)
        qkv = a @ np.asarray(ly["wqkv"], np.float64).T
        q = qkv[:, :Hq * d].reshape(M, Hq, d)
        k = qkv[:, Hq * d:(Hq + Hkv) * d].reshape(M, Hkv, d)
        v = qkv[:, (Hq + Hkv) * d:].reshape(M, Hkv, d)
        q = rope(rmsnorm(q, ly["w_qn"], eps), pos, theta)
        k = rope(rmsnorm(k, ly["w_kn"], eps), pos, theta)
        ck.append(k)
        cv.append(v)
        o = gated_attention(q, k, v, cu_kept, logsig, ly["gain"], ly["temp"])
        x = x + o.reshape(M, Hq * d) @ np.asarray(ly["wo"], np.float64).T
        b = rmsnorm(x, ly["w_ln2"], eps)
        hmid = silu(b @ np.asarray(ly["wg"], np.float64).T) * (b @ np.asarray(ly["wu"], np.float64).T)
        x = x + hmid @ np.asarray(ly["wd"], np.float64).T
    return x, np.stack(ck) if ck else np.zeros((0, M, Hkv, d)), np.stack(cv) if cv else np.zeros((0, M, Hkv, d))
