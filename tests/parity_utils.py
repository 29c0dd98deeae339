"""Shared helpers for the GPU parity tests (tolerances, device transfer, sampling)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances (|gpu - ref| <= atol + rtol*|ref|, element by element)
GATE_ATOL = 1e-3                  # gate scores, any dtype
ATTN_BF16 = (2e-2, 1e-2)          # attention output in bf16
ATTN_FP32 = (1e-4, 0.0)           # attention output in fp32
LSE_ATOL = 1e-3                   # fp32 log-sum-exp of the biased logits
LOGSIG_TOL = (1e-6, 1e-6)         # log sigmoid(z) computed in fp32
BF16_ULP_REL = 2.0 ** -7          # one bf16 ulp relative to the value (RoPE'd rows)


def assert_close(name, got, ref, atol, rtol):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{name}: {int(bad.sum())}/{bad.size} elements out of tolerance "
                             f"(atol={atol}, rtol={rtol}); max err {err.max():.3e}; first bad "
                             f"{idx.tolist()} got {got[tuple(idx[0])]} ref {ref[tuple(idx[0])]}")


def assert_rope_close(name, got_bf16, ref64):
    """RoPE'd rows: the GPU rotates in fp32 and rounds once to the storage dtype."""
    got = np.asarray(got_bf16, np.float64)
    err = np.abs(got - ref64)
    bound = BF16_ULP_REL * np.abs(ref64) + 1e-6
    bad = err > bound
    assert not bad.any(), f"{name}: {int(bad.sum())} elements beyond 1 bf16 ulp, max {err.max()}"


def dev(t, device="cuda"):
    return None if t is None else t.to(device, non_blocking=False).contiguous()


def host_f32(t):
    return t.detach().float().cpu().numpy()


def sample_rows(M, cu, n_random, seed, extra=()):
    """Query rows to check at full size: first/last rows of each prompt, tile
    boundaries (127/128/129 into a prompt), the end of the batch, and random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        if e <= s:
            continue
        for off in (0, 1, 126, 127, 128, 129, 255, 256):
            if s + off < e:
                rows.add(s + off)
        for off in (1, 2, 128, 129):
            if e - off >= s:
                rows.add(e - off)
    rows.update(int(x) for x in rng.integers(0, M, size=n_random))
    rows.update(int(x) for x in extra if 0 <= x < M)
    return np.array(sorted(rows), np.int64)


def kept_set_agrees(gpu_kept, ref_kept, z_ref, cu_seqlens, doc_begin, doc_end, budget, tol=1e-3):
    """Kept sets may differ only by document tokens whose oracle score lies within
    `tol` of that prompt's K-th largest document score."""
    g, r = set(gpu_kept.tolist()), set(ref_kept.tolist())
    diff = g ^ r
    if not diff:
        return True, 0
    for b in range(len(doc_begin)):
        s = int(cu_seqlens[b]) + int(doc_begin[b])
        e = int(cu_seqlens[b]) + int(doc_end[b])
        k = min(int(budget[b]), e - s)
        if k == 0 or k == e - s:
            continue
        kth = np.sort(z_ref[s:e])[::-1][k - 1]
        for x in diff:
            if s <= x < e and abs(z_ref[x] - kth) > tol:
                return False, len(diff)
    for x in diff:
        # a protected (question) token must never appear in the difference
        b = int(np.searchsorted(cu_seqlens, x, side="right") - 1)
        pos = x - int(cu_seqlens[b])
        if not (doc_begin[b] <= pos < doc_end[b]):
            return False, len(diff)
    return True, len(diff)
