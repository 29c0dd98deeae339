"""Seeded synthetic inputs for the gated-prefill hot path.

This module only draws numbers: it holds none of the method's arithmetic and
is the one piece of code that both the CUDA path's callers (tests, bench) and
the CPU oracle's callers share.  Every workload is fully determined by its
seed.  The pages measure on long-context tasks (RepoBench-P,
2WikiMultihopQA, MultiNews, BioDEX, needle-in-a-haystack) with trained
weights; none of that data is used.  Instead a block of "needle" residual rows
is pushed along the gate's first-order sensitive direction so that, with
random weights, those tokens score highest -- the structure of a
needle-in-a-haystack prompt, not its content.

Prompt layout: each prompt is [document | question]; the document span is
prunable, the question is always kept (pages: the document part of the prompt,
marked by a ``{state}`` placeholder, is the only part pruned).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

NEEDLE_BETA = 4.0  # needle strength in units of sqrt(d) along the sensitive direction


@dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple            # tokens per prompt
    question: tuple           # question tokens per prompt (at the end of the prompt)
    budgets: tuple            # max_kept_prefill_tokens per prompt (document tokens kept)
    d_model: int
    d_hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    dtype: str                # "bf16" or "fp32"
    needle: int               # needle block length per prompt
    seed: int
    rope_theta: float = 1e6

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    def kept_lengths(self):
        return [min(k, n - q) + q for n, q, k in zip(self.seqlens, self.question, self.budgets)]


def _w(name, seqlens, question, budgets, dtype, seed, d=2048, dg=256, hq=16, hkv=8, dh=128,
       needle=64):
    return Workload(name, tuple(seqlens), tuple(question), tuple(budgets), d, dg, hq, hkv, dh,
                    dtype, needle, seed)


# The five workloads: a tiny fp32 case and four Qwen3-1.7B-shaped bf16 layers.
WORKLOADS = {
    "tiny_fp32": _w("tiny_fp32", [1024], [64], [256], "fp32", 0, d=256, dg=64, hq=4, hkv=2,
                    dh=64, needle=32),
    "qwen_16k": _w("qwen_16k", [16384], [256], [2048], "bf16", 1),
    "qwen_32k_k1024": _w("qwen_32k_k1024", [32768], [256], [1024], "bf16", 2),
    "qwen_32k_k4096": _w("qwen_32k_k4096", [32768], [256], [4096], "bf16", 2),
    "qwen_32k_k8192": _w("qwen_32k_k8192", [32768], [256], [8192], "bf16", 2),
    "qwen_128k": _w("qwen_128k", [131072], [256], [8192], "bf16", 3),
    "ragged_4": _w("ragged_4", [8192, 24576, 49152, 65536], [128, 256, 384, 512],
                   [1024, 3072, 6144, 8192], "bf16", 4),
}


def scaled(w: Workload, factor: int, name=None) -> Workload:
    """Same structure with every length and budget divided by ``factor``."""
    seq = tuple(max(n // factor, 8) for n in w.seqlens)
    q = tuple(max(min(qq // factor, n // 2), 1) for qq, n in zip(w.question, seq))
    k = tuple(max(kk // factor, 1) for kk in w.budgets)
    return Workload(name or f"{w.name}/{factor}", seq, q, k, w.d_model, w.d_hidden, w.n_q_heads,
                    w.n_kv_heads, w.head_dim, w.dtype, max(min(w.needle, min(k) // 2), 1),
                    w.seed, w.rope_theta)


@dataclass
class Inputs:
    """Host-side tensors (torch CPU, storage dtype) plus prompt metadata."""
    w: Workload
    cu_seqlens: np.ndarray    # [B+1] int32
    doc_begin: np.ndarray     # [B] int32, relative to each prompt start
    doc_end: np.ndarray       # [B] int32
    budget: np.ndarray        # [B] int32
    needle_rows: list         # per prompt: global row ids of the needle block
    h: torch.Tensor           # [N, d]
    W1: torch.Tensor          # [dg, d]
    b1: torch.Tensor          # [dg] fp32
    w2: torch.Tensor          # [dg] fp32
    b2: float
    q: torch.Tensor           # [N, Hq, dh]
    k: torch.Tensor           # [N, Hkv, dh]
    v: torch.Tensor           # [N, Hkv, dh]
    gain: torch.Tensor        # [Hq] fp32
    temp: torch.Tensor        # [Hq] fp32
    extra: dict = field(default_factory=dict)

    def f32(self, name) -> np.ndarray:
        """A tensor's stored values widened to float32 (exact for bf16)."""
        return getattr(self, name).float().numpy()


def _tdtype(s):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[s]


def _normal(rng, shape, std=1.0):
    return rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)


_CHUNK_ROWS = 4096


def _normal_rows(seed, stream, shape, dtype):
    """N(0, 1) rows of a large tensor, drawn in chunks of _CHUNK_ROWS rows, chunk c
    from its own Philox stream keyed by (seed, stream, c): the values depend only
    on the seed, and the chunks are drawn on several threads (numpy releases the
    GIL while it fills an array).  Returned as a torch tensor of ``dtype``."""
    import concurrent.futures as cf
    import os

    n = shape[0]
    row = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(n, row)

    def chunk(c):
        lo, hi = c * _CHUNK_ROWS, min(n, (c + 1) * _CHUNK_ROWS)
        g = np.random.Generator(np.random.Philox(key=[seed, (stream << 32) | c]))
        block = g.standard_normal(size=(hi - lo, row), dtype=np.float32)
        flat[lo:hi] = torch.from_numpy(block).to(dtype)

    n_chunks = (n + _CHUNK_ROWS - 1) // _CHUNK_ROWS
    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(chunk, range(n_chunks)))
    return out


def make_inputs(w: Workload, with_qkv: bool = True) -> Inputs:
    """Draw every input of workload ``w`` from its seed (numpy Philox)."""
    rng = np.random.Generator(np.random.Philox(w.seed))
    dt = _tdtype(w.dtype)
    B = w.batch
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum(np.asarray(w.seqlens, np.int64)).astype(np.int32)
    doc_begin = np.zeros(B, np.int32)
    doc_end = np.asarray([n - q for n, q in zip(w.seqlens, w.question)], np.int32)
    budget = np.asarray(w.budgets, np.int32)

    W1 = torch.from_numpy(_normal(rng, (w.d_hidden, w.d_model), 0.02)).to(dt)
    b1 = torch.from_numpy(_normal(rng, (w.d_hidden,), 0.02))
    w2 = torch.from_numpy(_normal(rng, (w.d_hidden,), 0.02))
    b2 = float(_normal(rng, (1,), 0.02)[0])

    # the residual rows in fp32 first: the needle is added before the rounding
    h32 = _normal_rows(w.seed, 1, (w.total_tokens, w.d_model), torch.float32)
    # Needle direction: W1^T w2 (the residual direction that raises the hidden
    # units with positive output weight and lowers the others), unit length.
    W1f = W1.float().numpy()
    direction = W1f.T.astype(np.float64) @ w2.numpy().astype(np.float64)
    direction /= np.linalg.norm(direction)
    push = torch.from_numpy((NEEDLE_BETA * np.sqrt(w.d_model) * direction).astype(np.float32))
    needle_rows = []
    for b in range(B):
        n_doc = int(doc_end[b] - doc_begin[b])
        ln = min(w.needle, n_doc)
        off = int(rng.integers(0, max(n_doc - ln, 0) + 1))
        rows = np.arange(cu[b] + doc_begin[b] + off, cu[b] + doc_begin[b] + off + ln)
        h32[torch.from_numpy(rows)] += push
        needle_rows.append(rows.astype(np.int64))
    h = h32.to(dt)
    del h32

    N = w.total_tokens
    if with_qkv:
        q = _normal_rows(w.seed, 2, (N, w.n_q_heads, w.head_dim), dt)
        k = _normal_rows(w.seed, 3, (N, w.n_kv_heads, w.head_dim), dt)
        v = _normal_rows(w.seed, 4, (N, w.n_kv_heads, w.head_dim), dt)
    else:
        q = k = v = None
    gain = torch.from_numpy(rng.uniform(0.0, 1.0, w.n_q_heads).astype(np.float32))
    temp = torch.from_numpy(rng.uniform(0.8, 1.2, w.n_q_heads).astype(np.float32))
    return Inputs(w, cu, doc_begin, doc_end, budget, needle_rows, h, W1, b1, w2, b2, q, k, v,
                  gain, temp)


def random_keys(n: int, seed: int, bits: int = 32) -> np.ndarray:
    """i.i.d. uniform uint32 keys from a counter-based generator (Philox): the
    random numbers the random-K selector draws.  bits < 32 leaves only the low
    bits random, to plant many exact ties."""
    rng = np.random.Generator(np.random.Philox(seed))
    k = rng.integers(0, 1 << 32, n, dtype=np.uint64).astype(np.uint32)
    return k & np.uint32((1 << bits) - 1) if bits < 32 else k


def random_scores(n: int, seed: int, ties: bool = True, specials: bool = True) -> np.ndarray:
    """fp32 gate-score-like values with planted exact ties, +-0.0, +-inf and NaN."""
    rng = np.random.Generator(np.random.Philox(seed))
    z = _normal(rng, (n,), 0.2)
    if ties and n > 8:
        # quantise a third of the values so many exact ties exist
        sel = rng.random(n) < 0.33
        z[sel] = np.round(z[sel] * 64) / 64
    if specials and n > 16:
        idx = rng.choice(n, size=min(n // 16, 64), replace=False)
        pool = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-45, -1e-45], np.float32)
        z[idx] = pool[rng.integers(0, len(pool), size=idx.shape[0])]
    return z


def stack_inputs(M_list, n_layers, d_model, Hq, Hkv, dh, inter, seed, dtype="bf16", pos_span=4):
    """A compacted residual, the kept rows' original positions, log-gates and the
    random-init weights of n_layers Qwen3-shaped upper layers (stage-level tests
    and the stack benchmark).  Positions: sorted distinct draws from
    [0, pos_span * M_b) per prompt (a kept set of about 1 row in pos_span)."""
    rng = np.random.Generator(np.random.Philox(seed + 104729))
    dt = _tdtype(dtype)
    M = int(sum(M_list))
    cu = np.zeros(len(M_list) + 1, np.int32)
    cu[1:] = np.cumsum(M_list)
    pos = np.concatenate([np.sort(rng.choice(max(pos_span * m, 1), size=m, replace=False))
                          for m in M_list]).astype(np.int32) if M else np.zeros(0, np.int32)
    x0 = torch.from_numpy(_normal(rng, (M, d_model))).to(dt)
    ls = torch.from_numpy(-np.abs(_normal(rng, (M,), 2.0)))
    w = lambda *shape: torch.from_numpy(_normal(rng, shape, 0.02)).to(dt)  # noqa: E731
    norm_w = lambda n: torch.from_numpy((1.0 + _normal(rng, (n,), 0.1)).astype(np.float32)).to(dt)  # noqa: E731
    layers = []
    for _ in range(n_layers):
        layers.append(dict(
            w_ln1=norm_w(d_model), wqkv=w((Hq + 2 * Hkv) * dh, d_model), w_qn=norm_w(dh),
            w_kn=norm_w(dh), wo=w(d_model, Hq * dh), w_ln2=norm_w(d_model), wg=w(inter, d_model),
            wu=w(inter, d_model), wd=w(d_model, inter),
            gain=torch.from_numpy(rng.uniform(0.0, 1.0, Hq).astype(np.float32)),
            temp=torch.from_numpy(rng.uniform(0.8, 1.2, Hq).astype(np.float32))))
    return cu, pos, x0, ls, layers


def attention_output_grad(M, Hq, dh, seed, dtype="bf16"):
    """A seeded upstream gradient dL/dout [M, Hq, dh] for the attention backward."""
    rng = np.random.Generator(np.random.Philox(seed + 7919))
    return torch.from_numpy(_normal(rng, (M, Hq, dh))).to(_tdtype(dtype))


def attention_inputs(M_list, Hq, Hkv, dh, seed, dtype="bf16", bias=True):
    """Compacted-layout attention inputs drawn directly (for stage-level tests)."""
    rng = np.random.Generator(np.random.Philox(seed))
    dt = _tdtype(dtype)
    M = int(sum(M_list))
    cu = np.zeros(len(M_list) + 1, np.int32)
    cu[1:] = np.cumsum(M_list)
    q = torch.from_numpy(_normal(rng, (M, Hq, dh))).to(dt)
    k = torch.from_numpy(_normal(rng, (M, Hkv, dh))).to(dt)
    v = torch.from_numpy(_normal(rng, (M, Hkv, dh))).to(dt)
    # log-sigmoid-like bias values: non-positive, heavier near zero
    ls = torch.from_numpy(-np.abs(_normal(rng, (M,), 2.0))) if bias else None
    gain = torch.from_numpy(rng.uniform(0.0, 1.0, Hq).astype(np.float32))
    temp = torch.from_numpy(rng.uniform(0.8, 1.2, Hq).astype(np.float32))
    return cu, q, k, v, ls, gain, temp


def delta_inputs(M_list, H, d, seed, dtype="bf16", decay=0.1):
    """Kept-row inputs of a gated-delta-rule layer: q, k, v [M, H, d] ~ N(0, 1) in
    `dtype`; log_alpha = -U(0, decay) (per-token decays alpha in (e^-decay, 1]);
    beta = sigmoid(N(0, 1)) [M, H] fp32."""
    rng = np.random.Generator(np.random.Philox(seed))
    dt = _tdtype(dtype)
    M = int(sum(M_list))
    cu = np.zeros(len(M_list) + 1, np.int32)
    cu[1:] = np.cumsum(M_list)
    q = torch.from_numpy(_normal(rng, (M, H, d))).to(dt)
    k = torch.from_numpy(_normal(rng, (M, H, d))).to(dt)
    v = torch.from_numpy(_normal(rng, (M, H, d))).to(dt)
    la = torch.from_numpy(-rng.uniform(0.0, decay, (M, H)).astype(np.float32))
    beta = torch.from_numpy((1.0 / (1.0 + np.exp(-_normal(rng, (M, H))))).astype(np.float32))
    return cu, q, k, v, la, beta
