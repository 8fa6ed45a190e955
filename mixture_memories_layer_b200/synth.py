"""Seeded synthetic inputs for the Mixture-of-Memories layer.

This module draws random tensors and nothing else: it holds none of the
layer's arithmetic (no routing, projection, recurrence or combine), so both
the CUDA path and the CPU oracle may take their inputs from it.

Shapes and distributions follow the workloads the MoM pages describe
("MoM: Linear Sequence Modeling with Mixture-of-Memories", paper card,
Summary and Key points: 380M / 1.3B models, 4 memories with 2 active plus a
shared memory, memory-count scaling to 16):

* weights ~ N(0, 1/d_model) for the router, W_q, the shared and per-memory
  W_k / W_v, W_beta and W_a;
* A ~ U(0, 2.7) and b_a ~ U(-4, 0) per head (the log-decay parameters);
* X ~ N(0, 1); the router bias is zero, except in the skewed workload where
  memory 0 gets +2;
* varlen workloads draw sequence lengths U{512..2048} until the packed batch
  reaches the token budget, the last length clipped to the remainder;
* with per-memory gates, each routed memory's W_beta, W_a ~ N(0, 1/d_model),
  A ~ U(0, 2.7), b_a ~ U(-4, 0), from a stream of their own;
* with the Gated DeltaNet block around the memories, from a stream of their
  own: the output gate W_g ~ N(0, 1/d_model), the output projection W_o ~
  N(0, 1/(H d)), the short convolutions' weights (width 4, one filter per
  channel of q, k, v, shared and per memory) ~ U(-1/2, 1/2) (the default
  initialisation of a depthwise convolution of width 4: bound 1/sqrt(4)),
  float32, and the norm weight ~ U(0.5, 1.5) per head channel, float32.

Storage layout of every projection weight is [out_features, in_features]
(y = x @ W.T).  In bf16 workloads every array that the kernels read as bf16
is rounded to bf16 here, so both sides see bit-identical values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int          # sequences (decode: sequences stepped together)
    seq_len: int        # tokens per sequence (0 for varlen / decode)
    d_model: int
    heads: int
    d_head: int         # d_k = d_v
    n_mem: int          # routed memories M
    top_k: int
    dtype: str          # "f32" or "bf16" for activations / weights
    seed: int
    router_bias0: float = 0.0   # added to memory 0's router bias
    varlen_total: int = 0       # >0: packed varlen batch of this many tokens
    varlen_min: int = 512
    varlen_max: int = 2048
    decode_steps: int = 0       # >0: recurrent decode workload
    prefill_len: int = 0
    mem_gates: bool = False     # every routed memory has its own W_beta, W_a, A, b_a
    block: bool = False         # the Gated DeltaNet block around the memories (conv, norm, gate, W_o)
    conv_width: int = 4         # taps of the block's short convolutions

    @property
    def n_tokens(self) -> int:
        if self.varlen_total:
            return self.varlen_total
        if self.decode_steps:
            return self.batch
        return self.batch * self.seq_len


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 layer: the case the oracle finishes in well under a second
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 256, 2, 64, 4, 2, "f32", seed=0),
    # 380M-shape layer forward, balanced routing
    "mom380m": Workload("mom380m", 8, 2048, 1024, 4, 256, 4, 2, "bf16", seed=1),
    # 380M shape, skewed routing (+2 router bias on memory 0), varlen packing
    "mom380m_skew_varlen": Workload("mom380m_skew_varlen", 0, 0, 1024, 4, 256, 4, 2,
                                    "bf16", seed=2, router_bias0=2.0,
                                    varlen_total=16384),
    # the 380M-shape layer inside its Gated DeltaNet block (the same tokens and
    # memory weights as mom380m, the block's weights from a stream of their own)
    "mom380m_block": Workload("mom380m_block", 8, 2048, 1024, 4, 256, 4, 2, "bf16", seed=1, block=True),
    # 1.3B-shape memory-scaling forward: 16 memories, top-4
    "mom1p3b_m16": Workload("mom1p3b_m16", 4, 4096, 2048, 8, 256, 16, 4, "bf16", seed=3),
    # recurrent decode: 256 sequences, 8 memories top-2, one token per step
    "decode_b256": Workload("decode_b256", 256, 0, 1024, 4, 256, 8, 2, "bf16", seed=4,
                            decode_steps=512, prefill_len=256),
}


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _act(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return bf16_round(a) if dtype == "bf16" else a


def varlen_lengths(rng: np.random.Generator, total: int, lo: int, hi: int) -> np.ndarray:
    lens = []
    acc = 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    return np.asarray(lens, dtype=np.int64)


def make_cu_seqlens(w: Workload, rng: Optional[np.random.Generator] = None) -> np.ndarray:
    if w.varlen_total:
        lens = varlen_lengths(rng, w.varlen_total, w.varlen_min, w.varlen_max)
    elif w.decode_steps:
        lens = np.ones(w.batch, dtype=np.int64)
    else:
        lens = np.full(w.batch, w.seq_len, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


def make_weights(w: Workload, rng: np.random.Generator,
                 d_model: Optional[int] = None) -> Dict[str, np.ndarray]:
    """All parameters of one MoM layer, [out, in] layout, float32 arrays."""
    D = d_model or w.d_model
    Hd = w.heads * w.d_head
    std = 1.0 / np.sqrt(D)

    def lin(*shape):
        return _act(rng.standard_normal(shape, dtype=np.float32) * std, w.dtype)

    p = {}
    p["w_r"] = lin(w.n_mem, D)
    b_r = np.zeros(w.n_mem, dtype=np.float32)
    b_r[0] += w.router_bias0
    p["b_r"] = b_r
    p["w_q"] = lin(Hd, D)
    p["w_k_sh"] = lin(Hd, D)
    p["w_v_sh"] = lin(Hd, D)
    p["w_beta"] = lin(w.heads, D)
    p["w_a"] = lin(w.heads, D)
    p["A"] = rng.uniform(0.0, 2.7, size=w.heads).astype(np.float32)
    p["b_a"] = rng.uniform(-4.0, 0.0, size=w.heads).astype(np.float32)
    p["w_k"] = lin(w.n_mem, Hd, D)
    p["w_v"] = lin(w.n_mem, Hd, D)
    if w.mem_gates:
        # drawn from their own stream, so the other weights and the tokens are
        # those of the same workload without per-memory gates
        g = np.random.default_rng((w.seed, 1))
        p["w_beta_mem"] = _act(g.standard_normal((w.n_mem, w.heads, D), dtype=np.float32) * std, w.dtype)
        p["w_a_mem"] = _act(g.standard_normal((w.n_mem, w.heads, D), dtype=np.float32) * std, w.dtype)
        p["A_mem"] = g.uniform(0.0, 2.7, size=(w.n_mem, w.heads)).astype(np.float32)
        p["b_a_mem"] = g.uniform(-4.0, 0.0, size=(w.n_mem, w.heads)).astype(np.float32)
    if w.block:
        g = np.random.default_rng((w.seed, 2))
        W = w.conv_width
        conv = lambda *shape: g.uniform(-0.5, 0.5, size=shape + (W,)).astype(np.float32)
        p["w_g"] = _act(g.standard_normal((Hd, D), dtype=np.float32) * std, w.dtype)
        p["w_o"] = _act(g.standard_normal((D, Hd), dtype=np.float32) / np.sqrt(Hd), w.dtype)
        p["conv_q"] = conv(Hd)
        p["conv_k_sh"] = conv(Hd)
        p["conv_v_sh"] = conv(Hd)
        p["conv_k"] = conv(w.n_mem, Hd)
        p["conv_v"] = conv(w.n_mem, Hd)
        p["w_norm"] = g.uniform(0.5, 1.5, size=w.d_head).astype(np.float32)
    return p


def make_tokens(w: Workload, rng: np.random.Generator, n_tokens: int) -> np.ndarray:
    return _act(rng.standard_normal((n_tokens, w.d_model), dtype=np.float32), w.dtype)


def make_problem(w: Workload) -> Dict[str, np.ndarray]:
    """Weights, X and cu_seqlens for a forward workload (seeded by w.seed)."""
    rng = np.random.default_rng(w.seed)
    p = make_weights(w, rng)
    cu = make_cu_seqlens(w, rng)
    p["cu_seqlens"] = cu
    p["x"] = make_tokens(w, rng, int(cu[-1]))
    return p


def make_decode_problem(w: Workload, steps: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Weights, the prefill tokens [B*prefill_len, d_model] and per-step tokens
    [steps, B, d_model] for a decode workload."""
    rng = np.random.default_rng(w.seed)
    p = make_weights(w, rng)
    L = w.prefill_len
    p["cu_prefill"] = np.arange(0, (w.batch + 1) * L, L, dtype=np.int32)
    p["x_prefill"] = make_tokens(w, rng, w.batch * L)
    n = w.decode_steps if steps is None else steps
    p["x_steps"] = make_tokens(w, rng, n * w.batch).reshape(n, w.batch, w.d_model)
    return p


def small_workload(base: Workload, **over) -> Workload:
    """A copy of a workload with some fields replaced (test-sized variants)."""
    return dataclasses.replace(base, **over)
