"""Shared pieces of the GPU parity tests: running the CUDA layer on seeded
inputs and comparing with the oracle.

Error measure (the acceptance metric): max |gpu - ref| / max |ref| per
tensor.  Tolerances: 1e-4 with float32 inputs, 2e-2 with bf16 inputs and
float32 state.
"""
from __future__ import annotations

import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}


def max_abs_rel(gpu, ref) -> float:
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if gpu.size == 0:
        return 0.0
    return float(np.max(np.abs(gpu - ref)) / max(float(np.max(np.abs(ref))), 1e-30))


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def run_layer(w, p, scale=1.0, h0_shared=None, h0_mem=None, rule="gated_delta"):
    """Runs the CUDA layer on the problem p; returns (layer, numpy results)."""
    from mixture_memories_layer_b200 import layer as L
    dt = torch_dtype(w)
    weights = L.pack_weights(p, dt)
    lay = L.MoMLayer(weights, w.heads, w.d_head, w.top_k, scale, rule=rule)
    x = torch.as_tensor(p["x"]).to("cuda", dt)
    cu = torch.as_tensor(p["cu_seqlens"]).to("cuda", torch.int32)
    b = lay.forward(x, cu, h0_shared=h0_shared, h0_mem=h0_mem)
    torch.cuda.synchronize()
    res = {k: (to_np(v) if v.dtype not in (torch.int32,) else v.cpu().numpy())
           for k, v in b.items() if not k.startswith("ws")}
    return lay, res
