"""Upload seeded synthetic weights and inputs to torch tensors (device or pinned host).

Only moves the arrays drawn by :mod:`synth` into tensors; bf16 values stay as their bit
patterns (``torch.int16`` views reinterpreted as ``torch.bfloat16``).
"""
from __future__ import annotations

import numpy as np
import torch

from . import Dims, blob_bytes, layer_dense, layer_experts, shared_blob

_DENSE_KEYS = ("router_w", "norm_w", "lora_Ag", "lora_Bg", "lora_Au", "lora_Bu", "lora_Ad", "lora_Bd")
_HEAD_KEYS = ("fc1_w", "fc1_b", "fc2_w", "fc2_b")


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def layer_tensors(seed: int, layer: int, dims: Dims, device, resident: bool = True,
                  dense: dict | None = None, lora: bool = True, threads: int = 8) -> tuple:
    """(layer dict, head dict or None) of torch tensors for ``Context.register_model``."""
    dense = dense if dense is not None else layer_dense(seed, layer, dims)
    ly = {"shared": torch.from_numpy(shared_blob(seed, layer, dims)).to(device)}
    if resident:
        ly["experts"] = torch.from_numpy(layer_experts(seed, layer, dims, threads=threads)).to(device)
    for key in _DENSE_KEYS:
        if key.startswith("lora_") and not lora:
            continue
        ly[key] = bf16_tensor(dense[key], device)
    head = None
    if dense.get("head_w") is not None:
        head = {"w_lin": bf16_tensor(dense["head_w"], device)}
        for key in _HEAD_KEYS:
            if key in dense:
                head[key] = bf16_tensor(dense[key], device)
    return ly, head


def model_tensors(seed: int, dims: Dims, device, resident: bool = True, lora: bool = True,
                  threads: int = 8) -> tuple:
    layers, heads = [], []
    for n in range(dims.L):
        ly, hd = layer_tensors(seed, n, dims, device, resident=resident, lora=lora, threads=threads)
        layers.append(ly)
        heads.append(hd)
    return layers, heads


def pinned_expert_store(seed: int, dims: Dims, threads: int = 8) -> torch.Tensor:
    """All routed experts of every layer in one pinned host tensor ``[L, E, blob]``."""
    store = torch.empty((dims.L, dims.E, blob_bytes(dims.d, dims.I)), dtype=torch.uint8, pin_memory=True)
    arr = store.numpy()
    for n in range(dims.L):
        layer_experts(seed, n, dims, out=arr[n], threads=threads)
    return store


def hidden_tensor(seed: int, step: int, dims: Dims, B: int, device) -> torch.Tensor:
    from . import hidden
    return bf16_tensor(hidden(seed, step, dims.L, B, dims.d), device)
