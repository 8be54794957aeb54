"""Helpers of the GPU decode and streaming parity tests: run decode steps through the
library, run the oracle on the same seeded inputs, and compare the two."""
import numpy as np
import torch

import oracle as O
import synth
from synth.device import bf16_tensor, layer_tensors
from parity import bf16_bits_to_np, check_bf16, check_y, choose_following


def build(dims, seed, max_tokens, resident=True):
    import int4_expert_streaming_prerouter_b200 as e0
    ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, max_tokens,
                     head_hidden=dims.head_hidden, head_onehot=dims.head_onehot)
    lys, hds = zip(*[layer_tensors(seed, n, dims, "cuda", resident=resident) for n in range(dims.L)])
    ctx.register_model(list(lys), list(hds))
    return ctx, lys, hds


def run_steps(ctx, dims, seed, B, S, chained=False, streaming=False, after_step=None, t0=0):
    """Decode steps t0..t0+S-1 of B streams (inputs synth.hidden(seed, t)); returns bf16 y,
    fp32 y, routing and predictions stacked over the steps.  after_step(t) runs after each
    step has completed."""
    ys, y32s, idxs, preds = [], [], [], []
    for t in range(t0, t0 + S):
        h = bf16_tensor(synth.hidden(seed, t, dims.L, B, dims.d), "cuda")
        y32 = torch.empty((dims.L, B, dims.d), dtype=torch.float32, device="cuda")
        y = ctx.stack_decode(h, t, y_f32=y32, chained=chained, streaming=streaming)
        ctx.sync_status()
        idx, pred = ctx.get_routing(B)
        if after_step is not None:
            after_step(t)
        ys.append(bf16_bits_to_np(y))
        y32s.append(y32.cpu().numpy().astype(np.float64))
        idxs.append(idx)
        preds.append(pred)
    return np.stack(ys), np.stack(y32s), np.stack(idxs), np.stack(preds)


def oracle_steps(dims, seed, B, S, gpu_idx, gpu_pred, chained=False, weight_seed=None, prediction=True):
    """The oracle's decode of the same steps; at a near tie (fp32 gap < 1e-5) it follows
    the admissible set the GPU took, never otherwise."""
    ws = seed if weight_seed is None else weight_seed
    hs = np.stack([synth.hidden(seed, t, dims.L, B, dims.d) for t in range(S)])
    dense = {n: synth.layer_dense(ws, n, dims) for n in range(dims.L)}
    cache = {}

    def expert(n, e):
        if (n, e) not in cache:
            cache[(n, e)] = synth.expert_blob(ws, n, e, dims)
        return cache[(n, e)]

    sets = {}
    for t in range(S):
        for n in range(dims.L):
            for b in range(B):
                sets[("route", t, n, b)] = gpu_idx[t, n, b]
                sets[("head", t, n, b)] = gpu_pred[t, n, b]
    return O.stack_decode(hs, dense.__getitem__, expert, lambda n: synth.shared_blob(ws, n, dims), dims,
                          chained=chained, choose=choose_following(sets), prediction=prediction)


def compare_steps(dims, gpu, ref, prediction=True):
    yb, y32, idx, pred = gpu
    S, L, B = idx.shape[:3]
    assert np.array_equal(idx, ref["idx"]), "routing differs beyond admissible near ties"
    for n in range(L):
        if prediction and n in dims.head_layers:
            assert np.array_equal(pred[:, n], ref["pred"][:, n])
        else:
            assert np.all(pred[:, n] == -1)
    for t in range(S):
        for n in range(L):
            check_y(y32[t, n], ref["y"][t, n], f"step {t} layer {n}")
            check_bf16(yb[t, n], ref["y"][t, n], f"step {t} layer {n}", y32[t, n])
