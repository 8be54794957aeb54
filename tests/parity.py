"""Comparison rules shared by the GPU parity tests.

* Expert indices are bit-exact, except where the oracle's fp32 logit gap between rank k
  and rank k+1 is below 1e-5: there any admissible top-k (oracle.topk_alternatives) is
  accepted.
* MoE outputs (fp32): max |d| <= 2e-3 * rms(ref) and ||d||_2 / ||ref||_2 <= 1e-3.
* bf16 outputs: each must be the round-to-nearest-even bf16 of the GPU's own fp32 output
  (bit-exact), and lie within the fp32 tolerance plus one bf16 ulp of the oracle (bf16
  rounding alone moves a value by half an ulp, so fp32 is the tolerance check and this
  one catches layout or rounding-mode faults).
"""
import numpy as np

import oracle as O

TIE_GAP = 1e-5
MAX_ABS_REL_RMS = 2e-3
REL_L2 = 1e-3


def bf16_bits_to_np(t) -> np.ndarray:
    import torch
    return O.bf16_to_f64(t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def check_y(y_gpu, y_ref, what=""):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    d = y_gpu - y_ref
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    mx = float(np.max(np.abs(d))) if d.size else 0.0
    l2 = float(np.linalg.norm(d) / max(np.linalg.norm(y_ref), 1e-300))
    assert mx <= MAX_ABS_REL_RMS * rms, f"{what}: max|d| {mx:.3e} > {MAX_ABS_REL_RMS}*rms {rms:.3e}"
    assert l2 <= REL_L2, f"{what}: rel L2 {l2:.3e} > {REL_L2}"
    return mx / max(rms, 1e-300), l2


def check_bf16(y_gpu_bf16, y_ref, what="", y_gpu_f32=None):
    y_ref = np.asarray(y_ref, dtype=np.float64)
    if y_gpu_f32 is not None:
        exact = O.round_bf16(np.asarray(y_gpu_f32, dtype=np.float64))
        assert np.array_equal(y_gpu_bf16, exact), f"{what}: bf16 output is not the RNE rounding of the fp32 output"
    ref = O.round_bf16(y_ref)
    _, e = np.frexp(np.where(ref == 0, 1e-30, ref))
    ulp = np.ldexp(1.0, np.maximum(e, -125) - 8)
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    bad = np.abs(y_gpu_bf16 - y_ref) > MAX_ABS_REL_RMS * rms + ulp
    assert not bad.any(), f"{what}: {bad.sum()} bf16 outputs outside tolerance + 1 ulp"


def idx_ok(gpu_idx, ref_logits, ref_idx, k) -> bool:
    """GPU routing equals the oracle's, or is an admissible top-k at a near tie."""
    if np.array_equal(gpu_idx, ref_idx):
        return True
    alts = O.topk_alternatives(ref_logits, k, TIE_GAP)
    return any(np.array_equal(gpu_idx, a) for a in alts)


def choose_following(gpu_sets: dict):
    """A `choose` callback for the oracle: at a near tie follow the admissible set the GPU
    took (it must be one the oracle itself enumerates), else keep the canonical one."""
    def choose(key, canonical, alts):
        g = gpu_sets.get(key)
        if g is None or np.array_equal(g, canonical):
            return canonical
        for a in alts:
            if np.array_equal(a, g):
                return a
        return canonical
    return choose
