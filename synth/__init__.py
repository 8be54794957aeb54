"""Seeded synthetic inputs for the streaming int4 MoE block.

This module only *draws* inputs: int4 expert codes, bf16 scale/min, bf16 router,
prerouter-head, norm and LoRA weights, bf16 hidden states, and (for the
multi-stream decode workload) the target routing that the hidden states are
shaped to produce.  It computes no step of the MoE block.  Both the CPU oracle
(``oracle/``) and the GPU path read their inputs from here; neither imports the
other.

Every array is a deterministic function of ``(seed, tag, layer, index)``: each
expert blob, each layer's dense weights and each step's hidden states come from
their own ``SeedSequence``, so a test can regenerate one expert of a 40-layer
model without materialising the other 10,239.

Storage formats (the model description of the reading guide "The Other Half of
the Memory Wall", section "Temel fikirler" and the ai.info article "La versione
da 35B usa 256 esperti distribuiti su 40 livelli": int4 affine weights in groups
of 64):

* bf16 values are carried as ``uint16`` bit patterns (the top half of an IEEE
  binary32 word).
* One expert is one contiguous byte blob, sections in this order (all row-major,
  groups of 64 run along K, the input dimension)::

      gate.codes  [I, d/2]  u8   element 2i in the low nibble of byte i
      gate.scale  [I, d/64] bf16
      gate.min    [I, d/64] bf16
      up.codes / up.scale / up.min      (same shapes as gate)
      down.codes  [d, I/2]  u8
      down.scale  [d, I/64] bf16
      down.min    [d, I/64] bf16

  At d=2048, I=512 a blob is 1,769,472 bytes (4.5 bits per weight).
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# Stream tags: each kind of input draws from its own seed stream.
_T_EXPERT, _T_SHARED, _T_DENSE, _T_HIDDEN, _T_ROUTE, _T_HEADFULL = 11, 12, 13, 14, 15, 16


@dataclasses.dataclass(frozen=True)
class Dims:
    """Model geometry of one MoE stack."""
    d: int                  # hidden size
    E: int                  # routed experts per layer
    I: int                  # expert intermediate size
    k: int                  # routed experts per token
    r: int                  # LoRA rank on the shared expert
    L: int                  # layers
    head_layers: tuple      # layers that carry a prerouter head (head of N predicts N+1)
    group: int = 64
    head_hidden: int = 0    # 0: linear head d->E; >0: fc1(H)->gelu->fc2 plus the linear path
    head_onehot: int = 0    # 1: head input is [x; onehot(cur); onehot(prev)]
    eps: float = 1e-6
    lora_scale: float = 1.0

    @property
    def head_in(self) -> int:
        return self.d + (2 * self.E if self.head_onehot else 0)


def blob_sections(d: int, I: int):
    """(name, byte offset, byte size, shape, dtype) of each section of an expert blob."""
    out, off = [], 0
    for proj, rows, K in (("gate", I, d), ("up", I, d), ("down", d, I)):
        for part, shape, dt in (("codes", (rows, K // 2), np.uint8),
                                ("scale", (rows, K // 64), np.uint16),
                                ("min", (rows, K // 64), np.uint16)):
            n = int(np.prod(shape)) * np.dtype(dt).itemsize
            out.append((f"{proj}.{part}", off, n, shape, dt))
            off += n
    return out


def blob_bytes(d: int, I: int) -> int:
    s = blob_sections(d, I)[-1]
    return s[1] + s[2]


def _rng(*key) -> np.random.Generator:
    return np.random.Generator(np.random.SFC64(np.random.SeedSequence([int(v) for v in key])))


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even) and return the bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def _fill_blob(out: np.ndarray, rng: np.random.Generator, d: int, I: int,
               scale_lo=0.005, scale_hi=0.02, min_lo=-0.1, min_hi=0.1) -> None:
    for name, off, n, shape, dt in blob_sections(d, I):
        seg = out[off:off + n]
        if name.endswith("codes"):
            # uniform bytes = two independent uniform nibbles 0..15
            raw = rng.bit_generator.random_raw((n + 7) // 8)
            seg[:] = raw.view(np.uint8)[:n]
        else:
            lo, hi = (scale_lo, scale_hi) if name.endswith("scale") else (min_lo, max(min_hi, min_lo))
            v = lo + (hi - lo) * rng.random(n // 2, dtype=np.float32)
            seg.view(np.uint16)[:] = f32_to_bf16_bits(v)


def expert_blob(seed: int, layer: int, e: int, dims: Dims, out: np.ndarray | None = None) -> np.ndarray:
    """Routed expert ``e`` of ``layer``: codes uniform 0..15, scale ~U[0.005,0.02], min ~U[-0.1,0.1]."""
    nb = blob_bytes(dims.d, dims.I)
    if out is None:
        out = np.empty(nb, dtype=np.uint8)
    _fill_blob(out, _rng(seed, _T_EXPERT, layer, e), dims.d, dims.I)
    return out


def shared_blob(seed: int, layer: int, dims: Dims, out: np.ndarray | None = None) -> np.ndarray:
    """The always-on shared expert of ``layer`` (same distribution as the routed experts)."""
    nb = blob_bytes(dims.d, dims.I)
    if out is None:
        out = np.empty(nb, dtype=np.uint8)
    _fill_blob(out, _rng(seed, _T_SHARED, layer, 0), dims.d, dims.I)
    return out


def layer_experts(seed: int, layer: int, dims: Dims, out: np.ndarray | None = None,
                  threads: int = 8) -> np.ndarray:
    """All routed experts of one layer as ``[E, blob]`` uint8."""
    nb = blob_bytes(dims.d, dims.I)
    if out is None:
        out = np.empty((dims.E, nb), dtype=np.uint8)
    if threads <= 1 or dims.E < 8:
        for e in range(dims.E):
            expert_blob(seed, layer, e, dims, out[e])
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda e: expert_blob(seed, layer, e, dims, out[e]), range(dims.E)))
    return out


def _normal_bf16(rng, shape, std) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def layer_dense(seed: int, layer: int, dims: Dims, norm_random: bool = False) -> dict:
    """Router, head, RMSNorm and LoRA weights of one layer, as bf16 bit patterns.

    router_w [E,d] ~ N(0, 0.02^2); head_w [E, d(+2E)] ~ N(0, 0.02^2) when the layer has a
    head; LoRA A_g, A_u [r,d] ~ N(0, 1/d), A_d [r,I] ~ N(0, 1/I), B_g, B_u [I,r] and
    B_d [d,r] ~ N(0, 0.01^2); norm_w = ones (or ~U[0.5,1.5] with ``norm_random``).
    """
    d, E, I, r = dims.d, dims.E, dims.I, dims.r
    g = _rng(seed, _T_DENSE, layer, 0)
    out = {
        "router_w": _normal_bf16(g, (E, d), 0.02),
        "head_w": _normal_bf16(g, (E, dims.head_in), 0.02) if layer in dims.head_layers else None,
        "lora_Ag": _normal_bf16(g, (r, d), 1.0 / np.sqrt(d)),
        "lora_Bg": _normal_bf16(g, (I, r), 0.01),
        "lora_Au": _normal_bf16(g, (r, d), 1.0 / np.sqrt(d)),
        "lora_Bu": _normal_bf16(g, (I, r), 0.01),
        "lora_Ad": _normal_bf16(g, (r, I), 1.0 / np.sqrt(I)),
        "lora_Bd": _normal_bf16(g, (d, r), 0.01),
    }
    if norm_random:
        out["norm_w"] = f32_to_bf16_bits(0.5 + g.random(d, dtype=np.float32))
    else:
        out["norm_w"] = f32_to_bf16_bits(np.ones(d, dtype=np.float32))
    if dims.head_hidden and layer in dims.head_layers:
        h = _rng(seed, _T_HEADFULL, layer, 0)
        H = dims.head_hidden
        out["fc1_w"] = _normal_bf16(h, (H, dims.head_in), 0.02)
        out["fc1_b"] = _normal_bf16(h, (H,), 0.02)
        out["fc2_w"] = _normal_bf16(h, (E, H), 0.02)
        out["fc2_b"] = _normal_bf16(h, (E,), 0.02)
    return out


def hidden(seed: int, step: int, L: int, B: int, d: int) -> np.ndarray:
    """MoE inputs of one decode step, ``[L, B, d]`` bf16 bits, h ~ N(0, 1) per (layer, stream)."""
    return _normal_bf16(_rng(seed, _T_HIDDEN, step, 0), (L, B, d), 1.0)


def prefill_hidden(seed: int, layer: int, T: int, d: int) -> np.ndarray:
    """One prefill chunk's MoE input for ``layer``: ``[T, d]`` bf16 bits, N(0, 1)."""
    return _normal_bf16(_rng(seed, _T_HIDDEN, 1 << 20, layer), (T, d), 1.0)


def bf16_bits_from_f32(x) -> np.ndarray:
    """Public alias used by tests that hand-build weights."""
    return f32_to_bf16_bits(x)


# ---------------------------------------------------------------------------------------
# Named workloads.  Heads sit on layers 0..32 and predict layers 1..33; layers 0 and
# 34..39 route with their own router.
# ---------------------------------------------------------------------------------------
def _full(**kw) -> Dims:
    base = dict(d=2048, E=256, I=512, k=4, r=16, L=40, head_layers=tuple(range(33)))
    base.update(kw)
    return Dims(**base)


WORKLOADS = {
    "layer_d256_e16": dict(dims=Dims(d=256, E=16, I=128, k=4, r=8, L=1, head_layers=(0,)),
                           seed=0, batch=1, steps=1),
    "decode_b1_l40": dict(dims=_full(), seed=1, batch=1, steps=256),
    "decode_multistream_l40": dict(dims=_full(), seed=2, batch=(8, 32, 64), steps=128),
    "prefill_t4096_l40": dict(dims=_full(), seed=3, tokens=4096),
    "stream_b1_l40": dict(dims=_full(), seed=4, batch=1, steps=256),
    # the same geometry on a few layers: small cases for profiler captures
    "decode_b1_l4": dict(dims=_full(L=4, head_layers=(0, 1, 2)), seed=1, batch=1, steps=16),
    "prefill_t4096_l2": dict(dims=_full(L=2, head_layers=(0,)), seed=3, tokens=4096),
}


# ---------------------------------------------------------------------------------------
# Routing-shaped inputs for multi-stream decode: expert popularity is Zipf-like per layer
# and each stream keeps an expert into the next token with a fixed probability.
# ---------------------------------------------------------------------------------------
def zipf_popularity(E: int, s: float) -> np.ndarray:
    p = 1.0 / np.arange(1, E + 1, dtype=np.float64) ** s
    return p / p.sum()


def route_targets(seed: int, dims: Dims, B: int, steps: int, zipf_s: float = 1.0,
                  keep: float = 0.40) -> np.ndarray:
    """Target expert sets ``[steps, L, B, k]`` int32 with Zipf popularity and Markov reuse.

    Per layer a random permutation maps popularity rank to expert id.  Each stream draws
    its first set from the popularity law; at every later step each of its k experts is
    kept with probability ``keep`` and otherwise replaced by a fresh draw (not already in
    the set).  The realised reuse and popularity share are measured, not assumed.
    """
    g = _rng(seed, _T_ROUTE, 0, 0)
    E, k, L = dims.E, dims.k, dims.L
    pop = zipf_popularity(E, zipf_s)
    perms = np.stack([g.permutation(E) for _ in range(L)])
    out = np.empty((steps, L, B, k), dtype=np.int32)
    for layer in range(L):
        for b in range(B):
            cur: list[int] = []
            for t in range(steps):
                nxt = [e for e in cur if g.random() < keep]
                while len(nxt) < k:
                    e = int(perms[layer, g.choice(E, p=pop)])
                    if e not in nxt:
                        nxt.append(e)
                cur = nxt
                out[t, layer, b] = cur
    return out


def hidden_for_logits(W: np.ndarray, target: np.ndarray, d: int, rng: np.random.Generator) -> np.ndarray:
    """A vector ``h`` with ``W @ h = target`` (least norm) plus noise orthogonal to W's rows,
    scaled to unit RMS.  ``W`` is float64 ``[m, d]`` (m <= d)."""
    x, *_ = np.linalg.lstsq(W, target, rcond=None)
    noise = rng.standard_normal(d)
    q, _ = np.linalg.qr(W.T)
    noise -= q @ (q.T @ noise)
    need = d - float(x @ x)
    if need > 0:
        noise *= np.sqrt(need / float(noise @ noise))
        x = x + noise
    return x


def shaped_hidden(seed: int, wseed: int, dims: Dims, B: int, targets: np.ndarray, margin: float = 1.5) -> np.ndarray:
    """Decode inputs ``[steps, L, B, d]`` (bf16 bits) shaped so that the routing the stack
    takes is ``targets [steps, L, B, k]`` (e.g. from :func:`route_targets`).

    The routing of layer n at step t comes from layer n's router on its own input when n
    routes itself (step 0, layer 0, layers after a layer without a head), and from layer
    n-1's prerouter head on its input of step t-1 otherwise.  So the input of (t, n) is
    drawn to meet up to two sets of linear constraints: router rows giving logits whose
    top-k is targets[t, n] (when n routes itself at t), and head rows giving logits whose
    top-k is targets[t+1, n+1] (when n carries a head).  Target logits: the chosen experts
    at 3.0, 2.9, ... in rank order, the others ~ N(0, 0.4^2) clipped below 3.0 - margin.
    The least-norm solution plus noise orthogonal to the constraint rows, scaled to unit
    RMS, is rounded to bf16 (RMSNorm then leaves the top-k sets unchanged: it is a
    positive scale).  Uses the bf16 router/head weights of ``layer_dense(wseed, n)``; linear
    heads only.  The realised routing is measured by the caller, not assumed.
    """
    S, L, Bt, k = targets.shape
    assert Bt == B and L == dims.L and dims.head_hidden == 0 and not dims.head_onehot
    d, E = dims.d, dims.E
    g = _rng(seed, _T_ROUTE, 1, 0)
    out = np.empty((S, L, B, d), dtype=np.uint16)

    def target_logits(sets):                     # sets [N, k] -> [N, E]
        z = np.clip(g.standard_normal((sets.shape[0], E)) * 0.4, None, 3.0 - margin)
        for j in range(k):
            z[np.arange(sets.shape[0]), sets[:, j]] = 3.0 - 0.1 * j
        return z

    def bf(bits):
        return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    for n in range(L):
        dense = layer_dense(wseed, n, dims)
        Wr = bf(dense["router_w"])
        Wh = bf(dense["head_w"]) if dense.get("head_w") is not None else None
        own_always = n == 0 or (n - 1) not in dims.head_layers
        for step_set in ((0,), tuple(range(1, S))) if not own_always else (tuple(range(S)),):
            if not step_set:
                continue
            own = own_always or step_set == (0,)
            rows, zs = [], []
            ts = np.array(step_set)
            if own:
                rows.append(Wr)
                zs.append(target_logits(targets[ts, n].reshape(-1, k)).reshape(len(ts), B, E))
            if Wh is not None:
                nxt = np.minimum(ts + 1, S - 1)
                zh = target_logits(targets[nxt, min(n + 1, L - 1)].reshape(-1, k)).reshape(len(ts), B, E)
                rows.append(Wh)
                zs.append(zh)
            if not rows:
                x = g.standard_normal((len(ts) * B, d))
            else:
                W = np.concatenate(rows, 0)                          # [m, d]
                Z = np.concatenate(zs, 2).reshape(len(ts) * B, -1)   # [N, m]
                q, r = np.linalg.qr(W.T)                            # W.T = q r
                x = np.linalg.solve(r.T, Z.T).T @ q.T               # least-norm: W x = z
                noise = g.standard_normal(x.shape)
                noise -= (noise @ q) @ q.T
                need = d - np.sum(x * x, axis=1, keepdims=True)
                scale = np.sqrt(np.maximum(need, 0.0) / np.maximum(np.sum(noise * noise, axis=1, keepdims=True), 1e-30))
                x = x + noise * scale
            out[ts, n] = f32_to_bf16_bits(x.astype(np.float32)).reshape(len(ts), B, d)
    return out


def routing_stats(idx: np.ndarray) -> dict:
    """Realised next-token expert reuse and popularity concentration of a routing record
    ``[steps, L, B, k]``: reuse = mean over (step > 0, layer, stream) of the fraction of the
    k experts that the same stream used at the previous step; share95 = mean over layers
    of the fraction of experts that carry 95 % of that layer's assignments."""
    S, L, B, k = idx.shape
    reuse = []
    for t in range(1, S):
        for n in range(L):
            for b in range(B):
                reuse.append(len(set(idx[t, n, b].tolist()) & set(idx[t - 1, n, b].tolist())) / k)
    shares = []
    for n in range(L):
        c = np.sort(np.bincount(idx[:, n].reshape(-1), minlength=int(idx.max()) + 1))[::-1]
        cum = np.cumsum(c) / c.sum()
        E = max(int(idx.max()) + 1, 1)
        shares.append((int(np.searchsorted(cum, 0.95)) + 1) / E)
    return {"next_token_reuse": float(np.mean(reuse)) if reuse else None, "experts_for_95pct": float(np.mean(shares))}
