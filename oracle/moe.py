"""Plain, slow, float64 CPU oracle of the streaming int4 MoE block.  TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline may use
this module.  It shares no code with the CUDA path.

Sources (page title and section; no code is printed on any of them):

[G]  "The Other Half of the Memory Wall: Serving 35B MoEs from SSD with Trained Routing
     Prediction", reading guide: "Temel fikirler" (key ideas: SSD weight tier,
     prediction-as-routing, unmerged recovery LoRA), "Yöntem / Ön Yönlendirici Başlık
     Mimarisi" (prerouter head: input width d+2E, head = fc2(erf-gelu(fc1 u)) + l(u),
     l warm-started from the next layer's router), "Yöntem / Birleştirilmemiş Adaptör
     Yürütme" (y = W_int4 x + (alpha/r) B A x), "Yöntem / Üç Aşamalı Eğitim" (LoRA on the
     shared-expert projections, not on streamed experts), "Temel terimler" (staged
     decode, slot table), "Sorular" (one token ahead, all layers in one batch).
[A]  "Edge0 serve un MoE da 35B a 20 token al secondo in 3 GiB", section "La versione
     da 35B usa 256 esperti distribuiti su 40 livelli": 40 layers, 256 routed experts
     plus one shared expert, top-4 routing, int4 affine quantisation in groups of 64,
     33 prerouter heads.

Readings where the pages are silent (each taken as the plainest reading the rest supports):
  * affine int4: w = scale * q + min, q = 0..15 unsigned; groups of 64 run along K;
    element 2i of a row sits in the low nibble of byte i.
  * activation: SwiGLU, a = silu(gate) * up.
  * gates: softmax of the layer's own router logits, renormalised over the k selected
    experts (in the selection's order); under prediction-as-routing the indices come
    from the prediction and the weights from the layer's own router.
  * head one-hot inputs: layer N's own routing at t and t-1.
  * rounding points: x, a and y are stored as bf16 (y also as fp32); router and head
    logits are fp32; everything else is float64 here.
  * top-k: descending logit, ties to the lower expert index.
  * shared expert: weight 1, LoRA on its gate, up and down projections.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "bf16_to_f64", "round_bf16", "round_f32", "f64_to_bf16_bits",
    "parse_expert_blob", "dequant_int4", "expert_matrices",
    "rmsnorm", "router_logits", "topk", "topk_alternatives", "gates_softmax",
    "silu", "gelu_erf", "routed_expert", "shared_expert", "moe_layer",
    "head_input", "prerouter_head", "predicted_layers", "stack_decode", "staging_plan",
    "sticky_plan",
]


# ---------------------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """Decode bf16 bit patterns (uint16): a bf16 is the upper 16 bits of a binary32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even (result in float64).

    A bfloat16 carries 8 significant bits, so for |x| in [2^(e-1), 2^e) its spacing is
    2^(e-8); below the smallest normal (2^-126) the spacing stays 2^-133.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    e = np.maximum(e, -125)
    ulp = np.ldexp(1.0, e - 8)
    return np.round(x / ulp) * ulp          # np.round: half to even


def f64_to_bf16_bits(x) -> np.ndarray:
    """Bit patterns of ``round_bf16(x)``."""
    v = round_bf16(x).astype(np.float32)    # exact: a bf16 value is a binary32 value
    return (v.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def round_f32(x) -> np.ndarray:
    """Round float64 to binary32 (nearest, ties to even), result in float64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------------------
# int4 affine group-64 weights ([G] "Temel fikirler"; [A] int4 affine, groups of 64)
# ---------------------------------------------------------------------------------------
def parse_expert_blob(blob: np.ndarray, d: int, I: int) -> dict:
    """Split one expert's byte blob into its nine sections.

    Section order: gate (codes [I,d/2], scale [I,d/64], min [I,d/64]), up (same),
    down (codes [d,I/2], scale [d,I/64], min [d,I/64]).  Codes are uint8, scale and min
    are bf16 bit patterns.
    """
    blob = np.asarray(blob, dtype=np.uint8).reshape(-1)
    out, off = {}, 0
    for proj, rows, K in (("gate", I, d), ("up", I, d), ("down", d, I)):
        n_codes = rows * (K // 2)
        n_groups = rows * (K // 64)
        codes = blob[off:off + n_codes].reshape(rows, K // 2)
        off += n_codes
        scale = blob[off:off + 2 * n_groups].view(np.uint16).reshape(rows, K // 64)
        off += 2 * n_groups
        minv = blob[off:off + 2 * n_groups].view(np.uint16).reshape(rows, K // 64)
        off += 2 * n_groups
        out[proj] = (codes, scale, minv, rows, K)
    assert off == blob.size, "blob size does not match (d, I)"
    return out


def dequant_int4(codes, scale_bits, min_bits, rows: int, K: int) -> np.ndarray:
    """w[n, k] = scale[n, k // 64] * q[n, k] + min[n, k // 64], q = nibble k of row n.

    Nibble k of a row is the low nibble of byte k // 2 when k is even and the high
    nibble when k is odd.
    """
    c = np.asarray(codes, dtype=np.uint8).reshape(rows, K // 2)
    q = np.empty((rows, K), dtype=np.float64)
    q[:, 0::2] = c & 0x0F
    q[:, 1::2] = c >> 4
    s = np.repeat(bf16_to_f64(scale_bits).reshape(rows, K // 64), 64, axis=1)
    m = np.repeat(bf16_to_f64(min_bits).reshape(rows, K // 64), 64, axis=1)
    return s * q + m


def expert_matrices(blob: np.ndarray, d: int, I: int) -> dict:
    """Dequantised gate [I,d], up [I,d] and down [d,I] matrices of one expert blob."""
    p = parse_expert_blob(blob, d, I)
    return {name: dequant_int4(*p[name]) for name in ("gate", "up", "down")}


# ---------------------------------------------------------------------------------------
# RMSNorm, router, top-k, gates
# ---------------------------------------------------------------------------------------
def rmsnorm(h, gamma_bits, eps: float) -> np.ndarray:
    """x = bf16( h * gamma / sqrt(mean(h^2) + eps) ), per row; h is [T, d] float64.

    The norm is the post-attention layer norm that the router, the prerouter head and
    the experts all read ([G] "Ön Yönlendirici Başlık Mimarisi").
    """
    h = np.atleast_2d(np.asarray(h, dtype=np.float64))
    g = bf16_to_f64(gamma_bits)
    rinv = 1.0 / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + eps)
    return round_bf16(h * g[None, :] * rinv)


def router_logits(W_bits, x) -> np.ndarray:
    """logits = W @ x per token, accumulated in float64 and rounded to fp32.  x: [T, d]."""
    W = bf16_to_f64(W_bits)
    return round_f32(np.atleast_2d(x) @ W.T)


def topk(logits_row, k: int) -> np.ndarray:
    """Indices of the k largest logits, descending, equal values ordered by lower index."""
    order = np.argsort(-np.asarray(logits_row, dtype=np.float64), kind="stable")
    return order[:k].astype(np.int32)


def topk_alternatives(logits_row, k: int, tol: float) -> list:
    """Every ordered index set a correct top-k could return when logits within ``tol``
    of each other may be ranked either way.

    Returns the canonical ``topk`` first.  A set is admissible when each chosen logit is
    no more than ``tol`` below every logit left out, and it is listed in the order of
    its logits (ties by index).  Used only where the canonical gap at rank k is < tol.
    """
    l = np.asarray(logits_row, dtype=np.float64)
    base = topk(l, k)
    kth = l[base[-1]]
    # experts whose logit is within tol of the boundary may swap in or out
    sure = [int(e) for e in base if l[e] > kth + tol]
    fuzzy = [int(e) for e in np.nonzero(np.abs(l - kth) <= tol)[0]]
    alts = [base]
    need = k - len(sure)
    for comb in itertools.combinations(sorted(fuzzy), need):
        s = sure + list(comb)
        chosen = set(s)
        left = [e for e in range(l.size) if e not in chosen]
        if left and min(l[s]) < max(l[left]) - tol:
            continue
        ordered = np.array(sorted(s, key=lambda e: (-l[e], e)), dtype=np.int32)
        if not any(np.array_equal(ordered, a) for a in alts):
            alts.append(ordered)
    return alts


def gates_softmax(logits_row, idx) -> np.ndarray:
    """Gate weights: softmax of the router logits of the selected experts, renormalised
    over the selection, in the selection's order."""
    z = np.asarray(logits_row, dtype=np.float64)[np.asarray(idx)]
    e = np.exp(z - z.max())
    return e / e.sum()


def silu(z):
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def gelu_erf(z):
    """The exact (erf) GELU of the head's hidden layer ([G] head equation)."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


# ---------------------------------------------------------------------------------------
# Experts ([G] "Birleştirilmemiş Adaptör Yürütme", "Üç Aşamalı Eğitim"; [A])
# ---------------------------------------------------------------------------------------
def routed_expert(W: dict, x) -> tuple:
    """One routed expert on one token: a = bf16(silu(Wg x) * (Wu x)), y = Wd a."""
    x = np.asarray(x, dtype=np.float64)
    g = W["gate"] @ x
    u = W["up"] @ x
    a = round_bf16(silu(g) * u)
    return W["down"] @ a, a


def shared_expert(W: dict, lora: dict, c: float, x) -> tuple:
    """The always-on shared expert with its unmerged LoRA delta on gate, up and down:

    g = Wg x + c Bg (Ag x),  u = Wu x + c Bu (Au x),  a = bf16(silu(g) * u),
    y = Wd a + c Bd (Ad a),  c = alpha / r.
    LoRA weights are bf16 bit patterns; a missing LoRA (None) contributes nothing.
    """
    x = np.asarray(x, dtype=np.float64)
    g = W["gate"] @ x
    u = W["up"] @ x
    if lora is not None:
        Ag, Bg = bf16_to_f64(lora["lora_Ag"]), bf16_to_f64(lora["lora_Bg"])
        Au, Bu = bf16_to_f64(lora["lora_Au"]), bf16_to_f64(lora["lora_Bu"])
        g = g + c * (Bg @ (Ag @ x))
        u = u + c * (Bu @ (Au @ x))
    a = round_bf16(silu(g) * u)
    y = W["down"] @ a
    if lora is not None:
        Ad, Bd = bf16_to_f64(lora["lora_Ad"]), bf16_to_f64(lora["lora_Bd"])
        y = y + c * (Bd @ (Ad @ a))
    return y, a


def moe_layer(h_bits, dense: dict, expert_blob, shared_blob, dims, route_idx=None,
              choose=None) -> dict:
    """One MoE block on T tokens.

    h_bits       [T, d] bf16 bit patterns (the layer's MoE input).
    dense        the layer's bf16 weights: norm_w, router_w, lora_* (synth.layer_dense).
    expert_blob  callable e -> blob of routed expert e;  shared_blob: the shared blob.
    route_idx    None (own router top-k) or [T, k] int32; a row of -1 means "own router".
    choose       optional callable (t, canonical, alternatives) -> set, used by tests to
                 follow one admissible top-k when the canonical gap is below 1e-5.

    Returns x, logits (fp32, [T,E]), idx [T,k], gates [T,k], a [T,k+1,I] and y (float64,
    before rounding) with y_f32 and y_bf16.
    """
    d, E, I, k = dims.d, dims.E, dims.I, dims.k
    h = bf16_to_f64(np.asarray(h_bits).reshape(-1, d))
    T = h.shape[0]
    x = rmsnorm(h, dense["norm_w"], dims.eps)
    logits = router_logits(dense["router_w"], x)
    idx = np.zeros((T, k), dtype=np.int32)
    for t in range(T):
        if route_idx is not None and route_idx[t][0] >= 0:
            idx[t] = route_idx[t]
        else:
            idx[t] = topk(logits[t], k)
            if choose is not None:
                idx[t] = choose(t, idx[t], topk_alternatives(logits[t], k, 1e-5))
    gates = np.stack([gates_softmax(logits[t], idx[t]) for t in range(T)])
    cache = {}

    def mats(e):
        if e not in cache:
            cache[e] = expert_matrices(expert_blob(int(e)), d, I)
        return cache[e]

    Ws = expert_matrices(shared_blob, d, I)
    y = np.zeros((T, d))
    a_all = np.zeros((T, k + 1, I))
    for t in range(T):
        for j in range(k):
            ye, a_all[t, j] = routed_expert(mats(idx[t, j]), x[t])
            y[t] += gates[t, j] * ye
        ys, a_all[t, k] = shared_expert(Ws, dense, dims.lora_scale, x[t])
        y[t] += ys
    return {"x": x, "logits": logits, "idx": idx, "gates": gates, "a": a_all, "y": y,
            "y_f32": round_f32(y), "y_bf16": round_bf16(y)}


# ---------------------------------------------------------------------------------------
# Prerouter head ([G] "Ön Yönlendirici Başlık Mimarisi"; "Temel fikirler")
# ---------------------------------------------------------------------------------------
def head_input(x, cur_idx, prev_idx, dims) -> np.ndarray:
    """u = [x; onehot_k(cur); onehot_k(prev)] (width d + 2E) when the head takes the
    routing history, else u = x.  A missing (None or -1) routing is an all-zero one-hot."""
    x = np.asarray(x, dtype=np.float64)
    if not dims.head_onehot:
        return x
    oh = np.zeros(2 * dims.E)
    for base, idx in ((0, cur_idx), (dims.E, prev_idx)):
        if idx is not None:
            for e in np.asarray(idx).reshape(-1):
                if e >= 0:
                    oh[base + int(e)] = 1.0
    return np.concatenate([x, oh])


def prerouter_head(x, dense: dict, dims, cur_idx=None, prev_idx=None) -> tuple:
    """head(u) = l(u) [+ fc2(gelu_erf(fc1 u + b1)) + b2]; returns fp32 logits and top-k.

    The head of layer N runs on layer N's normed input at token t; its top-k is the
    routing of layer N+1 at token t+1.
    """
    u = head_input(x, cur_idx, prev_idx, dims)
    z = bf16_to_f64(dense["head_w"]) @ u
    if dims.head_hidden:
        h1 = gelu_erf(bf16_to_f64(dense["fc1_w"]) @ u + bf16_to_f64(dense["fc1_b"]))
        z = z + bf16_to_f64(dense["fc2_w"]) @ h1 + bf16_to_f64(dense["fc2_b"])
    z = round_f32(z)
    return z, topk(z, dims.k)


# ---------------------------------------------------------------------------------------
# Decode over the stack with prediction-as-routing ([G] "Temel fikirler", "Sorular")
# ---------------------------------------------------------------------------------------
def predicted_layers(dims) -> set:
    """Layers whose routing is the previous layer's head prediction (made one token
    earlier): N is predicted when N-1 carries a head."""
    return {n + 1 for n in dims.head_layers if n + 1 < dims.L}


def stack_decode(h_steps, dense_of, expert_of, shared_of, dims, chained: bool = False,
                 choose=None, prediction: bool = True) -> dict:
    """Decode ``S`` steps of ``B`` streams through all ``L`` layers.

    h_steps    [S, L, B, d] bf16 bit patterns (generated MoE inputs).
    dense_of   layer -> dense weights;  expert_of(layer, e) -> blob;  shared_of(layer).
    chained    when true, layer N's input is bf16(h_N + y_{N-1}) instead of h_N.

    Routing of layer N at step t: the head prediction of layer N-1 made at step t-1 when
    N is a predicted layer and t > 0, else the layer's own router top-k.  The heads of
    every layer run at every step and their top-k become the next step's routing.
    prediction=False is the fully reactive comparison point of [G] "Sonuçlar" (no
    prerouter): every layer routes with its own router and no head runs (pred stays -1).
    Returns y [S,L,B,d] (float64), y_bf16, idx [S,L,B,k], gates, pred [S,L,B,k] (-1 where
    a layer has no head) and head logits.
    """
    h_steps = np.asarray(h_steps)
    S, L, B, d = h_steps.shape
    k, E = dims.k, dims.E
    pl = predicted_layers(dims)
    y = np.zeros((S, L, B, d))
    idx = np.zeros((S, L, B, k), dtype=np.int32)
    gates = np.zeros((S, L, B, k))
    pred = np.full((S, L, B, k), -1, dtype=np.int32)
    hlog = np.zeros((S, L, B, E))
    for t in range(S):
        for n in range(L):
            dense = dense_of(n)
            h = bf16_to_f64(h_steps[t, n])
            if chained and n > 0:
                h = round_bf16(h + y[t, n - 1])
            hb = f64_to_bf16_bits(h)
            route = pred[t - 1, n - 1] if (prediction and t > 0 and n in pl) else None
            pick = None if choose is None else (lambda b, c, a, t=t, n=n: choose(("route", t, n, b), c, a))
            out = moe_layer(hb, dense, lambda e, n=n: expert_of(n, e), shared_of(n), dims,
                            route_idx=route, choose=pick)
            y[t, n], idx[t, n], gates[t, n] = out["y"], out["idx"], out["gates"]
            if prediction and n in dims.head_layers:
                for b in range(B):
                    prev = idx[t - 1, n, b] if t > 0 else None
                    z, p = prerouter_head(out["x"][b], dense, dims, idx[t, n, b], prev)
                    if choose is not None:
                        p = choose(("head", t, n, b), p, topk_alternatives(z, k, 1e-5))
                    hlog[t, n, b], pred[t, n, b] = z, p
    return {"y": y, "y_f32": round_f32(y), "y_bf16": round_bf16(y), "idx": idx,
            "gates": gates, "pred": pred, "head_logits": hlog}


def staging_plan(idx, dims) -> dict:
    """Which experts the streaming tier must hold for each (step, layer).

    Prediction-as-routing makes the staged set of a predicted layer equal to the routed
    set ([G] "Temel fikirler"): the union over streams of the layer's routing, in first-
    seen order.  Reactive layers (no predictor, or step 0) are staged on demand after
    their router runs; their set is the same union.  Nothing is dropped by construction.
    """
    idx = np.asarray(idx)
    S, L = idx.shape[:2]
    plan = {}
    pl = predicted_layers(dims)
    for t in range(S):
        for n in range(L):
            seen = []
            for e in idx[t, n].reshape(-1):
                if int(e) not in seen:
                    seen.append(int(e))
            plan[(t, n)] = {"experts": seen, "prefetched": bool(t > 0 and n in pl)}
    return plan


def sticky_plan(idx, dims, slots: int) -> dict:
    """Copies made by per-layer persistent expert slot sets (one set of ``slots`` slots
    per layer, kept across decode steps).

    [G] "Temel terimler" describes the incremental sticky-slot stack (``incr_stack``):
    persistent stacked expert tensors in which only the expert slots that changed are
    rewritten, in place.  Reading taken for which slot a new expert overwrites when the
    set has more slots than one step needs (then the set acts as an expert cache in front
    of the host store): the slot least recently needed among those not needed at this
    step, an empty slot counting as never needed and equal ages going to the lower slot.

    For every (step t, layer n) the step's experts are the distinct entries of idx[t, n]
    in first-seen order (streams, then rank).  An expert already in the set is a hit; each
    missing expert, in that order, is copied into the next victim slot.  Returns
    {(t, n): {"copies": [(slot, expert), ...], "hits": h, "content": [expert or -1 per
    slot after the step]}}.
    """
    idx = np.asarray(idx)
    S, L = idx.shape[:2]
    content = {n: [-1] * slots for n in range(L)}
    last = {n: [-1] * slots for n in range(L)}      # staging round that last needed a slot
    plan = {}
    rnd = 0
    for t in range(S):
        for n in range(L):
            rnd += 1
            need = []
            for e in idx[t, n].reshape(-1):
                if int(e) not in need:
                    need.append(int(e))
            assert len(need) <= slots, "a step routes to more experts than the set has slots"
            held, misses, hits = set(), [], 0
            for e in need:
                if e in content[n]:
                    s = content[n].index(e)
                    held.add(s)
                    last[n][s] = rnd
                    hits += 1
                else:
                    misses.append(e)
            victims = sorted((s for s in range(slots) if s not in held), key=lambda s: (last[n][s], s))
            copies = []
            for e, s in zip(misses, victims):
                content[n][s] = e
                last[n][s] = rnd
                copies.append((s, e))
            plan[(t, n)] = {"copies": copies, "hits": hits, "content": list(content[n])}
    return plan
