"""Host logic of the one-launch decode kernel: the per-CTA work-item lists.

The lists are built on the host (`e0_decode_items`, the function the context uses), so
their partition properties are checked here without a GPU: every unit of every phase of
every layer is covered exactly once across the CTAs, a reactive layer's top-k comes
before any item that needs its routing, the norm / down-input flags mark exactly the
first item of each layer, the flat schedule keeps its phase order, and no item exceeds
the ring's budget.  The GPU tests check that both schedules give bit-identical outputs.
"""
import itertools

import pytest

import int4_expert_streaming_prerouter_b200 as e0

R, TK, XR, GU, DN = range(5)
ITEM_BYTES = 58 * 1024

FULL = dict(d=2048, E=256, I=512, k=4, r=16, L=40, heads=tuple(range(33)))
SMALL = dict(d=256, E=16, I=128, k=4, r=8, L=6, heads=(0, 1, 2))


def lists(cfg, flat, step0, G, heads=None, lora=None):
    heads = cfg["heads"] if heads is None else heads
    L = cfg["L"]
    has_head = [l in heads for l in range(L)]
    has_lora = [cfg["r"] > 0] * L if lora is None else lora
    dims = e0.make_dims(cfg["d"], cfg["E"], cfg["I"], cfg["k"], cfg["r"])
    return [e0.decode_items(dims, L, has_head, has_lora, G, flat, step0, c) for c in range(G)], has_head, has_lora


def predicted(has_head, step0, l):
    return not step0 and l > 0 and has_head[l - 1]


def units(cfg, has_head, has_lora, step0, kind, l):
    E, k, r, I, d = cfg["E"], cfg["k"], cfg["r"], cfg["I"], cfg["d"]
    if kind == R:
        return 0 if predicted(has_head, step0, l) else E
    if kind == XR:
        return (E if has_head[l] else 0) + (2 * r if has_lora[l] else 0) + (k if predicted(has_head, step0, l) else 0)
    if kind == GU:
        return (k + 1) * I
    return d


TOP2 = dict(d=2048, E=64, I=512, k=2, r=0, L=7, heads=(0, 2, 3, 5))     # no LoRA, sparse heads
CASES = [(FULL, 148), (FULL, 37), (SMALL, 148), (SMALL, 5), (TOP2, 148), (TOP2, 11)]


@pytest.mark.parametrize("cfg,G", CASES)
@pytest.mark.parametrize("flat,step0", list(itertools.product([True, False], [False, True])))
def test_every_unit_covered_exactly_once(cfg, G, flat, step0):
    per_cta, has_head, has_lora = lists(cfg, flat, step0, G)
    cover = {}
    for items in per_cta:
        for kind, first, l, a, n in items:
            if kind == TK:
                assert n == 0
                continue
            assert n > 0
            cover.setdefault((kind, l), []).append((a, a + n))
    for l in range(cfg["L"]):
        for kind in (R, XR, GU, DN):
            want = units(cfg, has_head, has_lora, step0, kind, l)
            got = sorted(cover.get((kind, l), []))
            pos = 0
            for a, b in got:
                assert a == pos, f"kind {kind} layer {l}: gap or overlap at {pos} (next range {a}..{b})"
                pos = b
            assert pos == want, f"kind {kind} layer {l}: {pos} of {want} units"


@pytest.mark.parametrize("cfg,G", CASES)
@pytest.mark.parametrize("flat,step0", list(itertools.product([True, False], [False, True])))
def test_topk_precedes_every_item_that_needs_the_routing(cfg, G, flat, step0):
    per_cta, has_head, _ = lists(cfg, flat, step0, G)
    for items in per_cta:
        seen_tk = set()
        for kind, first, l, a, n in items:
            if kind == TK:
                assert not predicted(has_head, step0, l), "top-k item for a predicted layer"
                assert l not in seen_tk, "two top-k items for one layer"
                seen_tk.add(l)
            elif kind in (GU, DN) and not predicted(has_head, step0, l):
                assert l in seen_tk, f"layer {l}: gate/up or down before its top-k"


@pytest.mark.parametrize("cfg,G", CASES)
@pytest.mark.parametrize("flat,step0", list(itertools.product([True, False], [False, True])))
def test_first_flags_mark_each_layers_first_item(cfg, G, flat, step0):
    per_cta, _, _ = lists(cfg, flat, step0, G)
    for items in per_cta:
        last_x = last_d = None
        for kind, first, l, a, n in items:
            if kind in (R, XR, GU):
                assert first == (l != last_x)
                last_x = l
            elif kind == DN:
                assert first == (l != last_d)
                last_d = l
            else:
                assert first == 0


@pytest.mark.parametrize("cfg,G", CASES)
@pytest.mark.parametrize("step0", [False, True])
def test_flat_schedule_keeps_phase_order(cfg, G, step0):
    per_cta, _, _ = lists(cfg, True, step0, G)
    rank = {R: 0, XR: 1, TK: 2, GU: 3, DN: 4}
    for items in per_cta:
        ranks = [rank[kind] for kind, *_ in items]
        assert ranks == sorted(ranks)


@pytest.mark.parametrize("step0", [False, True])
def test_full_size_items_fit_the_ring_budget_and_the_cuts_are_balanced(step0):
    cfg = FULL
    d, I, k, r, E = cfg["d"], cfg["I"], cfg["k"], cfg["r"], cfg["E"]
    per_cta, _, _ = lists(cfg, True, step0, 148)
    gu_units = []
    for items in per_cta:
        gu = 0
        for kind, first, l, a, n in items:
            if kind == GU:
                assert n * 2 * (d // 2 + d // 16) <= ITEM_BYTES
                gu += n
            elif kind == DN:
                assert n * (k + 1) * (I // 2 + I // 16) + 2 * r * n <= ITEM_BYTES
            elif kind in (R, XR):
                assert n * 2 * d <= ITEM_BYTES
        gu_units.append(gu)
        assert len(items) <= 320
    mean = sum(gu_units) / len(gu_units)
    assert min(gu_units) > 0.6 * mean and max(gu_units) < 1.25 * mean


def test_headless_model_routes_every_layer_itself():
    per_cta, has_head, _ = lists(SMALL, True, False, 5, heads=())
    tk_layers = {l for items in per_cta for kind, _, l, _, _ in items if kind == TK}
    r_layers = {l for items in per_cta for kind, _, l, _, _ in items if kind == R}
    assert r_layers == set(range(SMALL["L"]))
    assert tk_layers == set(range(SMALL["L"]))


def test_rejects_bad_arguments():
    dims = e0.make_dims(256, 16, 128, 4, 8)
    with pytest.raises(e0.E0Error):
        e0.decode_items(dims, 2, [1, 1], [1, 1], 4, True, False, 4)     # cta out of range
    with pytest.raises(e0.E0Error):
        e0.decode_items(dims, 2, [1, 1], [1, 1], 0, True, False, 0)     # no CTAs
    with pytest.raises(e0.E0Error):
        e0.decode_items(dims, 0, [], [], 4, True, False, 0)             # no layers
