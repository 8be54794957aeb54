"""Pins of the CPU oracle against things other than itself (runs on CPU, no GPU).

Each test ties one oracle function to a closed form, a library routine, an invariant
stated by the pages, or the hand-derived worked example below, so that a dropped term,
a wrong sign, a swapped nibble or a transposed operand fails somewhere here.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle as O
import synth
from synth import Dims, blob_sections, f32_to_bf16_bits


# ---------------------------------------------------------------------------------------
# helpers that build blobs by hand (test side only)
# ---------------------------------------------------------------------------------------
def pack_codes(q: np.ndarray) -> np.ndarray:
    """Encode a [rows, K] array of nibbles: element 2i -> low nibble of byte i."""
    q = np.asarray(q, dtype=np.uint8)
    lo, hi = q[:, 0::2], q[:, 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def make_blob(d, I, proj: dict) -> np.ndarray:
    """proj[name] = (q [rows,K], scale [rows,K/64], min [rows,K/64]) as python floats."""
    nb = synth.blob_bytes(d, I)
    blob = np.zeros(nb, dtype=np.uint8)
    for name, off, n, shape, dt in blob_sections(d, I):
        p, part = name.split(".")
        q, s, m = proj[p]
        if part == "codes":
            blob[off:off + n] = pack_codes(q).reshape(-1)
        else:
            v = np.asarray(s if part == "scale" else m, dtype=np.float32).reshape(-1)
            blob[off:off + n].view(np.uint16)[:] = f32_to_bf16_bits(v)
    return blob


def torch_bf16_bits_to_f64(bits):
    t = torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16).copy())
    return t.view(torch.bfloat16).to(torch.float64).numpy()


# ---------------------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------------------
def test_bf16_decode_every_pattern_matches_torch():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_to_f64(bits)
    ref = torch_bf16_bits_to_f64(bits)
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_round_bf16_matches_torch_rne_including_ties():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    # exact ties: low half 0x8000 with even and odd upper halves
    u = rng.integers(0x3000, 0x4F00, 4000, dtype=np.uint32) << 16 | 0x8000
    x = np.concatenate([x, u.astype(np.uint32).view(np.float32), np.float32([0.0, -0.0, 1e-40, -3e-39])])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    ours = O.round_bf16(x.astype(np.float64))
    assert np.array_equal(ours, ref)
    # the bit view agrees with the value view
    assert np.array_equal(O.bf16_to_f64(O.f64_to_bf16_bits(x.astype(np.float64))), ref)


def test_round_bf16_spacing_closed_form():
    # values in [16, 32) sit on a grid of 1/8; in [4, 8) on a grid of 1/32
    assert O.round_bf16(31.42444)[()] == 31.375
    assert O.round_bf16(-4.303063)[()] == -4.3125
    assert O.round_bf16(20.617343)[()] == 20.625
    assert O.round_bf16(1.0 / math.sqrt(1.0 + 1e-6))[()] == 1.0
    # half-way between 1 and 1+2^-7 rounds to the even neighbour 1.0
    assert O.round_bf16(1.0 + 2.0 ** -8)[()] == 1.0
    assert O.round_bf16(1.0 + 3 * 2.0 ** -8)[()] == 1.0 + 2.0 ** -6


# ---------------------------------------------------------------------------------------
# int4 affine dequant: every nibble, nibble order, group index
# ---------------------------------------------------------------------------------------
def test_dequant_every_byte_and_group():
    rows, K = 8, 128                      # 2 groups of 64 per row, 64 bytes per row
    codes = np.arange(rows * K // 2, dtype=np.uint32).astype(np.uint8).reshape(rows, K // 2)
    assert set(codes.reshape(-1).tolist()) == set(range(256))
    # distinct scale and min per (row, group), as bf16 bit patterns
    s_vals = np.array([[0.5 + r + 0.25 * g for g in range(2)] for r in range(rows)], np.float32)
    m_vals = np.array([[-(r + 1) * 0.125 + g for g in range(2)] for r in range(rows)], np.float32)
    s_bits, m_bits = f32_to_bf16_bits(s_vals), f32_to_bf16_bits(m_vals)
    w = O.dequant_int4(codes, s_bits, m_bits, rows, K)
    s_ref, m_ref = torch_bf16_bits_to_f64(s_bits), torch_bf16_bits_to_f64(m_bits)
    for r in range(rows):
        for k in range(K):
            b = int(codes[r, k // 2])
            q = b % 16 if k % 2 == 0 else b // 16
            g = k // 64
            assert w[r, k] == s_ref[r, g] * q + m_ref[r, g], (r, k)


def test_byte_0x21_decodes_to_1_then_2():
    codes = np.full((1, 32), 0x21, dtype=np.uint8)
    one, zero = f32_to_bf16_bits(np.float32([[1.0]])), f32_to_bf16_bits(np.float32([[0.0]]))
    w = O.dequant_int4(codes, one, zero, 1, 64)
    assert w[0, 0] == 1.0 and w[0, 1] == 2.0 and w[0, 62] == 1.0 and w[0, 63] == 2.0


def test_blob_sizes_closed_form():
    # codes: 3 * I*d/2 ; scale+min: 3 * I*d/64 * 2 * 2
    assert synth.blob_bytes(2048, 512) == 3 * 512 * 2048 // 2 + 3 * 512 * 2048 // 64 * 4 == 1769472
    assert synth.blob_bytes(256, 128) == 55296
    d, I = 256, 128
    blob = synth.expert_blob(0, 0, 3, Dims(d=d, E=16, I=I, k=4, r=8, L=1, head_layers=(0,)))
    p = O.parse_expert_blob(blob, d, I)
    assert p["gate"][0].shape == (I, d // 2) and p["down"][0].shape == (d, I // 2)
    s = O.bf16_to_f64(p["up"][1])
    m = O.bf16_to_f64(p["down"][2])
    assert s.min() >= 0.005 - 1e-4 and s.max() <= 0.02 + 1e-4
    assert m.min() >= -0.1 - 1e-3 and m.max() <= 0.1 + 1e-3


# ---------------------------------------------------------------------------------------
# RMSNorm
# ---------------------------------------------------------------------------------------
def test_rmsnorm_ones_gives_exact_one():
    g = f32_to_bf16_bits(np.ones(2048, np.float32))
    x = O.rmsnorm(np.ones((1, 2048)), g, 1e-6)
    assert np.all(x == 1.0)
    x = O.rmsnorm(np.full((1, 64), 3.0), f32_to_bf16_bits(np.ones(64, np.float32)), 1e-6)
    assert np.all(x == 1.0)


def test_rmsnorm_eps_closed_form():
    # mean(h^2) = 1e-6 = eps, so x = 1e-3 / sqrt(2e-6) = 1/sqrt(2), rounded to bf16
    g = f32_to_bf16_bits(np.ones(128, np.float32))
    x = O.rmsnorm(np.full((1, 128), 1e-3), g, 1e-6)
    assert np.all(x == O.round_bf16(1.0 / math.sqrt(2.0)))
    x = O.rmsnorm(np.zeros((1, 128)), g, 1e-6)
    assert np.all(x == 0.0)


def test_rmsnorm_matches_torch_rms_norm():
    rng = np.random.default_rng(1)
    h = O.round_bf16(rng.standard_normal((6, 512)) * 3)
    gamma = f32_to_bf16_bits((0.5 + rng.random(512)).astype(np.float32))
    ref = F.rms_norm(torch.from_numpy(h), (512,), weight=torch.from_numpy(O.bf16_to_f64(gamma)),
                     eps=1e-6).numpy()
    assert np.array_equal(O.rmsnorm(h, gamma, 1e-6), O.round_bf16(ref))


# ---------------------------------------------------------------------------------------
# top-k, gates, activations
# ---------------------------------------------------------------------------------------
def test_topk_tie_rule_examples():
    assert O.topk(np.zeros(16), 4).tolist() == [0, 1, 2, 3]
    assert O.topk(np.array([1.0, 3.0, 3.0, 2.0, 3.0]), 2).tolist() == [1, 2]
    assert O.topk(np.array([5.0, -1.0, 7.0, 7.0]), 3).tolist() == [2, 3, 0]


def test_topk_matches_torch_on_distinct_values():
    rng = np.random.default_rng(2)
    for _ in range(50):
        l = rng.standard_normal(256)
        v, i = torch.topk(torch.from_numpy(l), 4)
        assert O.topk(l, 4).tolist() == i.tolist()


def test_topk_alternatives_enumerates_near_ties():
    l = np.array([3.0, 1.0, 2.0, 2.0 + 5e-6, 0.5])
    alts = O.topk_alternatives(l, 3, 1e-5)
    sets = [a.tolist() for a in alts]
    assert sets[0] == [0, 3, 2]
    assert [0, 3, 2] in sets and len(sets) == 1   # 2 and 3 both in: only order differs
    alts = O.topk_alternatives(l, 2, 1e-5)
    assert [a.tolist() for a in alts] == [[0, 3], [0, 2]]
    assert len(O.topk_alternatives(np.array([3.0, 1.0, 2.0]), 2, 1e-5)) == 1


def test_gates_with_all_experts_equal_full_softmax():
    rng = np.random.default_rng(3)
    l = O.round_f32(rng.standard_normal(16))
    idx = O.topk(l, 16)
    g = O.gates_softmax(l, idx)
    assert np.allclose(g, scipy.special.softmax(l)[idx], rtol=1e-14, atol=0)
    assert abs(g.sum() - 1.0) < 1e-15


def test_silu_and_gelu_closed_forms():
    z = np.linspace(-12, 12, 97)
    assert np.allclose(O.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)
    assert abs(O.gelu_erf(1.0) - 0.8413447460685429) < 1e-15
    assert abs(O.gelu_erf(-1.0) + 0.15865525393145707) < 1e-15
    assert np.allclose(O.gelu_erf(z), F.gelu(torch.from_numpy(z), approximate="none").numpy(),
                       rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------------------------------
# hand-derived worked example: d=128 (2 groups), I=64, E=2, k=2, h = ones, gamma = 1
# ---------------------------------------------------------------------------------------
def worked_example(lora: bool, k: int = 2):
    d, I, E = 128, 64, 2
    dims = Dims(d=d, E=E, I=I, k=k, r=1, L=1, head_layers=())
    ones = lambda rows, K, v: np.full((rows, K), v)
    sm = lambda rows, K, v: np.full((rows, K // 64), v)
    # expert 0: gate q=1 (group 0) and q=3 (group 1), s=2^-6 -> g=4; up q=8, s=2^-6,
    # m=-2^-4 -> u=8; down q=1, s=2^-6 -> y0 = bf16(silu(4)*8) = 31.375 in every row
    q_gate0 = np.concatenate([ones(I, 64, 1), ones(I, 64, 3)], axis=1)
    e0 = make_blob(d, I, {"gate": (q_gate0, sm(I, d, 2 ** -6), sm(I, d, 0.0)),
                          "up": (ones(I, d, 8), sm(I, d, 2 ** -6), sm(I, d, -2 ** -4)),
                          "down": (ones(d, I, 1), sm(d, I, 2 ** -6), sm(d, I, 0.0))})
    # expert 1: gate group 0 q=0, m=-1/8 -> -8 ; group 1 q=7, s=2^-6 -> +7 ; g=-1
    #           up q=4, s=2^-5 -> u=16 ; a = bf16(silu(-1)*16) = -4.3125 ; down q=2 -> -8.625
    q_gate1 = np.concatenate([ones(I, 64, 0), ones(I, 64, 7)], axis=1)
    s_gate1 = np.tile([2 ** -6, 2 ** -6], (I, 1))
    m_gate1 = np.tile([-0.125, 0.0], (I, 1))
    e1 = make_blob(d, I, {"gate": (q_gate1, s_gate1, m_gate1),
                          "up": (ones(I, d, 4), sm(I, d, 2 ** -5), sm(I, d, 0.0)),
                          "down": (ones(d, I, 2), sm(d, I, 2 ** -6), sm(d, I, 0.0))})
    zero = {"gate": (ones(I, d, 0), sm(I, d, 0.0), sm(I, d, 0.0)),
            "up": (ones(I, d, 0), sm(I, d, 0.0), sm(I, d, 0.0)),
            "down": (ones(d, I, 0), sm(d, I, 0.0), sm(d, I, 0.0))}
    shared = make_blob(d, I, zero)
    bf = lambda a: f32_to_bf16_bits(np.asarray(a, np.float32))
    router = np.zeros((E, d), np.float32)
    router[0, :] = 2 ** -7                       # l = [1, 0]
    dense = {"norm_w": bf(np.ones(d)), "router_w": bf(router)}
    if lora:
        # A x = 1 for gate and up; B_g = 2, B_u = 3 -> g_s = 2, u_s = 3;
        # a_s = bf16(silu(2)*3) = 5.28125 ; A_d a_s = 5.28125 ; B_d = 1
        dense.update(lora_Ag=bf(np.full((1, d), 2 ** -7)), lora_Bg=bf(np.full((I, 1), 2.0)),
                     lora_Au=bf(np.full((1, d), 2 ** -7)), lora_Bu=bf(np.full((I, 1), 3.0)),
                     lora_Ad=bf(np.full((1, I), 2 ** -6)), lora_Bd=bf(np.full((d, 1), 1.0)))
    else:
        dense.update(lora_Ag=bf(np.zeros((1, d))), lora_Bg=bf(np.zeros((I, 1))),
                     lora_Au=bf(np.zeros((1, d))), lora_Bu=bf(np.zeros((I, 1))),
                     lora_Ad=bf(np.zeros((1, I))), lora_Bd=bf(np.zeros((d, 1))))
    h = bf(np.ones((1, d)))
    return O.moe_layer(h, dense, lambda e: (e0, e1)[e], shared, dims)


def test_worked_example_two_experts():
    out = worked_example(lora=False)
    assert np.all(out["x"] == 1.0)
    assert out["logits"][0].tolist() == [1.0, 0.0]
    assert out["idx"][0].tolist() == [0, 1]
    w0 = math.e / (1 + math.e)
    assert abs(out["gates"][0, 0] - w0) < 1e-15
    assert np.all(out["a"][0, 0] == 31.375) and np.all(out["a"][0, 1] == -4.3125)
    expect = w0 * 31.375 + (1 - w0) * -8.625          # = 20.617343...
    assert abs(expect - 20.617343) < 1e-6
    assert np.allclose(out["y"][0], expect, rtol=0, atol=1e-12)
    assert np.all(out["y_bf16"][0] == 20.625)


def test_worked_example_top1_and_lora():
    out = worked_example(lora=False, k=1)
    assert np.all(out["y"][0] == 31.375)
    out = worked_example(lora=True)
    assert np.all(out["a"][0, 2] == 5.28125)
    w0 = math.e / (1 + math.e)
    expect = w0 * 31.375 + (1 - w0) * -8.625 + 5.28125   # = 25.898593...
    assert abs(expect - 25.898593) < 1e-6
    assert np.allclose(out["y"][0], expect, rtol=0, atol=1e-12)
    assert np.all(out["y_bf16"][0] == 25.875)


# ---------------------------------------------------------------------------------------
# invariants on random weights
# ---------------------------------------------------------------------------------------
SMALL = Dims(d=256, E=16, I=128, k=4, r=8, L=3, head_layers=(0, 1))


def _torch_expert(W, x):
    """The same FFN written with torch float64 library ops (round_bf16 is pinned above)."""
    tx = torch.from_numpy(np.asarray(x, np.float64))
    g = F.linear(tx, torch.from_numpy(W["gate"]))
    u = F.linear(tx, torch.from_numpy(W["up"]))
    a = torch.from_numpy(O.round_bf16((F.silu(g) * u).numpy()))
    return F.linear(a, torch.from_numpy(W["down"])).numpy()


def test_routed_expert_matches_torch_ffn():
    blob = synth.expert_blob(7, 0, 0, SMALL)
    W = O.expert_matrices(blob, SMALL.d, SMALL.I)
    x = O.round_bf16(np.random.default_rng(0).standard_normal(SMALL.d))
    y, _ = O.routed_expert(W, x)
    assert np.allclose(y, _torch_expert(W, x), rtol=1e-12, atol=1e-12)


def test_dense_mixture_all_experts_uniform_gates():
    """k = E with a zero router: y = (1/E) sum_e y_e + y_s (pins gates and combine)."""
    dims = Dims(d=256, E=16, I=128, k=16, r=8, L=1, head_layers=())
    dense = synth.layer_dense(9, 0, dims)
    dense["router_w"] = np.zeros_like(dense["router_w"])
    for key in ("lora_Bg", "lora_Bu", "lora_Bd"):
        dense[key] = np.zeros_like(dense[key])
    h = synth.hidden(9, 0, 1, 2, dims.d)[0]
    blobs = [synth.expert_blob(9, 0, e, dims) for e in range(dims.E)]
    sh = synth.shared_blob(9, 0, dims)
    out = O.moe_layer(h, dense, lambda e: blobs[e], sh, dims)
    assert np.allclose(out["gates"], 1.0 / 16, rtol=0, atol=1e-15)
    for t in range(2):
        x = out["x"][t]
        ref = sum(_torch_expert(O.expert_matrices(b, dims.d, dims.I), x) for b in blobs) / 16
        ref = ref + _torch_expert(O.expert_matrices(sh, dims.d, dims.I), x)
        assert np.allclose(out["y"][t], ref, rtol=1e-10, atol=1e-10)


def test_lora_b_zero_is_base_path_bit_for_bit():
    dense = synth.layer_dense(4, 0, SMALL)
    for key in ("lora_Bg", "lora_Bu", "lora_Bd"):
        dense[key] = np.zeros_like(dense[key])
    W = O.expert_matrices(synth.shared_blob(4, 0, SMALL), SMALL.d, SMALL.I)
    x = O.round_bf16(np.random.default_rng(4).standard_normal(SMALL.d))
    y1, a1 = O.shared_expert(W, dense, 1.0, x)
    y0, a0 = O.shared_expert(W, None, 1.0, x)
    assert np.array_equal(y1, y0) and np.array_equal(a1, a0)


def test_lora_unmerged_equals_merged_weights():
    """(W + c B A) x = W x + c B (A x) with large B, so a dropped branch cannot hide."""
    rng = np.random.default_rng(6)
    dense = synth.layer_dense(6, 0, SMALL)
    for key, shape in (("lora_Bg", (SMALL.I, SMALL.r)), ("lora_Bu", (SMALL.I, SMALL.r)),
                       ("lora_Bd", (SMALL.d, SMALL.r))):
        dense[key] = f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))
    c = 0.5
    W = O.expert_matrices(synth.shared_blob(6, 0, SMALL), SMALL.d, SMALL.I)
    x = O.round_bf16(rng.standard_normal(SMALL.d))
    y, a = O.shared_expert(W, dense, c, x)
    f = lambda k: torch.from_numpy(torch_bf16_bits_to_f64(dense[k]))
    Wg = torch.from_numpy(W["gate"]) + c * f("lora_Bg") @ f("lora_Ag")
    Wu = torch.from_numpy(W["up"]) + c * f("lora_Bu") @ f("lora_Au")
    Wd = torch.from_numpy(W["down"]) + c * f("lora_Bd") @ f("lora_Ad")
    tx = torch.from_numpy(x)
    a_ref = O.round_bf16((F.silu(Wg @ tx) * (Wu @ tx)).numpy())
    assert np.array_equal(a, a_ref)
    assert np.allclose(y, (Wd @ torch.from_numpy(a_ref)).numpy(), rtol=1e-11, atol=1e-11)
    # and the branch matters: dropping it moves y by much more than the tolerance
    y0, _ = O.shared_expert(W, None, c, x)
    assert np.linalg.norm(y - y0) > 0.1 * np.linalg.norm(y0)


# ---------------------------------------------------------------------------------------
# prerouter head
# ---------------------------------------------------------------------------------------
def test_head_warm_started_from_next_router_reproduces_its_routing():
    """l warm-started from layer N+1's router: on layer N+1's input the head's top-k is
    that router's top-k (the warm-start relation of the head architecture)."""
    d0 = synth.layer_dense(8, 0, SMALL)
    d1 = synth.layer_dense(8, 1, SMALL)
    d0["head_w"] = d1["router_w"].copy()
    h = synth.hidden(8, 0, 2, 3, SMALL.d)[1]
    out1 = O.moe_layer(h, d1, lambda e: synth.expert_blob(8, 1, e, SMALL),
                       synth.shared_blob(8, 1, SMALL), SMALL)
    for t in range(3):
        z, p = O.prerouter_head(out1["x"][t], d0, SMALL)
        assert np.array_equal(z, out1["logits"][t]) and np.array_equal(p, out1["idx"][t])


def test_full_head_matches_torch_mlp_and_onehot_columns():
    dims = Dims(d=64, E=16, I=64, k=4, r=2, L=2, head_layers=(0,), head_hidden=64, head_onehot=1)
    dense = synth.layer_dense(10, 0, dims)
    assert dense["head_w"].shape == (16, 64 + 32)
    x = O.round_bf16(np.random.default_rng(10).standard_normal(64))
    cur, prev = np.array([3, 1, 7, 0]), np.array([2, 3, 9, 15])
    z, p = O.prerouter_head(x, dense, dims, cur, prev)
    u = np.concatenate([x, np.isin(np.arange(16), cur).astype(float),
                        np.isin(np.arange(16), prev).astype(float)])
    t = lambda k: torch.from_numpy(torch_bf16_bits_to_f64(dense[k]))
    tu = torch.from_numpy(u)
    ref = F.linear(tu, t("head_w")) + F.linear(
        F.gelu(F.linear(tu, t("fc1_w"), t("fc1_b")), approximate="none"), t("fc2_w"), t("fc2_b"))
    assert np.array_equal(z, ref.numpy().astype(np.float32).astype(np.float64))
    # one-hot columns: with x = 0 and no MLP the linear path sums the selected columns
    lin = Dims(d=64, E=16, I=64, k=4, r=2, L=2, head_layers=(0,), head_onehot=1)
    z0, _ = O.prerouter_head(np.zeros(64), dense, lin, cur, None)
    W = torch_bf16_bits_to_f64(dense["head_w"])
    assert np.allclose(z0, W[:, 64 + cur].sum(axis=1), rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------------------------------
# prediction-as-routing over the stack, and the staging plan
# ---------------------------------------------------------------------------------------
def test_stack_decode_consumes_predictions_as_routing():
    S, B = 3, 2
    hs = np.stack([synth.hidden(11, t, SMALL.L, B, SMALL.d) for t in range(S)])
    dense = {n: synth.layer_dense(11, n, SMALL) for n in range(SMALL.L)}
    out = O.stack_decode(hs, dense.__getitem__, lambda n, e: synth.expert_blob(11, n, e, SMALL),
                         lambda n: synth.shared_blob(11, n, SMALL), SMALL)
    assert O.predicted_layers(SMALL) == {1, 2}
    for t in range(S):
        for n in range(SMALL.L):
            # own-router layers: the routed set is the top-k of the layer's own logits
            x = O.rmsnorm(O.bf16_to_f64(hs[t, n]), dense[n]["norm_w"], SMALL.eps)
            own = O.router_logits(dense[n]["router_w"], x)
            for b in range(B):
                if t == 0 or n == 0:
                    assert out["idx"][t, n, b].tolist() == O.topk(own[b], SMALL.k).tolist()
                else:
                    # predicted layer: routing is the head prediction made one token earlier
                    assert out["idx"][t, n, b].tolist() == out["pred"][t - 1, n - 1, b].tolist()
    assert np.all(out["pred"][:, 2] == -1)          # layer 2 has no head
    plan = O.staging_plan(out["idx"], SMALL)
    for (t, n), st in plan.items():
        routed = set(out["idx"][t, n].reshape(-1).tolist())
        assert set(st["experts"]) == routed           # staged == routed, nothing dropped
        assert st["prefetched"] == (t > 0 and n > 0)


def test_head_onehot_history_uses_current_and_previous_routing():
    dims = Dims(d=64, E=16, I=64, k=4, r=2, L=2, head_layers=(0,), head_onehot=1)
    dense = {n: synth.layer_dense(12, n, dims) for n in range(2)}
    hs = np.stack([synth.hidden(12, t, 2, 1, 64) for t in range(3)])
    out = O.stack_decode(hs, dense.__getitem__, lambda n, e: synth.expert_blob(12, n, e, dims),
                         lambda n: synth.shared_blob(12, n, dims), dims)
    for t in range(3):
        x = O.rmsnorm(O.bf16_to_f64(hs[t, 0]), dense[0]["norm_w"], dims.eps)[0]
        prev = out["idx"][t - 1, 0, 0] if t else None
        z, p = O.prerouter_head(x, dense[0], dims, out["idx"][t, 0, 0], prev)
        assert np.array_equal(out["head_logits"][t, 0, 0], z)
        assert out["pred"][t, 0, 0].tolist() == p.tolist()


# ---------------------------------------------------------------------------------------
# the fully reactive mode (no prerouter) and the persistent sticky-slot sets
# ---------------------------------------------------------------------------------------
def test_reactive_stack_is_each_layer_on_its_own_router():
    """prediction=False: every layer of every step equals the single-layer oracle with the
    layer's own router (a brute-force reduction), and no head runs."""
    S, B = 2, 2
    hs = np.stack([synth.hidden(13, t, SMALL.L, B, SMALL.d) for t in range(S)])
    dense = {n: synth.layer_dense(13, n, SMALL) for n in range(SMALL.L)}
    out = O.stack_decode(hs, dense.__getitem__, lambda n, e: synth.expert_blob(13, n, e, SMALL),
                         lambda n: synth.shared_blob(13, n, SMALL), SMALL, prediction=False)
    assert np.all(out["pred"] == -1)
    for t in range(S):
        for n in range(SMALL.L):
            ref = O.moe_layer(hs[t, n], dense[n], lambda e, n=n: synth.expert_blob(13, n, e, SMALL),
                              synth.shared_blob(13, n, SMALL), SMALL)
            assert np.array_equal(out["idx"][t, n], ref["idx"])
            assert np.array_equal(out["y"][t, n], ref["y"])


def test_sticky_plan_hand_worked_example():
    """One layer, one stream, k=2, three slots; worked by hand:
    t0 [0,1]: copies 0->slot0, 1->slot1 (empty slots, lower first)          -> [0, 1, -]
    t1 [1,2]: 1 hit; 2 -> slot2 (empty, never needed, before slot0)        -> [0, 1, 2]
    t2 [3,0]: 0 hit; 3 -> slot1 (slots 1 and 2 both last needed at t1)     -> [0, 3, 2]
    t3 [1,2]: 2 hit; 1 -> slot0 (slots 0 and 1 both last needed at t2)     -> [1, 3, 2]"""
    dims = Dims(d=64, E=8, I=64, k=2, r=0, L=1, head_layers=())
    idx = np.array([[[[0, 1]]], [[[1, 2]]], [[[3, 0]]], [[[1, 2]]]], np.int32)
    plan = O.sticky_plan(idx, dims, 3)
    assert plan[(0, 0)]["copies"] == [(0, 0), (1, 1)] and plan[(0, 0)]["hits"] == 0
    assert plan[(1, 0)]["copies"] == [(2, 2)] and plan[(1, 0)]["hits"] == 1
    assert plan[(2, 0)]["copies"] == [(1, 3)] and plan[(2, 0)]["hits"] == 1
    assert plan[(3, 0)]["copies"] == [(0, 1)] and plan[(3, 0)]["hits"] == 1
    assert plan[(3, 0)]["content"] == [1, 3, 2]


def test_sticky_plan_invariants():
    """k slots at one stream rewrite exactly the experts that changed since the previous
    token; with a set as large as every expert the layer ever sees, each expert is copied
    once; every step's experts are resident after its copies (nothing dropped)."""
    dims = Dims(d=64, E=16, I=64, k=4, r=0, L=3, head_layers=())
    rng = np.random.default_rng(5)
    S = 12
    idx = np.stack([[rng.permutation(16)[:4][None] for _ in range(3)] for _ in range(S)]).astype(np.int32)
    plan = O.sticky_plan(idx, dims, 4)
    for t in range(S):
        for n in range(3):
            now = set(idx[t, n, 0].tolist())
            before = set(idx[t - 1, n, 0].tolist()) if t else set()
            assert len(plan[(t, n)]["copies"]) == len(now - before)
            assert plan[(t, n)]["hits"] == len(now & before)
            assert now <= set(plan[(t, n)]["content"])
    big = O.sticky_plan(idx, dims, 16)
    for n in range(3):
        total = sum(len(big[(t, n)]["copies"]) for t in range(S))
        assert total == len(set(idx[:, n].reshape(-1).tolist()))
