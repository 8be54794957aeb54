"""GPU parity of the decode loop over the stack (prediction-as-routing) against the oracle,
on a small stack in full and on the full-size 40-layer model on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from synth import Dims
from synth.device import bf16_tensor, layer_tensors
from parity import bf16_bits_to_np, check_bf16, check_y, choose_following, idx_ok
from stack_helpers import build, compare_steps, oracle_steps, run_steps

pytestmark = pytest.mark.gpu

SMALL = Dims(d=256, E=16, I=128, k=4, r=8, L=4, head_layers=(0, 1, 2))


@pytest.mark.parametrize("B", [1, 5])
def test_small_stack_decode_matches_oracle(cuda_ok, B):
    ctx, _, _ = build(SMALL, 60 + B, 16)
    S = 4
    gpu = run_steps(ctx, SMALL, 60 + B, B, S)
    ref = oracle_steps(SMALL, 60 + B, B, S, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    # prediction is the routing: every predicted layer at t > 0 used the t-1 prediction
    for t in range(1, S):
        for n in range(1, SMALL.L):
            assert np.array_equal(gpu[2][t, n], gpu[3][t - 1, n - 1])
    ctx.close()


def test_small_stack_chained_matches_oracle(cuda_ok):
    ctx, _, _ = build(SMALL, 70, 8)
    gpu = run_steps(ctx, SMALL, 70, 2, 3, chained=True)
    ref = oracle_steps(SMALL, 70, 2, 3, gpu[2], gpu[3], chained=True)
    compare_steps(SMALL, gpu, ref)
    ctx.close()


def test_onehot_head_stack(cuda_ok):
    dims = Dims(d=256, E=16, I=128, k=4, r=8, L=3, head_layers=(0, 1), head_onehot=1)
    ctx, _, _ = build(dims, 71, 8)
    gpu = run_steps(ctx, dims, 71, 3, 4)
    ref = oracle_steps(dims, 71, 3, 4, gpu[2], gpu[3])
    compare_steps(dims, gpu, ref)
    ctx.close()


def test_step_sequence_is_enforced(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    ctx, _, _ = build(SMALL, 72, 8)
    h = bf16_tensor(synth.hidden(72, 0, SMALL.L, 2, SMALL.d), "cuda")
    with pytest.raises(e0.E0Error):
        ctx.stack_decode(h, 3)
    ctx.stack_decode(h, 0)
    with pytest.raises(e0.E0Error):
        ctx.stack_decode(h[:, :1].contiguous(), 1)   # B changed mid-sequence
    ctx.close()


# ---------------------------------------------------------------------------------------
# full-size model (40 layers, d=2048, E=256, I=512, r=16, heads on 0..32), batch 1
# ---------------------------------------------------------------------------------------
FULL = synth.WORKLOADS["decode_b1_l40"]["dims"]


@pytest.fixture(scope="module")
def full_model(cuda_ok):
    ctx, lys, hds = build(FULL, 1, 64)
    yield ctx
    ctx.close()


@pytest.mark.parametrize("mode", [4, 1])
def test_full_size_decode_b1_sampled(full_model, mode):
    """Two steps of the 40-layer stack at B=1 (the phased kernels, the default, and the
    one-launch kernel): every layer's routing and head prediction exactly, and y on every
    layer of both steps."""
    S = 2
    full_model.debug_decode_mode(mode)
    try:
        gpu = run_steps(full_model, FULL, 1, 1, S)
    finally:
        full_model.debug_decode_mode(0)
    ref = oracle_steps(FULL, 1, 1, S, gpu[2], gpu[3])
    compare_steps(FULL, gpu, ref)


def test_full_size_decode_b8_sampled_layers(full_model):
    """B=8 streams, one step, every layer's routing; y checked on a sample of layers."""
    B, dims = 8, FULL
    gpu = run_steps(full_model, dims, 2, B, 1)       # inputs from seed 2, weights from seed 1
    hs = synth.hidden(2, 0, dims.L, B, dims.d)
    for n in (0, 1, 17, 33, 34, 39):
        dense = synth.layer_dense(1, n, dims)
        ref = O.moe_layer(hs[n], dense, lambda e: synth.expert_blob(1, n, e, dims), synth.shared_blob(1, n, dims),
                          dims, choose=lambda t, c, a: next((x for x in a if np.array_equal(x, gpu[2][0, n, t])), c))
        for b in range(B):
            assert idx_ok(gpu[2][0, n, b], ref["logits"][b], ref["idx"][b], dims.k)
        check_y(gpu[1][0, n], ref["y"], f"layer {n}")


# ---------------------------------------------------------------------------------------
# the one-launch decode kernel (B = 1) against the per-layer kernels and the oracle
# ---------------------------------------------------------------------------------------
def test_one_launch_decode_equals_general_path_small(cuda_ok):
    ctx, _, _ = build(SMALL, 90, 4)
    ctx.debug_decode_mode(1)
    ref, _, _ = build(SMALL, 90, 4)
    ref.debug_force_general(True)
    for t in range(5):
        h = bf16_tensor(synth.hidden(91, t, SMALL.L, 1, SMALL.d), "cuda")
        ya32 = torch.empty((SMALL.L, 1, SMALL.d), dtype=torch.float32, device="cuda")
        yb32 = torch.empty_like(ya32)
        ctx.stack_decode(h, t, y_f32=ya32)
        ref.stack_decode(h, t, y_f32=yb32)
        ctx.sync_status()
        ref.sync_status()
        ia, pa = ctx.get_routing(1)
        ib, pb = ref.get_routing(1)
        assert np.array_equal(ia, ib) and np.array_equal(pa, pb)
        for n in range(SMALL.L):
            check_y(ya32[n].cpu().numpy(), yb32[n].cpu().numpy().astype(np.float64), f"t{t} l{n}")
    ctx.close()
    ref.close()


def _decode_bits(ctx, dims, seed, S, flat):
    ctx.debug_decode_mode(1)
    ctx.debug_decode_flat(flat)
    out = []
    for t in range(S):
        h = bf16_tensor(synth.hidden(seed, t, dims.L, 1, dims.d), "cuda")
        y32 = torch.empty((dims.L, 1, dims.d), dtype=torch.float32, device="cuda")
        y = ctx.stack_decode(h, t, y_f32=y32)
        ctx.sync_status()
        idx, pred = ctx.get_routing(1)
        out.append((y.view(torch.int16).cpu().numpy().copy(), y32.cpu().numpy().copy(), idx, pred))
    return out


def _same(base, got, what):
    for t, (a, b) in enumerate(zip(base, got)):
        for u, v in zip(a, b):
            assert np.array_equal(u, v), f"{what} step {t}"


@pytest.mark.parametrize("heads", [(0, 1, 2), (0, 2), ()])
def test_one_launch_decode_flat_schedule_is_bitwise_in_order(cuda_ok, heads):
    """The flat schedule (each phase's units over all layers split across the CTAs)
    changes who computes what and in which order, not the arithmetic: outputs, routing and
    predictions are bit-identical to in-order execution, for stacks of mostly predicted
    layers, reactive layers in between, and no heads at all (every layer reactive)."""
    dims = Dims(d=256, E=16, I=128, k=4, r=8, L=6, head_layers=heads)
    ctx, _, _ = build(dims, 95, 4)
    base = _decode_bits(ctx, dims, 96, 4, 0)
    _same(base, _decode_bits(ctx, dims, 96, 4, 1), "flat")
    ctx.close()


def test_full_size_decode_flat_schedule_is_bitwise_in_order(full_model):
    """The bench's configuration (40 layers, flat schedule) against in-order execution."""
    try:
        base = _decode_bits(full_model, FULL, 7, 2, 0)
        got = _decode_bits(full_model, FULL, 7, 2, 1)
    finally:
        full_model.debug_decode_flat(1)
        full_model.debug_decode_mode(0)
    _same(base, got, "flat")


def test_one_launch_decode_chained_b1(cuda_ok):
    ctx, _, _ = build(SMALL, 92, 4)
    ctx.debug_decode_mode(1)
    gpu = run_steps(ctx, SMALL, 92, 1, 3, chained=True)
    ref = oracle_steps(SMALL, 92, 1, 3, gpu[2], gpu[3], chained=True)
    compare_steps(SMALL, gpu, ref)
    ctx.close()


def test_one_launch_decode_onehot_head_b1(cuda_ok):
    dims = Dims(d=256, E=16, I=128, k=4, r=8, L=3, head_layers=(0, 1), head_onehot=1)
    ctx, _, _ = build(dims, 93, 4)
    ctx.debug_decode_mode(1)
    gpu = run_steps(ctx, dims, 93, 1, 4)
    ref = oracle_steps(dims, 93, 1, 4, gpu[2], gpu[3])
    compare_steps(dims, gpu, ref)
    ctx.close()


def test_one_launch_decode_bounded_wait_reports_timeout(cuda_ok):
    """A CTA that waits on a word nothing writes gives up after the budget; the launch ends,
    the status is TIMEOUT, and the context decodes correctly afterwards."""
    import int4_expert_streaming_prerouter_b200 as e0
    ctx, _, _ = build(SMALL, 94, 4)
    ctx.debug_decode_mode(1)
    h = bf16_tensor(synth.hidden(94, 0, SMALL.L, 1, SMALL.d), "cuda")
    ctx.debug_decode_stall(0, 20_000_000)          # 20 ms budget
    ctx.stack_decode(h, 0)
    with pytest.raises(e0.E0Error) as ei:
        ctx.sync_status()
    assert ei.value.status == "TIMEOUT"
    ctx.debug_decode_stall(-1, 0)
    gpu = run_steps(ctx, SMALL, 94, 1, 2)
    ref = oracle_steps(SMALL, 94, 1, 2, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    ctx.close()


def test_one_launch_decode_reports_activations_beyond_fp16(cuda_ok):
    """The one-launch kernel holds activations as fp16 tensor-core operands: a finite
    activation beyond that range latches a device error instead of a silent infinity, and
    once the input is back in range the context decodes correctly again."""
    import int4_expert_streaming_prerouter_b200 as e0
    ctx, lys, _ = build(SMALL, 95, 4)
    ctx.debug_decode_mode(1)
    gamma = lys[1]["norm_w"]
    saved = gamma.clone()
    gamma.fill_(2.0e5)     # |x| = |RMSNorm(h)| * 2e5 reaches well past 65520 (finite in bf16)
    h = bf16_tensor(synth.hidden(95, 0, SMALL.L, 1, SMALL.d), "cuda")
    ctx.stack_decode(h, 0)
    with pytest.raises(e0.E0Error) as ei:
        ctx.sync_status()
    assert ei.value.status == "DEVICE"
    gamma.copy_(saved)
    gpu = run_steps(ctx, SMALL, 95, 1, 2)
    ref = oracle_steps(SMALL, 95, 1, 2, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    ctx.close()


@pytest.mark.parametrize("B", [1, 5])
def test_graph_replay_decode_matches_oracle(cuda_ok, B):
    """The decode step replayed as a captured CUDA graph of the per-layer kernels."""
    ctx, _, _ = build(SMALL, 95 + B, 8)
    ctx.debug_decode_mode(2)
    S = 3
    gpu = run_steps(ctx, SMALL, 95 + B, B, S)
    ref = oracle_steps(SMALL, 95 + B, B, S, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    ctx.close()


@pytest.mark.parametrize("B", [1, 3])
def test_host_buffer_decode_matches_device_buffers(cuda_ok, B):
    """e0_moe_stack_decode_host (pinned host input and outputs, copies overlapped with the
    kernels through two alternating staging buffers) gives bit-identical outputs and
    routing to the device-buffer call over a sequence of steps."""
    seed, S = 71, 5
    ctx_d, _, _ = build(SMALL, seed, 4)
    ctx_h, _, _ = build(SMALL, seed, 4)
    ys, y32s, idxs, preds = run_steps(ctx_d, SMALL, seed, B, S)
    shape = (SMALL.L, B, SMALL.d)
    h_host = [bf16_tensor(synth.hidden(seed, t, SMALL.L, B, SMALL.d), "cpu").pin_memory() for t in range(S)]
    y_host = [torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(S)]
    f_host = [torch.empty(shape, dtype=torch.float32).pin_memory() for _ in range(S)]
    for t in range(S):
        ctx_h.stack_decode_host(h_host[t], t, y_host[t], y_f32_host=f_host[t])
    ctx_h.host_io_wait()
    torch.cuda.synchronize()
    ctx_h.sync_status()
    idx, pred = ctx_h.get_routing(B)
    assert np.array_equal(idx, idxs[-1]) and np.array_equal(pred, preds[-1])
    for t in range(S):
        assert np.array_equal(bf16_bits_to_np(y_host[t]), ys[t]), f"bf16 outputs differ at step {t}"
        assert np.array_equal(f_host[t].numpy().astype(np.float64), y32s[t]), f"fp32 outputs differ at step {t}"


# ---------------------------------------------------------------------------------------
# batched decode on the full model (the multi-stream batches 32 and 64)
# ---------------------------------------------------------------------------------------
def _oracle_routing(dims, hs_layer, dense):
    """x, router logits and (for a head layer) head logits of every token of one layer."""
    x = O.rmsnorm(O.bf16_to_f64(hs_layer), dense["norm_w"], dims.eps)
    lg = O.router_logits(dense["router_w"], x)
    hl = O.router_logits(dense["head_w"], x) if dense.get("head_w") is not None else None
    return x, lg, hl


@pytest.mark.parametrize("B", [32, 64])
def test_full_size_decode_batched_routing_and_sampled_outputs(full_model, B):
    """Two steps of B streams through the 40-layer model: every layer's routing of every
    stream (own router at step 0 and on layers without a predictor; the previous step's
    head prediction elsewhere) and every head prediction against the oracle's logits, and
    y of sampled streams on sampled layers of both steps against the oracle's MoE block."""
    dims, wseed, iseed, S = FULL, 1, 3 + B, 2
    gpu = run_steps(full_model, dims, iseed, B, S)
    _, y32, idx, pred = gpu
    pl = O.predicted_layers(dims)
    streams = sorted({0, 1, B // 2, B - 1} | set(range(3, B, max(1, B // 4))))
    for t in range(S):
        hs = synth.hidden(iseed, t, dims.L, B, dims.d)
        for n in range(dims.L):
            dense = synth.layer_dense(wseed, n, dims)
            x, lg, hl = _oracle_routing(dims, hs[n], dense)
            for b in range(B):
                if t > 0 and n in pl:
                    assert np.array_equal(idx[t, n, b], pred[t - 1, n - 1, b]), (t, n, b)
                else:
                    assert idx_ok(idx[t, n, b], lg[b], O.topk(lg[b], dims.k), dims.k), (t, n, b)
                if hl is not None:
                    assert idx_ok(pred[t, n, b], hl[b], O.topk(hl[b], dims.k), dims.k), ("head", t, n, b)
            if n in (0, 1, 33, 34, 39):
                ref = O.moe_layer(hs[n][streams], dense, lambda e: synth.expert_blob(wseed, n, e, dims),
                                  synth.shared_blob(wseed, n, dims), dims, route_idx=idx[t, n][streams])
                check_y(y32[t, n][streams], ref["y"], f"B={B} step {t} layer {n}")


# ---------------------------------------------------------------------------------------
# exact ties: equal logits must resolve to the lowest indices, with no alternative admitted
# ---------------------------------------------------------------------------------------
def test_exact_ties_take_the_lowest_indices(cuda_ok):
    """Zero router and head weights make every logit 0: every routing and every prediction
    must be exactly [0, 1, 2, 3] at E = 256, on the one-launch kernel (B = 1), the per-layer
    kernels (B = 3), one MoE block, and the tensor-core prefill path (T = 160); the gates
    are then 1/4 each and y matches the oracle."""
    import int4_expert_streaming_prerouter_b200 as e0
    dims = Dims(d=256, E=256, I=128, k=4, r=8, L=3, head_layers=(0, 1))
    seed = 97
    lys, hds = [], []
    denses = []
    for n in range(dims.L):
        dense = synth.layer_dense(seed, n, dims)
        dense["router_w"] = np.zeros_like(dense["router_w"])
        if dense["head_w"] is not None:
            dense["head_w"] = np.zeros_like(dense["head_w"])
        denses.append(dense)
        ly, hd = layer_tensors(seed, n, dims, "cuda", dense=dense)
        lys.append(ly)
        hds.append(hd)
    want = np.arange(dims.k, dtype=np.int32)
    for B in (1, 3):
        ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, 256)
        ctx.register_model(lys, hds)
        for t in range(2):
            h = bf16_tensor(synth.hidden(seed, t, dims.L, B, dims.d), "cuda")
            y32 = torch.empty((dims.L, B, dims.d), dtype=torch.float32, device="cuda")
            ctx.stack_decode(h, t, y_f32=y32)
            ctx.sync_status()
            idx, pred = ctx.get_routing(B)
            for n in range(dims.L):
                for b in range(B):
                    assert np.array_equal(idx[n, b], want), (B, t, n, b, idx[n, b])
                    if n in dims.head_layers:
                        assert np.array_equal(pred[n, b], want), (B, t, n, b, pred[n, b])
            hs = synth.hidden(seed, t, dims.L, B, dims.d)
            for n in (0, 2):
                ref = O.moe_layer(hs[n], denses[n], lambda e, n=n: synth.expert_blob(seed, n, e, dims),
                                  synth.shared_blob(seed, n, dims), dims)
                assert np.array_equal(ref["idx"], np.tile(want, (B, 1)))
                check_y(y32[n].cpu().numpy().astype(np.float64), ref["y"], f"ties B={B} t={t} n={n}")
        # one block and the tensor-core prefill path
        for T, path in ((5, 1), (160, 2)):
            ctx.debug_prefill_path(path)
            hb = synth.hidden(seed + T, 0, 1, T, dims.d)[0]
            idx_t = torch.empty((T, dims.k), dtype=torch.int32, device="cuda")
            gates = torch.empty((T, dims.k), dtype=torch.float32, device="cuda")
            ctx.moe_layer_forward(0, bf16_tensor(hb, "cuda"), idx=idx_t, gates=gates)
            ctx.sync_status()
            assert np.array_equal(idx_t.cpu().numpy(), np.tile(want, (T, 1))), (T, path)
            assert np.allclose(gates.cpu().numpy(), 0.25, rtol=0, atol=1e-7)
        ctx.close()


# ---------------------------------------------------------------------------------------
# the phased kernels (unchained steps, B <= 8): every head form, routing width and batch
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("heads,onehot,hidden,k,B", [
    ((0, 1, 2), 0, 0, 4, 1), ((0, 1, 2), 0, 0, 4, 3), ((0, 1, 2), 0, 0, 4, 8), ((0, 2), 0, 0, 4, 2),
    ((), 0, 0, 4, 1), ((0, 1, 2), 1, 0, 4, 2), ((0, 1, 2), 1, 64, 4, 1), ((0, 1), 0, 32, 4, 5),
    ((0, 1, 2), 0, 0, 2, 1), ((0, 1, 2), 0, 0, 8, 3), ((0, 1, 2), 0, 0, 4, 20), ((0, 2), 1, 32, 4, 11)])
def test_phased_decode_matches_oracle(cuda_ok, heads, onehot, hidden, k, B):
    dims = Dims(d=256, E=16, I=128, k=k, r=8, L=4, head_layers=heads, head_onehot=onehot, head_hidden=hidden)
    seed = 120 + 7 * k + B + hidden
    ctx, _, _ = build(dims, seed, max(B, 8))
    ctx.debug_decode_mode(4)
    S = 3
    gpu = run_steps(ctx, dims, seed, B, S)
    ref = oracle_steps(dims, seed, B, S, gpu[2], gpu[3])
    compare_steps(dims, gpu, ref)
    ctx.close()


def test_phased_decode_full_head_k8_full_size(cuda_ok):
    """The full prerouter head (fc1 -> erf-GELU -> fc2 plus the linear path over
    u = [x; onehot(cur); onehot(prev)], width d + 2E = 2560, hidden 256) with routing width
    k = 8 on the full-size geometry, 6 layers, two steps at B = 2."""
    dims = Dims(d=2048, E=256, I=512, k=8, r=16, L=6, head_layers=(0, 1, 2, 3), head_onehot=1, head_hidden=256)
    ctx, _, _ = build(dims, 130, 8)
    ctx.debug_decode_mode(4)
    gpu = run_steps(ctx, dims, 130, 2, 2)
    ref = oracle_steps(dims, 130, 2, 2, gpu[2], gpu[3])
    compare_steps(dims, gpu, ref)
    ctx.close()
