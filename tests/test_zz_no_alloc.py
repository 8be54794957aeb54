"""The allocation-free MoE block entry point, for callers that cannot allocate device
memory (a serving runtime whose memory plan is fixed at start-up, code running while
another component owns the allocator, code that must not risk an allocation's implicit
synchronisation).  It must give the same output as the context-based entry point, and
the oracle's, on two calls in a row (the second call reuses the library's fixed scratch
array left by the first), with its own router or a given routing; it must report bad
routing through the caller's status word and reject sizes beyond its scratch."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from synth import Dims
from synth.device import bf16_tensor, layer_tensors
from parity import check_y, idx_ok

pytestmark = pytest.mark.gpu

DIMS = Dims(d=2048, E=256, I=512, k=4, r=16, L=1, head_layers=(0,))


def _oracle(seed, h_bits, route=None):
    dense = synth.layer_dense(seed, 0, DIMS)
    return O.moe_layer(h_bits, dense, lambda e: synth.expert_blob(seed, 0, e, DIMS),
                       synth.shared_blob(seed, 0, DIMS), DIMS, route_idx=route)


def test_noalloc_forward_matches_context_forward_and_oracle_twice(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    seed = 33
    ly, hd = layer_tensors(seed, 0, DIMS, "cuda")
    ctx = e0.Context(DIMS.d, DIMS.E, DIMS.I, DIMS.k, DIMS.r, 1, 64)
    ctx.register_model([ly], [hd])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, T in enumerate((7, 33)):
        hb = synth.hidden(330 + call, 0, 1, T, DIMS.d)[0]
        h = bf16_tensor(hb, "cuda")
        ref = torch.empty((T, DIMS.d), dtype=torch.float32, device="cuda")
        ctx.moe_layer_forward(0, h, y_f32=ref)
        ctx.sync_status()
        out = torch.empty((T, DIMS.d), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, DIMS.k), dtype=torch.int32, device="cuda")
        e0.moe_layer_forward_noalloc(ctx.dims, ly, h, y_f32=out, idx=idx, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        check_y(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), f"call {call} vs context")
        orc = _oracle(seed, hb)
        gi = idx.cpu().numpy()
        for t in range(T):
            assert idx_ok(gi[t], orc["logits"][t], orc["idx"][t], DIMS.k), (call, t)
        if np.array_equal(gi, orc["idx"]):
            check_y(out.cpu().numpy(), orc["y"], f"call {call} vs oracle")
        else:   # a near tie went the other admissible way: follow it
            check_y(out.cpu().numpy(), _oracle(seed, hb, route=gi)["y"], f"call {call} vs oracle")
    ctx.close()


def test_noalloc_with_given_routing_and_without_status_word(cuda_ok):
    """route_idx given (prediction as routing; a row of -1 uses the own router), once with
    the status word and once without it."""
    import int4_expert_streaming_prerouter_b200 as e0
    seed, T = 34, 9
    ly, _ = layer_tensors(seed, 0, DIMS, "cuda")
    hb = synth.hidden(340, 0, 1, T, DIMS.d)[0]
    rng = np.random.default_rng(34)
    route = np.stack([rng.permutation(DIMS.E)[:DIMS.k] for _ in range(T)]).astype(np.int32)
    route[3] = -1
    orc = _oracle(seed, hb, route=route)
    dims = e0.make_dims(DIMS.d, DIMS.E, DIMS.I, DIMS.k, DIMS.r)
    for with_status in (True, False):
        status = torch.zeros(1, dtype=torch.int32, device="cuda") if with_status else None
        out = torch.empty((T, DIMS.d), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, DIMS.k), dtype=torch.int32, device="cuda")
        e0.moe_layer_forward_noalloc(dims, ly, bf16_tensor(hb, "cuda"), route_idx=torch.from_numpy(route).cuda(),
                                     y_f32=out, idx=idx, dev_status=status)
        torch.cuda.synchronize()
        if with_status:
            assert int(status.item()) == 0
        gi = idx.cpu().numpy()
        for t in range(T):
            if route[t, 0] >= 0:
                assert np.array_equal(gi[t], route[t])
            else:
                assert idx_ok(gi[t], orc["logits"][t], orc["idx"][t], DIMS.k)
        check_y(out.cpu().numpy(), _oracle(seed, hb, route=gi)["y"], f"given routing, status={with_status}")


def test_noalloc_reports_bad_routing_in_the_status_word(cuda_ok):
    """An index out of range sets bit 1 and a duplicated index bit 2 (the kernels clamp the
    bad index and go on; nothing is read out of bounds)."""
    import int4_expert_streaming_prerouter_b200 as e0
    ly, _ = layer_tensors(35, 0, DIMS, "cuda")
    dims = e0.make_dims(DIMS.d, DIMS.E, DIMS.I, DIMS.k, DIMS.r)
    h = bf16_tensor(synth.hidden(350, 0, 1, 2, DIMS.d)[0], "cuda")
    for bad, bit in (([[1, 2, 3, 999], [0, 1, 2, 3]], 1), ([[4, 4, 5, 6], [0, 1, 2, 3]], 2)):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        e0.moe_layer_forward_noalloc(dims, ly, h, route_idx=torch.tensor(bad, dtype=torch.int32, device="cuda"),
                                     dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == bit, (bad, int(status.item()))


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    ly, _ = layer_tensors(34, 0, DIMS, "cuda")
    h = torch.zeros((4096, DIMS.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(e0.E0Error) as ei:
        e0.moe_layer_forward_noalloc(e0.make_dims(DIMS.d, DIMS.E, DIMS.I, DIMS.k, DIMS.r), ly, h)
    assert ei.value.status == "INVALID_ARG" and "scratch" in str(ei.value)
