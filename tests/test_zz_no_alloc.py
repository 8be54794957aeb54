"""The allocation-free MoE block entry point (for callers that cannot allocate device
memory) must give the same output as the context-based entry point, on two calls in a
row (the second call reuses the library's fixed scratch array left by the first)."""
import numpy as np
import pytest
import torch

import synth
from synth import Dims
from synth.device import bf16_tensor, layer_tensors
from parity import check_y

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_context_forward_twice(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    dims = Dims(d=2048, E=256, I=512, k=4, r=16, L=1, head_layers=(0,))
    ly, hd = layer_tensors(33, 0, dims, "cuda")
    ctx = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, 1, 64)
    ctx.register_model([ly], [hd])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call, T in enumerate((7, 33)):
        h = bf16_tensor(synth.hidden(330 + call, 0, 1, T, dims.d)[0], "cuda")
        ref = torch.empty((T, dims.d), dtype=torch.float32, device="cuda")
        ctx.moe_layer_forward(0, h, y_f32=ref)
        ctx.sync_status()
        out = torch.empty((T, dims.d), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, dims.k), dtype=torch.int32, device="cuda")
        e0.moe_layer_forward_noalloc(ctx.dims, ly, h, y_f32=out, idx=idx, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        check_y(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), f"call {call}")
    ctx.close()


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    dims = Dims(d=2048, E=256, I=512, k=4, r=16, L=1, head_layers=(0,))
    ly, _ = layer_tensors(34, 0, dims, "cuda")
    h = torch.zeros((4096, dims.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(e0.E0Error) as ei:
        e0.moe_layer_forward_noalloc(e0.make_dims(dims.d, dims.E, dims.I, dims.k, dims.r), ly, h)
    assert ei.value.status == "INVALID_ARG" and "scratch" in str(ei.value)
