"""Streaming tier on the GPU: experts live in pinned host memory and are staged into an
HBM slot pool.  Every streamed step must match the oracle (routing, head predictions and
outputs of every layer); the slot tags that each layer's expert kernels read must hold
exactly the experts of the oracle's routing (prediction-as-routing: staged set = routed
set, nothing dropped); the persistent per-layer sets must copy exactly what the oracle's
sticky-slot plan copies; and host-injected faults (a refused copy, a wrong slot tag) must
come back as errors."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from synth import Dims
from synth.device import bf16_tensor, layer_tensors, pinned_expert_store
from stack_helpers import compare_steps, oracle_steps, run_steps

pytestmark = pytest.mark.gpu

SMALL = Dims(d=256, E=16, I=128, k=4, r=8, L=5, head_layers=(0, 1, 2))


def device_bytes(ptr: int, n: int) -> np.ndarray:
    """Copy n bytes at a device address to the host (a read-only view through the CUDA
    array interface)."""
    class _View:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "|u1", "data": (ptr, False), "version": 3}
    torch.cuda.synchronize()
    return torch.as_tensor(_View(), device="cuda").cpu().numpy()


def build_streaming(dims, seed, B, pool_layers=2, slots=None, store=None):
    import int4_expert_streaming_prerouter_b200 as e0
    lys, hds = zip(*[layer_tensors(seed, n, dims, "cuda", resident=False) for n in range(dims.L)])
    st = e0.Context(dims.d, dims.E, dims.I, dims.k, dims.r, dims.L, B)
    st.register_model(list(lys), list(hds))
    store = pinned_expert_store(seed, dims) if store is None else store
    slots = slots or min(dims.E, B * dims.k)
    st.stream_register(store, pool_layers=pool_layers, slots_per_layer=slots)
    log = torch.full((dims.L, slots), -7, dtype=torch.int32, device="cuda")
    st.debug_stream_log(log)
    return st, store, log, slots


def run_logged(st, dims, seed, B, S, log):
    """Streamed steps; the per-layer slot tags the expert kernels read, after each step."""
    logs = []
    gpu = run_steps(st, dims, seed, B, S, streaming=True, after_step=lambda t: logs.append(log.cpu().numpy().copy()))
    return gpu, np.stack(logs)


def check_slot_sets_hold_the_oracle_routing(ref_idx, logs, exact=True):
    S, L = ref_idx.shape[:2]
    for t in range(S):
        for n in range(L):
            routed = set(ref_idx[t, n].reshape(-1).tolist())
            held = set(int(e) for e in logs[t, n] if e >= 0)
            if exact:
                assert held == routed, (t, n, sorted(held), sorted(routed))
            else:
                assert routed <= held, (t, n, sorted(held), sorted(routed))


@pytest.mark.parametrize("B", [1, 3])
def test_streaming_matches_oracle_and_slot_sets_hold_the_routed_experts(cuda_ok, B):
    """Double-buffered slot sets (2 sets for 5 layers): routing, predictions and y of every
    layer and step equal the oracle's; the slot tags each layer's kernels read hold exactly
    the oracle's routed experts; the last two layers' slots hold the host store's bytes;
    the counters add up (prefetched = the predicted layers' experts, nothing dropped)."""
    S, seed = 4, 80 + B
    st, store, log, slots = build_streaming(SMALL, seed, B)
    gpu, logs = run_logged(st, SMALL, seed, B, S, log)
    ref = oracle_steps(SMALL, seed, B, S, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    check_slot_sets_hold_the_oracle_routing(ref["idx"], logs)
    plan = O.staging_plan(ref["idx"], SMALL)
    pre = sum(len(p["experts"]) for p in plan.values() if p["prefetched"])
    ond = sum(len(p["experts"]) for p in plan.values() if not p["prefetched"])
    stats = st.stats()
    assert stats["dropped"] == 0 and stats["hit_experts"] == 0
    assert stats["prefetched_experts"] == pre and stats["ondemand_experts"] == ond
    assert stats["staged_experts"] == pre + ond
    assert stats["staged_bytes"] == stats["staged_experts"] * synth.blob_bytes(SMALL.d, SMALL.I)
    assert stats["stage_ms"] > 0
    # the bytes in the pool: sets 1 and 0 last held layers 3 and 4 of the last step
    nb = synth.blob_bytes(SMALL.d, SMALL.I)
    for n in (SMALL.L - 2, SMALL.L - 1):
        for s, e in enumerate(logs[-1, n]):
            if e < 0:
                continue
            got = device_bytes(st.debug_pool_slot(n % 2, s), nb)
            assert np.array_equal(got, store[n, e].numpy()), (n, s, e)
    st.close()


@pytest.mark.parametrize("B,slots", [(1, 4), (2, 12)])
def test_persistent_sets_copy_only_what_the_sticky_plan_copies(cuda_ok, B, slots):
    """One persistent set per layer (sticky slots): with k slots at one stream only the
    experts that changed since the previous token are copied; with 12 slots at two streams
    the sets act as least-recently-used caches.  Copies, hits and the slot contents each
    layer computed with equal the oracle's sticky-slot plan on the oracle's routing, and
    the outputs equal the oracle's."""
    S, seed = 6, 84 + B
    st, store, log, _ = build_streaming(SMALL, seed, B, pool_layers=SMALL.L, slots=slots)
    gpu, logs = run_logged(st, SMALL, seed, B, S, log)
    ref = oracle_steps(SMALL, seed, B, S, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    plan = O.sticky_plan(ref["idx"], SMALL, slots)
    copies = sum(len(p["copies"]) for p in plan.values())
    hits = sum(p["hits"] for p in plan.values())
    stats = st.stats()
    assert stats["staged_experts"] == copies and stats["hit_experts"] == hits and stats["dropped"] == 0
    for (t, n), p in plan.items():
        assert logs[t, n].tolist() == p["content"], (t, n, logs[t, n].tolist(), p["content"])
    check_slot_sets_hold_the_oracle_routing(ref["idx"], logs, exact=False)
    st.close()


def test_reactive_mode_matches_the_oracle_without_prediction(cuda_ok):
    """Fully reactive streaming (no prerouter): every layer routes with its own router and
    stages on demand; the oracle without prediction gives the same routing and outputs;
    every copy is on demand and no prediction is reported."""
    B, S, seed = 2, 3, 88
    st, store, log, _ = build_streaming(SMALL, seed, B)
    st.stream_mode(True)
    gpu, logs = run_logged(st, SMALL, seed, B, S, log)
    ref = oracle_steps(SMALL, seed, B, S, gpu[2], gpu[3], prediction=False)
    compare_steps(SMALL, gpu, ref, prediction=False)
    check_slot_sets_hold_the_oracle_routing(ref["idx"], logs)
    stats = st.stats()
    assert stats["prefetched_experts"] == 0
    assert stats["ondemand_experts"] == sum(len(set(ref["idx"][t, n].reshape(-1).tolist()))
                                            for t in range(S) for n in range(SMALL.L))
    # back to prefetch: a new sequence must start at step 0
    import int4_expert_streaming_prerouter_b200 as e0
    st.stream_mode(False)
    with pytest.raises(e0.E0Error):
        st.stack_decode(bf16_tensor(synth.hidden(seed, S, SMALL.L, B, SMALL.d), "cuda"), S, streaming=True)
    st.close()


FULL = synth.WORKLOADS["stream_b1_l40"]["dims"]


def test_full_size_streaming_two_steps_every_layer(cuda_ok):
    """The streaming workload's geometry (40 layers, d=2048, 256 experts in pinned host
    memory, 2 x 4 slots): two steps at batch 1 against the oracle on every layer, and the
    slot tags of every layer against the oracle's routing."""
    B, S, seed = 1, 2, 4
    st, store, log, _ = build_streaming(FULL, seed, B)
    gpu, logs = run_logged(st, FULL, seed, B, S, log)
    ref = oracle_steps(FULL, seed, B, S, gpu[2], gpu[3])
    compare_steps(FULL, gpu, ref)
    check_slot_sets_hold_the_oracle_routing(ref["idx"], logs)
    assert st.stats()["dropped"] == 0
    st.close()


def test_refused_staging_copy_is_reported(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    B, seed = 1, 81
    st, store, log, _ = build_streaming(SMALL, seed, B)
    h = bf16_tensor(synth.hidden(seed, 0, SMALL.L, B, SMALL.d), "cuda")
    st.debug_fail_staging_after(2)
    with pytest.raises(e0.E0Error) as ei:
        st.stack_decode(h, 0, streaming=True)
    assert ei.value.status == "STAGING"
    torch.cuda.synchronize()
    # a new sequence on the same context works again and matches the oracle
    gpu = run_steps(st, SMALL, seed, B, 1, streaming=True)
    ref = oracle_steps(SMALL, seed, B, 1, gpu[2], gpu[3])
    compare_steps(SMALL, gpu, ref)
    st.close()


def test_wrong_slot_tag_is_caught_by_the_kernels(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    B, seed = 1, 82
    st, store, log, _ = build_streaming(SMALL, seed, B)
    h = bf16_tensor(synth.hidden(seed, 0, SMALL.L, B, SMALL.d), "cuda")
    st.debug_set_slot_tag(1, 0, 15)      # next staging into pool set 1 mislabels slot 0
    st.stack_decode(h, 0, streaming=True)
    with pytest.raises(e0.E0Error) as ei:
        st.sync_status()
    assert ei.value.status == "SLOT_MISMATCH"
    st.close()


def test_explicit_stage_call_and_argument_checks(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    st, store, log, _ = build_streaming(SMALL, 83, 1)
    st.stage_experts(1, [3, 5, 7, 3, 9])
    torch.cuda.synchronize()
    assert st.stats()["staged_experts"] == 4          # duplicates collapse
    with pytest.raises(e0.E0Error):
        st.stage_experts(1, [99])
    with pytest.raises(e0.E0Error):
        st.stage_experts(1, list(range(9)))            # more experts than the 4 slots
    st.close()
