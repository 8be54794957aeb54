"""Streaming tier on the GPU: experts live in pinned host memory and are staged into an
HBM slot pool.  The staged set must equal the routed set (prediction-as-routing: nothing
dropped), the output must equal the resident path's bit for bit, and host-injected faults
(a refused copy, a wrong slot tag) must come back as errors."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from synth import Dims
from synth.device import bf16_tensor, layer_tensors, pinned_expert_store

pytestmark = pytest.mark.gpu

SMALL = Dims(d=256, E=16, I=128, k=4, r=8, L=5, head_layers=(0, 1, 2))


def build(seed, B, slots=None):
    import int4_expert_streaming_prerouter_b200 as e0
    lys, hds = zip(*[layer_tensors(seed, n, SMALL, "cuda", resident=True) for n in range(SMALL.L)])
    res = e0.Context(SMALL.d, SMALL.E, SMALL.I, SMALL.k, SMALL.r, SMALL.L, B)
    res.register_model(list(lys), list(hds))
    st = e0.Context(SMALL.d, SMALL.E, SMALL.I, SMALL.k, SMALL.r, SMALL.L, B)
    lys2 = [{k: v for k, v in ly.items() if k != "experts"} for ly in lys]
    st.register_model(lys2, list(hds))
    store = pinned_expert_store(seed, SMALL)
    st.stream_register(store, pool_layers=2, slots_per_layer=slots or min(SMALL.E, B * SMALL.k))
    return res, st, store


def test_streaming_equals_resident_and_stages_the_routed_sets(cuda_ok):
    B, S, seed = 3, 4, 80
    res, st, store = build(seed, B)
    routed, predicted_unique, reactive_unique = [], 0, 0
    for t in range(S):
        h = bf16_tensor(synth.hidden(seed, t, SMALL.L, B, SMALL.d), "cuda")
        y_r = res.stack_decode(h, t)
        y_s = st.stack_decode(h, t, streaming=True)
        st.sync_status()
        res.sync_status()
        assert torch.equal(y_r.view(torch.int16), y_s.view(torch.int16))
        idx_r, pred_r = res.get_routing(B)
        idx_s, pred_s = st.get_routing(B)
        assert np.array_equal(idx_r, idx_s) and np.array_equal(pred_r, pred_s)
        for n in range(SMALL.L):
            u = len(set(idx_s[n].reshape(-1).tolist()))
            if t > 0 and (n - 1) in SMALL.head_layers:
                predicted_unique += u
            else:
                reactive_unique += u
        routed.append(idx_s)
    stats = st.stats()
    assert stats["dropped"] == 0
    assert stats["prefetched_experts"] == predicted_unique
    assert stats["ondemand_experts"] == reactive_unique
    assert stats["staged_experts"] == predicted_unique + reactive_unique
    assert stats["staged_bytes"] == stats["staged_experts"] * synth.blob_bytes(SMALL.d, SMALL.I)
    assert stats["stage_ms"] > 0
    # the oracle's staging plan: staged set == routed set for every (step, layer)
    plan = O.staging_plan(np.stack(routed), SMALL)
    for (t, n), p in plan.items():
        assert set(p["experts"]) == set(routed[t][n].reshape(-1).tolist())
    res.close()
    st.close()


def test_refused_staging_copy_is_reported(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    B, seed = 1, 81
    res, st, store = build(seed, B)
    h = bf16_tensor(synth.hidden(seed, 0, SMALL.L, B, SMALL.d), "cuda")
    st.debug_fail_staging_after(2)
    with pytest.raises(e0.E0Error) as ei:
        st.stack_decode(h, 0, streaming=True)
    assert ei.value.status == "STAGING"
    torch.cuda.synchronize()
    # a new sequence on the same context works again
    y = st.stack_decode(h, 0, streaming=True)
    st.sync_status()
    assert torch.equal(y.view(torch.int16), res.stack_decode(h, 0).view(torch.int16))
    res.close()
    st.close()


def test_wrong_slot_tag_is_caught_by_the_kernels(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    B, seed = 1, 82
    res, st, store = build(seed, B)
    h = bf16_tensor(synth.hidden(seed, 0, SMALL.L, B, SMALL.d), "cuda")
    st.debug_set_slot_tag(1, 0, 15)      # next staging into pool set 1 mislabels slot 0
    st.stack_decode(h, 0, streaming=True)
    with pytest.raises(e0.E0Error) as ei:
        st.sync_status()
    assert ei.value.status == "SLOT_MISMATCH"
    res.close()
    st.close()


def test_explicit_stage_call_and_argument_checks(cuda_ok):
    import int4_expert_streaming_prerouter_b200 as e0
    res, st, store = build(83, 1)
    st.stage_experts(1, [3, 5, 7, 3, 9])
    torch.cuda.synchronize()
    assert st.stats()["staged_experts"] == 4          # duplicates collapse
    with pytest.raises(e0.E0Error):
        st.stage_experts(1, [99])
    with pytest.raises(e0.E0Error):
        st.stage_experts(1, list(range(9)))            # more experts than the 4 slots
    res.close()
    st.close()
