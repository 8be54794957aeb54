"""Python binding of ``libe0moe.so``: argument marshalling only.

Every step of the MoE block runs in the library's CUDA kernels; this module turns torch
tensors into device pointers and CUDA streams, calls the C ABI declared in
``include/e0moe.h`` and raises :class:`E0Error` on a non-zero status.  PyTorch is used
for device memory, pinned host memory and streams only.

There is no fallback: if the shared library is missing this module raises at import of
:func:`lib` time, and every call needs a CUDA device.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libe0moe.so")

E0_OK = 0
STATUS = {0: "OK", -1: "INVALID_ARG", -2: "CUDA", -3: "OOM", -4: "STAGING", -5: "SLOT_MISMATCH",
          -6: "TIMEOUT", -7: "DEVICE"}


class E0Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code
        self.status = STATUS.get(code, str(code))


class Dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("n_experts", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("top_k", ctypes.c_int), ("group", ctypes.c_int), ("lora_rank", ctypes.c_int),
                ("head_hidden", ctypes.c_int), ("head_onehot", ctypes.c_int),
                ("rms_eps", ctypes.c_float), ("lora_scale", ctypes.c_float)]


class Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("experts", "shared", "lora_Ag", "lora_Bg", "lora_Au", "lora_Bu", "lora_Ad", "lora_Bd",
                 "router_w", "norm_w")]


class Head(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_lin", "fc1_w", "fc1_b", "fc2_w", "fc2_b")]


class Stats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_uint64), ("staged_experts", ctypes.c_uint64),
                ("staged_bytes", ctypes.c_uint64), ("prefetched_experts", ctypes.c_uint64),
                ("ondemand_experts", ctypes.c_uint64), ("dropped", ctypes.c_uint64),
                ("stage_ms", ctypes.c_double), ("exposed_wait_ms", ctypes.c_double),
                ("kernel_launches", ctypes.c_uint64), ("gemm_timed", ctypes.c_uint64),
                ("gemm_ms", ctypes.c_double), ("hit_experts", ctypes.c_uint64)]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int

# name -> (restype, argtypes); one entry per function declared in include/e0moe.h
_SIGS = {
    "e0_create": (_I, [ctypes.POINTER(Dims), _I, _I, ctypes.POINTER(_P)]),
    "e0_destroy": (_I, [_P]),
    "e0_register_model": (_I, [_P, ctypes.POINTER(Layer), ctypes.POINTER(Head)]),
    "e0_moe_layer_forward": (_I, [_P, _I, _P, _I, _P, _P, _P, _P, _P, _P]),
    "e0_prerouter_predict": (_I, [_P, _I, _P, _I, _P, _P, _P, _P, _P]),
    "e0_stream_register": (_I, [_P, _P, ctypes.c_size_t, _I, _I]),
    "e0_stage_experts": (_I, [_P, _I, ctypes.POINTER(ctypes.c_int32), _I, _P]),
    "e0_moe_stack_decode": (_I, [_P, _P, _I, _I, _P, _P, _I, _I, _P]),
    "e0_moe_stack_decode_host": (_I, [_P, _P, _I, _I, _P, _P, _I, _I, _P]),
    "e0_host_io_wait": (_I, [_P, _P]),
    "e0_get_routing": (_I, [_P, _I, _P, _P]),
    "e0_moe_prefill_stack": (_I, [_P, _P, _I, _P, _P, _P, _P]),
    "e0_moe_prefill_stack_host": (_I, [_P, _P, _I, _P, _P, _P, _P]),
    "e0_get_stats": (_I, [_P, ctypes.POINTER(Stats)]),
    "e0_sync_status": (_I, [_P]),
    "e0_last_error": (ctypes.c_char_p, []),
    "e0_moe_layer_forward_noalloc": (_I, [ctypes.POINTER(Dims), ctypes.POINTER(Layer), _P, _I, _P, _P, _P, _P,
                                          _P, _P, _P]),
    "e0_stream_mode": (_I, [_P, _I]),
    "e0_debug_stream_log": (_I, [_P, _P]),
    "e0_debug_pool_slot": (_I, [_P, _I, _I, ctypes.POINTER(_P)]),
    "e0_debug_fail_staging_after": (_I, [_P, _I]),
    "e0_debug_set_slot_tag": (_I, [_P, _I, _I, _I]),
    "e0_debug_decode_stall": (_I, [_P, _I, ctypes.c_ulonglong]),
    "e0_debug_force_general": (_I, [_P, _I]),
    "e0_debug_decode_trace": (_I, [_P, _P]),
    "e0_debug_prefill_path": (_I, [_P, _I]),
    "e0_prefill_fixed_order": (_I, [_P, _I]),
    "e0_debug_decode_mode": (_I, [_P, _I]),
    "e0_debug_decode_flat": (_I, [_P, _I]),
    "e0_debug_time_gemm": (_I, [_P, _I]),
    "e0_debug_phase_timing": (_I, [_P, _I]),
    "e0_debug_phase_times": (_I, [_P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_ulonglong)]),
    "e0_decode_items": (_I, [ctypes.POINTER(Dims), _I, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint8),
                             _I, _I, _I, _I, ctypes.POINTER(ctypes.c_uint64), _I, ctypes.POINTER(_I)]),
}


def lib():
    """Load ``libe0moe.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m int4_expert_streaming_prerouter_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != E0_OK:
        raise E0Error(rc, lib().e0_last_error().decode(errors="replace"))


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_dims(d, E, I, k, r, head_hidden=0, head_onehot=0, eps=1e-6, lora_scale=1.0) -> Dims:
    return Dims(d, E, I, k, 64, r, head_hidden, head_onehot, eps, lora_scale)


def decode_items(dims: Dims, n_layers: int, has_head, has_lora, n_ctas: int, flat: bool, step0: bool, cta: int):
    """The one-launch decode kernel's work-item list of CTA `cta` (host only; see the C
    header): a list of (kind, first, layer, first_unit, n_units) with kind 0 router rows,
    1 top-k, 2 x rows, 3 gate/up units, 4 down rows."""
    cap = 512
    out = (ctypes.c_uint64 * cap)()
    n = ctypes.c_int(0)
    hh = (ctypes.c_uint8 * n_layers)(*[1 if v else 0 for v in has_head])
    hl = (ctypes.c_uint8 * n_layers)(*[1 if v else 0 for v in has_lora])
    _check(lib().e0_decode_items(ctypes.byref(dims), n_layers, hh, hl, n_ctas, int(flat), int(step0), cta, out, cap,
                                 ctypes.byref(n)))
    return [(w & 15, (w >> 4) & 1, (w >> 8) & 255, (w >> 16) & 0xFFFFFF, w >> 40) for w in out[:n.value]]


def moe_layer_forward_noalloc(dims: Dims, layer: dict, h, route_idx=None, y=None, y_f32=None, idx=None,
                              gates=None, dev_status=None, stream=None):
    """One MoE block without any device allocation by the library (see the C header).
    `layer` is a dict of torch tensors as for Context.register_model."""
    import torch
    L = Layer()
    for f, _ in Layer._fields_:
        setattr(L, f, _ptr(layer.get(f)))
    T = h.shape[0]
    if y is None:
        y = torch.empty((T, dims.d_model), dtype=torch.bfloat16, device=h.device)
    _check(lib().e0_moe_layer_forward_noalloc(ctypes.byref(dims), ctypes.byref(L), _ptr(h), T, _ptr(route_idx),
                                              _ptr(y), _ptr(y_f32), _ptr(idx), _ptr(gates), _ptr(dev_status),
                                              _stream(stream)))
    return y


class Context:
    """One ``e0_ctx``: workspaces, routing tables and (optionally) the streaming pool."""

    def __init__(self, d, E, I, k, r, n_layers, max_tokens, head_hidden=0, head_onehot=0,
                 eps=1e-6, lora_scale=1.0):
        self.dims = make_dims(d, E, I, k, r, head_hidden, head_onehot, eps, lora_scale)
        self.n_layers, self.max_tokens = n_layers, max_tokens
        self._keep = []
        h = _P()
        _check(lib().e0_create(ctypes.byref(self.dims), n_layers, max_tokens, ctypes.byref(h)))
        self._h = h

    # -- lifetime ---------------------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            lib().e0_destroy(self._h)
            self._h = None
            self._keep = []

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- weights ----------------------------------------------------------------------
    def register_model(self, layers: list, heads: Optional[list] = None):
        """layers[l]: dict with torch tensors experts [E, blob] (or None), shared [blob],
        router_w [E, d], norm_w [d], and optionally lora_Ag..lora_Bd.  heads[l]: dict with
        w_lin (and fc1_w, fc1_b, fc2_w, fc2_b) or None."""
        L = (Layer * self.n_layers)()
        H = (Head * self.n_layers)()
        for i, ly in enumerate(layers):
            for f, _ in Layer._fields_:
                t = ly.get(f)
                setattr(L[i], f, _ptr(t))
                self._keep.append(t)
            hd = heads[i] if heads is not None else None
            for f, _ in Head._fields_:
                t = hd.get(f) if hd else None
                setattr(H[i], f, _ptr(t))
                self._keep.append(t)
        _check(lib().e0_register_model(self._h, L, H))

    # -- one MoE block ------------------------------------------------------------------
    def moe_layer_forward(self, layer, h, route_idx=None, y=None, y_f32=None, idx=None, gates=None,
                          stream=None):
        import torch
        T = h.shape[0]
        d, k = self.dims.d_model, self.dims.top_k
        if y is None:
            y = torch.empty((T, d), dtype=torch.bfloat16, device=h.device)
        _check(lib().e0_moe_layer_forward(self._h, layer, _ptr(h), T, _ptr(route_idx), _ptr(y), _ptr(y_f32),
                                          _ptr(idx), _ptr(gates), _stream(stream)))
        return y

    def prerouter_predict(self, layer, x, cur=None, prev=None, pred=None, logits=None, stream=None):
        import torch
        T = x.shape[0]
        if pred is None:
            pred = torch.empty((T, self.dims.top_k), dtype=torch.int32, device=x.device)
        _check(lib().e0_prerouter_predict(self._h, layer, _ptr(x), T, _ptr(cur), _ptr(prev), _ptr(pred),
                                          _ptr(logits), _stream(stream)))
        return pred

    # -- streaming tier ------------------------------------------------------------------
    def stream_register(self, host_blob, pool_layers=2, slots_per_layer=None):
        if slots_per_layer is None:
            slots_per_layer = self.dims.top_k
        if not host_blob.is_pinned():
            raise ValueError("the host expert store must be pinned memory")
        self._keep.append(host_blob)
        blob = host_blob.shape[-1]
        _check(lib().e0_stream_register(self._h, _ptr(host_blob), blob, pool_layers, slots_per_layer))

    def stream_mode(self, reactive: bool):
        """False: prerouter prefetch (default); True: every layer routes itself and stages
        on demand (no prediction).  Starts a new sequence."""
        _check(lib().e0_stream_mode(self._h, int(reactive)))

    def debug_stream_log(self, log):
        """log: int32 CUDA tensor [L, slots_per_layer] or None."""
        self._keep.append(log)
        _check(lib().e0_debug_stream_log(self._h, _ptr(log)))

    def debug_pool_slot(self, pool_set, slot) -> int:
        out = _P()
        _check(lib().e0_debug_pool_slot(self._h, pool_set, slot, ctypes.byref(out)))
        return int(out.value)

    def stage_experts(self, layer, experts, stream=None):
        arr = (ctypes.c_int32 * len(experts))(*[int(e) for e in experts])
        _check(lib().e0_stage_experts(self._h, layer, arr, len(experts), _stream(stream)))

    # -- decode over the stack ------------------------------------------------------------
    def stack_decode(self, h_in, step, y_out=None, y_f32=None, streaming=False, chained=False, stream=None):
        import torch
        L, B, d = h_in.shape
        if y_out is None:
            y_out = torch.empty((L, B, d), dtype=torch.bfloat16, device=h_in.device)
        _check(lib().e0_moe_stack_decode(self._h, _ptr(h_in), B, step, _ptr(y_out), _ptr(y_f32),
                                         int(streaming), int(chained), _stream(stream)))
        return y_out

    def stack_decode_host(self, h_host, step, y_host, y_f32_host=None, streaming=False, chained=False, stream=None):
        """One decode step with host (pinned) tensors; the library overlaps the copies with
        the kernels.  The outputs are complete after host_io_wait(stream) and a
        synchronisation of the stream."""
        L, B, d = h_host.shape
        assert not h_host.is_cuda and not y_host.is_cuda and (y_f32_host is None or not y_f32_host.is_cuda)
        _check(lib().e0_moe_stack_decode_host(self._h, _ptr(h_host), B, step, _ptr(y_host), _ptr(y_f32_host),
                                              int(streaming), int(chained), _stream(stream)))
        return y_host

    def host_io_wait(self, stream=None):
        _check(lib().e0_host_io_wait(self._h, _stream(stream)))

    def prefill_stack_host(self, h_host, y_host, y_f32_host=None, idx=None, stream=None):
        """prefill_stack with pinned host tensors h_host, y_host [L, T, d] bf16 (y_f32_host
        [L, T, d] fp32 or None; idx a CUDA int32 tensor [L, T, k] or None).  The library
        overlaps each layer's copies with the neighbouring layers' kernels; the outputs are
        complete after host_io_wait(stream) and a synchronisation of the stream."""
        L, T, d = h_host.shape
        assert not h_host.is_cuda and not y_host.is_cuda and (y_f32_host is None or not y_f32_host.is_cuda)
        _check(lib().e0_moe_prefill_stack_host(self._h, _ptr(h_host), T, _ptr(y_host), _ptr(y_f32_host), _ptr(idx),
                                               _stream(stream)))
        return y_host

    def prefill_stack(self, h_in, y_out=None, y_f32=None, idx=None, stream=None):
        """h_in [L, T, d] bf16 -> y_out [L, T, d] bf16 (prediction-as-routing, one token ahead)."""
        import torch
        L, T, d = h_in.shape
        if y_out is None:
            y_out = torch.empty((L, T, d), dtype=torch.bfloat16, device=h_in.device)
        _check(lib().e0_moe_prefill_stack(self._h, _ptr(h_in), T, _ptr(y_out), _ptr(y_f32), _ptr(idx),
                                          _stream(stream)))
        return y_out

    def get_routing(self, B):
        import numpy as np
        k = self.dims.top_k
        idx = np.zeros((self.n_layers, B, k), dtype=np.int32)
        pred = np.zeros((self.n_layers, B, k), dtype=np.int32)
        _check(lib().e0_get_routing(self._h, B, idx.ctypes.data, pred.ctypes.data))
        return idx, pred

    def stats(self) -> dict:
        s = Stats()
        _check(lib().e0_get_stats(self._h, ctypes.byref(s)))
        return {f: getattr(s, f) for f, _ in Stats._fields_}

    def sync_status(self):
        _check(lib().e0_sync_status(self._h))

    # -- host-side fault injection (tests) ------------------------------------------------
    def debug_fail_staging_after(self, n):
        _check(lib().e0_debug_fail_staging_after(self._h, n))

    def debug_set_slot_tag(self, pool_set, slot, expert):
        _check(lib().e0_debug_set_slot_tag(self._h, pool_set, slot, expert))

    def debug_decode_stall(self, cta, timeout_ns):
        _check(lib().e0_debug_decode_stall(self._h, cta, timeout_ns))

    def debug_decode_trace(self, buf):
        """buf: int64 CUDA tensor [grid, L, 16] or None; returns the grid size."""
        return lib().e0_debug_decode_trace(self._h, _ptr(buf))

    def debug_decode_mode(self, mode: int):
        _check(lib().e0_debug_decode_mode(self._h, mode))

    def debug_phase_timing(self, on: bool):
        _check(lib().e0_debug_phase_timing(self._h, int(on)))

    def debug_phase_times(self):
        """(per-kernel summed ms of the phased decode kernels [norm, rows, route, gate/up,
        sums+t_d, down], steps timed)."""
        ms = (ctypes.c_double * 6)()
        n = ctypes.c_ulonglong(0)
        _check(lib().e0_debug_phase_times(self._h, ms, ctypes.byref(n)))
        return list(ms), int(n.value)

    def debug_time_gemm(self, on: bool):
        _check(lib().e0_debug_time_gemm(self._h, int(on)))

    def debug_decode_flat(self, on: bool):
        _check(lib().e0_debug_decode_flat(self._h, int(on)))

    def debug_prefill_path(self, mode: int):
        _check(lib().e0_debug_prefill_path(self._h, mode))

    def prefill_fixed_order(self, on: bool):
        """Tensor-core prefill combine in slot order (bit-reproducible y) instead of
        completion-order reductions."""
        _check(lib().e0_prefill_fixed_order(self._h, int(on)))

    def debug_force_general(self, on: bool):
        _check(lib().e0_debug_force_general(self._h, int(on)))
