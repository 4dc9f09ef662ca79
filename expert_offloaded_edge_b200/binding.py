"""ctypes binding of libftm.so (see include/ftm.h for the contract)."""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(PKG, "libftm.so")

FTM_OK, FTM_ERR_INVALID_ARG, FTM_ERR_UNSUPPORTED, FTM_ERR_CAPACITY, FTM_ERR_CUDA = range(5)
FTM_F32, FTM_BF16, FTM_FP8_E4M3_B128, FTM_NVFP4, FTM_MXFP4 = range(5)
(FTM_K_ROUTE, FTM_K_PERMUTE, FTM_K_LRU, FTM_K_GATHER, FTM_K_GEMM1, FTM_K_GEMM2, FTM_K_COMBINE) = range(7)
KERNEL_NAMES = ("route", "permute", "lru", "gather", "gemm1", "gemm2", "combine")
_WDTYPE = {"f32": FTM_F32, "bf16": FTM_BF16, "fp8": FTM_FP8_E4M3_B128, "nvfp4": FTM_NVFP4, "mxfp4": FTM_MXFP4}

c_i32, c_i64, c_u64, c_p, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_size_t


class LayerDesc(ctypes.Structure):
    _fields_ = [("d", c_i32), ("E", c_i32), ("k", c_i32), ("I", c_i32), ("has_shared", c_i32), ("S", c_i32),
                ("wdtype", c_i32), ("reserved", c_i32)]


class BankLayout(ctypes.Structure):
    _fields_ = [("bank_bytes", c_u64), ("w_gu_off", c_u64), ("w_gu_bytes", c_u64), ("w_d_off", c_u64),
                ("w_d_bytes", c_u64), ("s_gu_off", c_u64), ("s_gu_bytes", c_u64), ("s_d_off", c_u64),
                ("s_d_bytes", c_u64), ("s_t_off", c_u64), ("s_t_bytes", c_u64)]


class SlotCache(ctypes.Structure):
    _fields_ = [("slot_of_expert", c_p), ("expert_of_slot", c_p), ("last_use", c_p), ("step", c_i64),
                ("slot_pool", c_p), ("host_pool", c_p), ("host_scratch", c_p), ("last_distinct", c_i32),
                ("last_hits", c_i32), ("last_misses", c_i32), ("fail_before_copy", c_i32), ("n_keys", c_i32),
                ("key_base", c_i32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("w_router", c_p), ("router_bias", c_p), ("slot_pool", c_p), ("slot_of_expert", c_p),
                ("shared_bank", c_p), ("act_scale", c_p)]


class Hybrid(ctypes.Structure):
    """ftm_hybrid: the bandwidth-adaptive miss split's parameters, host buffer and results."""
    _fields_ = [("pcie_gbs", ctypes.c_double), ("host_gbs", ctypes.c_double), ("threads", c_i32),
                ("last_misses", c_i32), ("last_host", c_i32), ("last_host_rows", c_i32),
                ("last_host_ms", ctypes.c_double), ("host_ws", c_p), ("host_ws_bytes", c_sz)]


class FtmError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"ftm status {status}: {msg}")
        self.status = status


_lib = None


def library() -> ctypes.CDLL:
    """Load libftm.so; fails loudly when the CUDA library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} is missing: build it with `python -m expert_offloaded_edge_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(SO)
        P = ctypes.POINTER
        L.ftm_last_error.restype = ctypes.c_char_p
        L.ftm_device_status.argtypes = [c_i32]
        L.ftm_device_status.restype = c_i32
        L.ftm_get_bank_layout.argtypes = [P(LayerDesc), P(BankLayout)]
        L.ftm_route.argtypes = [P(LayerDesc), c_p, c_i32, c_p, c_p, c_p, c_p, c_p]
        L.ftm_permute.argtypes = [P(LayerDesc), c_p, c_i32, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]
        L.ftm_permute_workspace_bytes.argtypes = [P(LayerDesc), c_i32]
        L.ftm_permute_workspace_bytes.restype = c_sz
        L.ftm_slot_host_scratch_ints.argtypes = [P(LayerDesc)]
        L.ftm_slot_host_scratch_ints.restype = c_sz
        L.ftm_slot_workspace_bytes.argtypes = [P(LayerDesc)]
        L.ftm_slot_workspace_bytes.restype = c_sz
        L.ftm_slot_lookup_update.argtypes = [P(LayerDesc), P(SlotCache), c_p, c_i32, c_p, c_sz, c_p, c_p]
        L.ftm_slot_resize.argtypes = [P(LayerDesc), P(SlotCache), c_i32, P(SlotCache), c_p, c_sz, c_p]
        L.ftm_slot_stage_layer.argtypes = [P(LayerDesc), P(SlotCache), c_i32, c_i32, c_p, c_p, c_sz, c_p, c_p]
        L.ftm_moe_layers_forward.argtypes = [P(LayerDesc), c_i32, P(LayerWeights), P(SlotCache), P(c_p), c_i32,
                                             P(c_p), c_i32, P(c_i32), c_p, c_sz, c_p, c_p]
        L.ftm_last_warning.restype = ctypes.c_char_p
        L.ftm_expert_ffn.argtypes = [P(LayerDesc), c_p, c_i32, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]
        L.ftm_ffn_workspace_bytes.argtypes = [P(LayerDesc), c_i32]
        L.ftm_ffn_workspace_bytes.restype = c_sz
        L.ftm_combine.argtypes = [P(LayerDesc), c_p, c_p, c_p, c_i32, c_p, c_p]
        L.ftm_moe_layer_forward.argtypes = [P(LayerDesc), P(LayerWeights), P(SlotCache), c_p, c_i32, c_p, c_p, c_sz,
                                            c_p, c_p]
        L.ftm_moe_layer_forward_noalloc.argtypes = [P(LayerDesc), P(LayerWeights), c_p, c_i32, c_p, c_p]
        L.ftm_moe_layer_forward_noalloc.restype = c_i32
        L.ftm_set_profile_events.argtypes = [c_i32, c_p, c_p]
        L.ftm_set_profile_events.restype = c_i32
        L.ftm_kernel_launches.argtypes = []
        L.ftm_kernel_launches.restype = c_u64
        L.ftm_selftest_bounded_wait.argtypes = [P(c_i32), c_p]
        L.ftm_workspace_bytes.argtypes = [P(LayerDesc), c_i32]
        L.ftm_workspace_bytes.restype = c_sz
        L.ftm_hybrid_split.argtypes = [c_i32, ctypes.c_double, ctypes.c_double]
        L.ftm_hybrid_split.restype = c_i32
        for name in ("ftm_hybrid_workspace_bytes", "ftm_hybrid_host_bytes", "ftm_host_ffn_scratch_bytes"):
            getattr(L, name).argtypes = [P(LayerDesc), c_i32]
            getattr(L, name).restype = c_sz
        L.ftm_host_expert_ffn.argtypes = [P(LayerDesc), c_p, c_p, c_i32, c_p, c_p, c_p, c_sz, c_i32]
        L.ftm_moe_layer_forward_hybrid.argtypes = [P(LayerDesc), P(LayerWeights), P(SlotCache), P(Hybrid), c_p,
                                                   c_i32, c_p, c_p, c_sz, c_p, c_p]
        for name in ("ftm_get_bank_layout", "ftm_route", "ftm_permute", "ftm_slot_lookup_update", "ftm_slot_resize",
                     "ftm_slot_stage_layer", "ftm_expert_ffn", "ftm_combine", "ftm_moe_layer_forward",
                     "ftm_moe_layers_forward", "ftm_host_expert_ffn", "ftm_moe_layer_forward_hybrid"):
            getattr(L, name).restype = c_i32
        _lib = L
    return _lib


def desc_for(cfg) -> LayerDesc:
    """LayerDesc of a synthetic layer configuration (fields d, E, k, I, has_shared, S, wdtype)."""
    return LayerDesc(cfg.d, cfg.E, cfg.k, cfg.I, int(cfg.has_shared), cfg.S, _WDTYPE[cfg.wdtype], 0)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data   # numpy array (host)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != FTM_OK:
        raise FtmError(status, library().ftm_last_error().decode())


def ftm_last_error() -> str:
    return library().ftm_last_error().decode()


def ftm_device_status(reset: bool = True) -> int:
    return library().ftm_device_status(1 if reset else 0)


def ftm_get_bank_layout(desc: LayerDesc) -> BankLayout:
    out = BankLayout()
    _check(library().ftm_get_bank_layout(ctypes.byref(desc), ctypes.byref(out)))
    return out


def ftm_route(desc, x, T, w_router, bias, topk_ids, topk_w, stream=None):
    _check(library().ftm_route(ctypes.byref(desc), _ptr(x), T, _ptr(w_router), _ptr(bias), _ptr(topk_ids),
                               _ptr(topk_w), _stream(stream)))


def ftm_permute_workspace_bytes(desc, T) -> int:
    return int(library().ftm_permute_workspace_bytes(ctypes.byref(desc), T))


def ftm_permute(desc, topk_ids, T, counts, offsets, perm, inv, workspace, ws_bytes, stream=None):
    _check(library().ftm_permute(ctypes.byref(desc), _ptr(topk_ids), T, _ptr(counts), _ptr(offsets), _ptr(perm),
                                 _ptr(inv), _ptr(workspace), ws_bytes, _stream(stream)))


def ftm_slot_host_scratch_ints(desc) -> int:
    return int(library().ftm_slot_host_scratch_ints(ctypes.byref(desc)))


def ftm_slot_workspace_bytes(desc) -> int:
    return int(library().ftm_slot_workspace_bytes(ctypes.byref(desc)))


def ftm_slot_lookup_update(desc, cache: SlotCache, topk_ids, T, workspace, ws_bytes, compute_stream=None,
                           copy_stream=None):
    _check(library().ftm_slot_lookup_update(ctypes.byref(desc), ctypes.byref(cache), _ptr(topk_ids), T,
                                            _ptr(workspace), ws_bytes, _stream(compute_stream),
                                            _stream(copy_stream)))


def ftm_slot_resize(desc, cache: SlotCache, S_new: int, new_cache: SlotCache, workspace, ws_bytes, stream=None):
    _check(library().ftm_slot_resize(ctypes.byref(desc), ctypes.byref(cache), S_new, ctypes.byref(new_cache),
                                     _ptr(workspace), ws_bytes, _stream(stream)))


def ftm_slot_stage_layer(desc, cache: SlotCache, layer: int, hold_previous: bool, after_event, workspace, ws_bytes,
                         copy_stream=None, ready_event=None):
    """after_event / ready_event: torch.cuda.Event (or None)."""
    _check(library().ftm_slot_stage_layer(ctypes.byref(desc), ctypes.byref(cache), layer, 1 if hold_previous else 0,
                                          None if after_event is None else after_event.cuda_event, _ptr(workspace),
                                          ws_bytes, _stream(copy_stream),
                                          None if ready_event is None else ready_event.cuda_event))


def ftm_moe_layers_forward(desc, weights, cache: SlotCache, xs, T, outs, overlap: bool, workspace, ws_bytes,
                           stream=None, copy_stream=None) -> bool:
    """weights: sequence of LayerWeights; xs / outs: sequences of device tensors.
    Returns whether the copy/compute overlap ran."""
    n = len(weights)
    W = (LayerWeights * n)(*weights)
    X = (c_p * n)(*[_ptr(t) for t in xs])
    O = (c_p * n)(*[_ptr(t) for t in outs])
    used = c_i32(0)
    _check(library().ftm_moe_layers_forward(ctypes.byref(desc), n, W, ctypes.byref(cache), X, T, O,
                                            1 if overlap else 0, ctypes.byref(used), _ptr(workspace), ws_bytes,
                                            _stream(stream), _stream(copy_stream)))
    return bool(used.value)


def ftm_last_warning() -> str:
    return library().ftm_last_warning().decode()


def ftm_ffn_workspace_bytes(desc, T) -> int:
    return int(library().ftm_ffn_workspace_bytes(ctypes.byref(desc), T))


def ftm_expert_ffn(desc, x, T, offsets, perm, slot_of_expert, slot_pool, shared_bank, y, workspace, ws_bytes,
                   stream=None, act_scale=None):
    """act_scale: device fp32[2] (NVFP4 activation global scales of x and h) or None."""
    _check(library().ftm_expert_ffn(ctypes.byref(desc), _ptr(x), T, _ptr(offsets), _ptr(perm), _ptr(slot_of_expert),
                                    _ptr(slot_pool), _ptr(shared_bank), _ptr(act_scale), _ptr(y), _ptr(workspace),
                                    ws_bytes, _stream(stream)))


def ftm_combine(desc, y, inv, topk_w, T, out, stream=None):
    _check(library().ftm_combine(ctypes.byref(desc), _ptr(y), _ptr(inv), _ptr(topk_w), T, _ptr(out),
                                 _stream(stream)))


def ftm_set_profile_events(which: int, start_event=None, stop_event=None):
    """start/stop: torch.cuda.Event(enable_timing=True) (or None to clear)."""
    sp = None if start_event is None else start_event.cuda_event
    ep = None if stop_event is None else stop_event.cuda_event
    _check(library().ftm_set_profile_events(which, sp, ep))


def ftm_kernel_launches() -> int:
    return int(library().ftm_kernel_launches())


def ftm_selftest_bounded_wait(stream=None) -> int:
    """Run the bounded-wait self-test kernel; returns the device status it left (1 = the wait gave up)."""
    v = ctypes.c_int32(-1)
    _check(library().ftm_selftest_bounded_wait(ctypes.byref(v), _stream(stream)))
    return int(v.value)


def ftm_workspace_bytes(desc, T_max) -> int:
    return int(library().ftm_workspace_bytes(ctypes.byref(desc), T_max))


def ftm_moe_layer_forward(desc, weights: LayerWeights, cache: Optional[SlotCache], x, T, out, workspace, ws_bytes,
                          stream=None, copy_stream=None):
    _check(library().ftm_moe_layer_forward(ctypes.byref(desc), ctypes.byref(weights),
                                           ctypes.byref(cache) if cache is not None else None, _ptr(x), T, _ptr(out),
                                           _ptr(workspace), ws_bytes, _stream(stream),
                                           _stream(copy_stream) if cache is not None else None))


def ftm_moe_layer_forward_noalloc(desc, weights: LayerWeights, x, T, out, stream=None):
    """Resident layer forward whose scratch is the library's static device array
    (for callers that cannot allocate device memory; see include/ftm.h)."""
    _check(library().ftm_moe_layer_forward_noalloc(ctypes.byref(desc), ctypes.byref(weights), _ptr(x), T, _ptr(out),
                                                   _stream(stream)))


def ftm_hybrid_split(m: int, pcie_gbs: float, host_gbs: float) -> int:
    """q of the bandwidth-adaptive miss split (-1 on invalid arguments)."""
    return int(library().ftm_hybrid_split(m, pcie_gbs, host_gbs))


def ftm_hybrid_workspace_bytes(desc, T_max) -> int:
    return int(library().ftm_hybrid_workspace_bytes(ctypes.byref(desc), T_max))


def ftm_hybrid_host_bytes(desc, T_max) -> int:
    return int(library().ftm_hybrid_host_bytes(ctypes.byref(desc), T_max))


def ftm_host_ffn_scratch_bytes(desc, n) -> int:
    return int(library().ftm_host_ffn_scratch_bytes(ctypes.byref(desc), n))


def ftm_host_expert_ffn(desc, bank, x, n, y, scratch, scratch_bytes, threads: int = 0, act_scale=None):
    """One expert's FFN on the host (host buffers: numpy arrays, CPU tensors or addresses;
    act_scale: host fp32[2] NVFP4 activation global scales or None)."""
    _check(library().ftm_host_expert_ffn(ctypes.byref(desc), _ptr(bank), _ptr(x), n, _ptr(y), _ptr(act_scale),
                                         _ptr(scratch), scratch_bytes, threads))


def ftm_moe_layer_forward_hybrid(desc, weights: LayerWeights, cache: SlotCache, hybrid: Hybrid, x, T, out, workspace,
                                 ws_bytes, stream=None, copy_stream=None):
    _check(library().ftm_moe_layer_forward_hybrid(ctypes.byref(desc), ctypes.byref(weights), ctypes.byref(cache),
                                                  ctypes.byref(hybrid), _ptr(x), T, _ptr(out), _ptr(workspace),
                                                  ws_bytes, _stream(stream), _stream(copy_stream)))
