"""ORACLE -- test infrastructure only.

Python handle on the plain C oracle in ``ftm_oracle.c``: a slow, obviously
correct CPU restatement of one routed-MoE layer (router, top-k gating,
permutation, LRU slot step, SwiGLU experts, combine).  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the product library never does and shares no code with it.

This module only marshals arrays and orders the oracle's own steps; every
arithmetic step runs in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "ftm_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src, "-lm"])
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        p, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.orc_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_dequant_bf16.argtypes = [p, i64, p]
        L.orc_dequant_fp8_b128.argtypes = [p, p, i32, i32, p]
        L.orc_dequant_nvfp4.argtypes = [p, p, ctypes.c_float, i32, i32, p]
        L.orc_qa_fp8_g128.argtypes = [p, i32, i32]
        L.orc_qa_nvfp4_g16.argtypes = [p, i32, i32]
        L.orc_qa_nvfp4_g16_gs.argtypes = [p, i32, i32, ctypes.c_float]
        L.orc_expert_ffn_gs.argtypes = [p, i32, i32, i32, p, p, p, i32, ctypes.c_float, ctypes.c_float, p]
        L.orc_e8m0_value.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_value.restype = ctypes.c_double
        L.orc_mx_scale_code.argtypes = [p, i32]
        L.orc_mx_scale_code.restype = ctypes.c_uint8
        L.orc_quant_mxfp4.argtypes = [p, i32, i32, p, p]
        L.orc_dequant_mxfp4.argtypes = [p, p, i32, i32, p]
        L.orc_qa_mxfp4_g32.argtypes = [p, i32, i32]
        L.orc_router_logits.argtypes = [p, i32, i32, p, p, i32, p]
        L.orc_margin_ok.argtypes = [p, i32, i32, i32, ctypes.c_double, p]
        L.orc_topk_gates.argtypes = [p, i32, i32, i32, p, p]
        L.orc_permute.argtypes = [p, i32, i32, i32, p, p, p, p]
        L.orc_lru_step.argtypes = [i32, i32, p, p, p, i64, p, i32, p, p, p, p, p]
        L.orc_lru_step.restype = i32
        L.orc_lru_step_reserve.argtypes = [i32, i32, p, p, p, i64, i64, p, i32, p, p, p, p, p]
        L.orc_lru_step_reserve.restype = i32
        L.orc_hybrid_split.argtypes = [i32, p, p, ctypes.c_double, ctypes.c_double, p, p, p]
        L.orc_hybrid_split.restype = i32
        L.orc_lru_resize.argtypes = [i32, i32, p, p, p, i32, p, p, p, p]
        L.orc_lru_resize.restype = i32
        L.orc_expert_ffn.argtypes = [p, i32, i32, i32, p, p, p, i32, p]
        L.orc_combine.argtypes = [p, p, i32, i32, i32, p, p]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def threads() -> int:
    return int(lib().orc_threads())


def set_threads(n: int) -> None:
    """OpenMP threads for the oracle calls of the calling thread."""
    lib().orc_set_threads(int(n))


# ---- formats -----------------------------------------------------------------

def e4m3_value(q: int) -> float:
    return float(lib().orc_e4m3_value(q))


def e2m1_value(nib: int) -> float:
    return float(lib().orc_e2m1_value(nib))


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(v))


def e2m1_encode(v: float) -> int:
    return int(lib().orc_e2m1_encode(v))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float32)
    lib().orc_dequant_bf16(_p(bits), bits.size, _p(out))
    return out


def dequant_fp8_b128(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = _f32(s)
    R, C = q.shape
    out = np.empty((R, C), dtype=np.float32)
    lib().orc_dequant_fp8_b128(_p(q), _p(s), R, C, _p(out))
    return out


def dequant_nvfp4(qp: np.ndarray, s16: np.ndarray, s_t: float) -> np.ndarray:
    qp = np.ascontiguousarray(qp, dtype=np.uint8)
    s16 = np.ascontiguousarray(s16, dtype=np.uint8)
    R, C = qp.shape[0], qp.shape[1] * 2
    out = np.empty((R, C), dtype=np.float32)
    lib().orc_dequant_nvfp4(_p(qp), _p(s16), ctypes.c_float(s_t), R, C, _p(out))
    return out


def qa_fp8(v: np.ndarray) -> np.ndarray:
    v = _f32(v).copy()
    rows, K = v.reshape(-1, v.shape[-1]).shape
    lib().orc_qa_fp8_g128(_p(v), rows, K)
    return v


def qa_nvfp4(v: np.ndarray, gs: Optional[float] = None) -> np.ndarray:
    """gs: the per-tensor global scale (None: the scale-1 quantiser)."""
    v = _f32(v).copy()
    rows, K = v.reshape(-1, v.shape[-1]).shape
    if gs is None:
        lib().orc_qa_nvfp4_g16(_p(v), rows, K)
    else:
        lib().orc_qa_nvfp4_g16_gs(_p(v), rows, K, ctypes.c_float(gs))
    return v


def e8m0_value(c: int) -> float:
    return float(lib().orc_e8m0_value(c))


def mx_scale_code(v: np.ndarray) -> int:
    v = _f32(v).ravel().copy()
    return int(lib().orc_mx_scale_code(_p(v), v.size))


def quant_mxfp4(w: np.ndarray):
    """w [R][C] (C a multiple of 32) -> (packed e2m1 [R][C/2], E8M0 scale codes [R][C/32])."""
    w = _f32(w)
    R, C = w.shape
    q = np.empty((R, C // 2), dtype=np.uint8)
    s = np.empty((R, C // 32), dtype=np.uint8)
    lib().orc_quant_mxfp4(_p(w), R, C, _p(q), _p(s))
    return q, s


def dequant_mxfp4(qp: np.ndarray, s: np.ndarray) -> np.ndarray:
    qp = np.ascontiguousarray(qp, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.uint8)
    R, C = qp.shape[0], qp.shape[1] * 2
    out = np.empty((R, C), dtype=np.float32)
    lib().orc_dequant_mxfp4(_p(qp), _p(s), R, C, _p(out))
    return out


def qa_mxfp4(v: np.ndarray) -> np.ndarray:
    v = _f32(v).copy()
    rows, K = v.reshape(-1, v.shape[-1]).shape
    lib().orc_qa_mxfp4_g32(_p(v), rows, K)
    return v


# ---- router / gating ----------------------------------------------------------

def router_logits(x: np.ndarray, Wr: np.ndarray, b: Optional[np.ndarray]) -> np.ndarray:
    x, Wr = _f32(x), _f32(Wr)
    T, d = x.shape
    E = Wr.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    lib().orc_router_logits(_p(x), T, d, _p(Wr), _p(None if b is None else _f32(b)), E, _p(out))
    return out


def margin_ok(logits: np.ndarray, k: int, margin: float = 1e-3) -> np.ndarray:
    logits = _f32(logits)
    T, E = logits.shape
    ok = np.zeros(T, dtype=np.uint8)
    lib().orc_margin_ok(_p(logits), T, E, k, margin, _p(ok))
    return ok.astype(bool)


def topk_gates(logits: np.ndarray, k: int) -> Tuple[np.ndarray, np.ndarray]:
    logits = _f32(logits)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    g = np.empty((T, k), dtype=np.float32)
    lib().orc_topk_gates(_p(logits), T, E, k, _p(ids), _p(g))
    return ids, g


def route(x, Wr, b, k):
    lg = router_logits(x, Wr, b)
    ids, g = topk_gates(lg, k)
    return ids, g, lg


# ---- permutation ---------------------------------------------------------------

def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    P = T * k
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(P, dtype=np.int32)
    inv = np.empty(P, dtype=np.int32)
    lib().orc_permute(_p(ids), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm, inv


# ---- LRU slot cache --------------------------------------------------------------

class LRUState:
    def __init__(self, E: int, S: int):
        self.E, self.S = E, S
        self.slot_of_expert = np.full(E, -1, dtype=np.int32)
        self.expert_of_slot = np.full(S, -1, dtype=np.int32)
        self.last_use = np.full(S, -1, dtype=np.int64)
        self.step = 0

    def copy(self) -> "LRUState":
        c = LRUState(self.E, self.S)
        c.slot_of_expert[:] = self.slot_of_expert
        c.expert_of_slot[:] = self.expert_of_slot
        c.last_use[:] = self.last_use
        c.step = self.step
        return c

    def update(self, ids: np.ndarray):
        """One step.  Returns (status, misses [(expert, slot)], distinct, hits)."""
        ids = np.ascontiguousarray(ids, dtype=np.int32).ravel()
        me = np.empty(self.E, dtype=np.int32)
        ms = np.empty(self.E, dtype=np.int32)
        nd, nh, nm = (np.zeros(1, dtype=np.int32) for _ in range(3))
        rc = lib().orc_lru_step(self.E, self.S, _p(self.slot_of_expert), _p(self.expert_of_slot),
                                _p(self.last_use), self.step, _p(ids), ids.size, _p(me), _p(ms),
                                _p(nd), _p(nh), _p(nm))
        if rc == 0:
            self.step += 1
        misses = [(int(me[i]), int(ms[i])) for i in range(int(nm[0]))]
        return rc, misses, int(nd[0]), int(nh[0])

    def update_reserve(self, keys: np.ndarray, reserve: int):
        """One step whose misses may only take slots with last_use < reserve
        (see orc_lru_step_reserve).  Returns (status, misses, distinct, hits)."""
        keys = np.ascontiguousarray(keys, dtype=np.int32).ravel()
        mk = np.empty(max(1, self.E), dtype=np.int32)
        ms = np.empty(max(1, self.E), dtype=np.int32)
        nd, nh, nm = (np.zeros(1, dtype=np.int32) for _ in range(3))
        rc = lib().orc_lru_step_reserve(self.E, self.S, _p(self.slot_of_expert), _p(self.expert_of_slot),
                                        _p(self.last_use), self.step, int(reserve), _p(keys), keys.size, _p(mk),
                                        _p(ms), _p(nd), _p(nh), _p(nm))
        if rc == 0:
            self.step += 1
        misses = [(int(mk[i]), int(ms[i])) for i in range(int(nm[0]))]
        return rc, misses, int(nd[0]), int(nh[0])

    def stage_layer(self, layer: int, E: int, overlap: bool):
        """One staging step of a cache shared by layers of E experts (this
        state's E is then n_layers * E): all E experts of `layer` become
        resident.  overlap: the step runs while the previous step's layer
        computes, so that step's slots are kept (reserve = step - 1)."""
        keys = np.arange(layer * E, (layer + 1) * E, dtype=np.int32)
        return self.update_reserve(keys, self.step - 1 if overlap else self.step)

    def resize(self, S_new: int):
        """Elastic resize to S_new slots (see orc_lru_resize).  Returns the new
        state and move_from: slot i of the new pool holds the bank of old slot
        move_from[i]."""
        n = LRUState(self.E, S_new)
        n.step = self.step
        mf = np.empty(max(1, min(self.S, S_new)), dtype=np.int32)
        kept = lib().orc_lru_resize(self.E, self.S, _p(self.slot_of_expert), _p(self.expert_of_slot),
                                    _p(self.last_use), S_new, _p(n.slot_of_expert), _p(n.expert_of_slot),
                                    _p(n.last_use), _p(mf))
        return n, mf[:kept].copy()


def hybrid_split(counts: np.ndarray, resident: np.ndarray, bp: float, bh: float):
    """Bandwidth-adaptive miss split (see orc_hybrid_split).  counts: pairs per
    expert; resident: nonzero where the expert is in the cache.  Returns
    (m, q, host experts in order)."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    resident = np.ascontiguousarray(resident, dtype=np.int32)
    E = counts.size
    host = np.empty(max(1, E), dtype=np.int32)
    m, q = np.zeros(1, dtype=np.int32), np.zeros(1, dtype=np.int32)
    n = lib().orc_hybrid_split(E, _p(counts), _p(resident), ctypes.c_double(bp), ctypes.c_double(bh), _p(host),
                               _p(m), _p(q))
    return int(m[0]), int(q[0]), [int(v) for v in host[:n]]


# ---- expert FFN / combine -----------------------------------------------------------

QA_NONE, QA_FP8, QA_NVFP4, QA_MXFP4 = 0, 1, 2, 3


def expert_ffn(x: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray, qa: int = QA_NONE,
               act_scale: Optional[Tuple[float, float]] = None) -> np.ndarray:
    """act_scale: NVFP4 activation global scales (of x, of h); None: 1, 1."""
    x, Wg, Wu, Wd = _f32(x), _f32(Wg), _f32(Wu), _f32(Wd)
    n, d = x.shape
    I = Wg.shape[0]
    y = np.empty((n, d), dtype=np.float32)
    if act_scale is None:
        lib().orc_expert_ffn(_p(x), n, d, I, _p(Wg), _p(Wu), _p(Wd), qa, _p(y))
    else:
        lib().orc_expert_ffn_gs(_p(x), n, d, I, _p(Wg), _p(Wu), _p(Wd), qa, ctypes.c_float(act_scale[0]),
                                ctypes.c_float(act_scale[1]), _p(y))
    return y


def combine(y_pairs: np.ndarray, gates: np.ndarray, ysh: Optional[np.ndarray]) -> np.ndarray:
    gates = _f32(gates)
    T, k = gates.shape
    y_pairs = _f32(y_pairs)
    d = y_pairs.shape[1]
    out = np.empty((T, d), dtype=np.float32)
    lib().orc_combine(_p(y_pairs), _p(gates), T, k, d, _p(None if ysh is None else _f32(ysh)), _p(out))
    return out


# ---- weights of a synthetic layer in oracle form ------------------------------------

def expert_weights_f32(layer, e: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Dequantised (gate, up, down) of expert e (e == E: the shared expert)."""
    w = layer.cfg.wdtype
    ew = layer.expert(e)
    if w == "f32":
        return ew.gate, ew.up, ew.down
    if w == "bf16":
        return bf16_to_f32(ew.gate), bf16_to_f32(ew.up), bf16_to_f32(ew.down)
    if w == "fp8":
        return tuple(dequant_fp8_b128(q, s) for (q, s) in (ew.gate, ew.up, ew.down))
    if w == "nvfp4":
        return tuple(dequant_nvfp4(q, s16, st) for (q, s16, st) in (ew.gate, ew.up, ew.down))
    if w == "mxfp4":
        return tuple(dequant_mxfp4(q, s) for (q, s) in (ew.gate, ew.up, ew.down))
    raise ValueError(w)


def qa_mode(wdtype: str) -> int:
    return {"f32": QA_NONE, "bf16": QA_NONE, "fp8": QA_FP8, "nvfp4": QA_NVFP4, "mxfp4": QA_MXFP4}[wdtype]


def moe_rows(layer, x: np.ndarray, rows: Sequence[int], ids: np.ndarray, gates: np.ndarray,
             qa: Optional[int] = None, weight_cache: Optional[Dict[int, tuple]] = None,
             act_scale: Optional[Tuple[float, float]] = None) -> np.ndarray:
    """Layer output for the selected token rows (routing given by the oracle's
    own ids/gates for all tokens).  Returns [len(rows), d] float32."""
    cfg = layer.cfg
    qa = qa_mode(cfg.wdtype) if qa is None else qa
    rows = list(rows)
    k = cfg.k
    keep = weight_cache is not None      # without a cache, each expert's weights are dropped after use
    cache = {} if weight_cache is None else weight_cache
    y_pairs = np.zeros((len(rows) * k, cfg.d), dtype=np.float32)
    # group (row, pick) by expert so each expert's weights are dequantised once
    want: Dict[int, List[Tuple[int, int]]] = {}
    for ri, t in enumerate(rows):
        for j in range(k):
            want.setdefault(int(ids[t, j]), []).append((ri, j))
    for e, lst in sorted(want.items()):
        if e not in cache:
            cache[e] = expert_weights_f32(layer, e)
        Wg, Wu, Wd = cache[e]
        xs = np.stack([x[rows[ri]] for ri, _ in lst])
        ys = expert_ffn(xs, Wg, Wu, Wd, qa, act_scale)
        for (ri, j), yv in zip(lst, ys):
            y_pairs[ri * k + j] = yv
        if not keep:
            del cache[e]
    ysh = None
    if cfg.has_shared:
        if cfg.E not in cache:
            cache[cfg.E] = expert_weights_f32(layer, cfg.E)
        Wg, Wu, Wd = cache[cfg.E]
        ysh = expert_ffn(np.stack([x[t] for t in rows]), Wg, Wu, Wd, qa, act_scale)
    g = np.stack([gates[t] for t in rows])
    return combine(y_pairs, g, ysh)
