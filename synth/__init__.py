"""Seeded synthetic inputs for the routed-MoE layer (shared by tests, bench and oracle).

Holds no layer arithmetic: it draws weights and hidden states, rounds them to
their storage formats and builds the seed-shuffled permutations.  The five
layer configurations below restate the workloads the layer is measured on; the
page "FreeToken" (chenxutan.com, section on why bandwidth is the bottleneck)
names the model classes (35B-A3B, 284B with 6 routed experts per token, 753B),
and the sizes come from those model classes.

Stream tags (Philox key word 1) and sub-stream counters (a, b, c):
  router W     TAG_ROUTER   (0, 0, 0)            elements row-major [E][d]
  router bias  TAG_BIAS     (0, 0, 0)
  expert mats  TAG_EXPERT   (expert, matrix, 0)  matrix 0 = gate [I][d], 1 = up [I][d], 2 = down [d][I];
                                                 the shared expert uses expert index E
  hidden rows  TAG_HIDDEN   (step, row, attempt) one row of d values
  slot shuffle TAG_SLOTS    Fisher-Yates
  Zipf order   TAG_ZIPF     Fisher-Yates
"""
from __future__ import annotations

import ctypes
import json
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")

TAG_ROUTER, TAG_BIAS, TAG_EXPERT, TAG_HIDDEN, TAG_SLOTS, TAG_ZIPF = 1, 2, 3, 4, 5, 6
WEIGHT_SIGMA = 0.02
MARGIN = 1e-3


def build(force: bool = False) -> str:
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", _SO, src, "-lm"])
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u32, i64, i32 = ctypes.c_uint32, ctypes.c_int64, ctypes.c_int32
        p = ctypes.c_void_p
        _lib.synth_philox.argtypes = [p, p, p]
        _lib.synth_normal.argtypes = [u32, u32, u32, u32, u32, i64, ctypes.c_double, p]
        _lib.synth_uniform.argtypes = [u32, u32, u32, u32, u32, i64, ctypes.c_double, ctypes.c_double, p]
        _lib.synth_permutation.argtypes = [u32, u32, i32, p]
        _lib.synth_bf16_from_f32.argtypes = [p, i64, p]
        _lib.synth_quant_fp8_b128.argtypes = [p, i32, i32, p, p]
        _lib.synth_quant_nvfp4.argtypes = [p, i32, i32, p, p, p]
        _lib.synth_quant_mxfp4.argtypes = [p, i32, i32, p, p]
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def philox(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().synth_philox(_ptr(c), _ptr(k), _ptr(out))
    return out


def normal(seed, tag, a, b, c, n, sigma=1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_normal(seed, tag, a, b, c, n, sigma, _ptr(out))
    return out


def uniform(seed, tag, a, b, c, n, lo, hi) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    lib().synth_uniform(seed, tag, a, b, c, n, lo, hi, _ptr(out))
    return out


def permutation(seed, tag, n) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    lib().synth_permutation(seed, tag, n, _ptr(out))
    return out


def bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().synth_bf16_from_f32(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def quant_fp8_b128(W: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    W = np.ascontiguousarray(W, dtype=np.float32)
    R, C = W.shape
    assert R % 128 == 0 and C % 128 == 0
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty((R // 128, C // 128), dtype=np.float32)
    lib().synth_quant_fp8_b128(_ptr(W), R, C, _ptr(q), _ptr(s))
    return q, s


def quant_nvfp4(W: np.ndarray) -> Tuple[np.ndarray, np.ndarray, float]:
    W = np.ascontiguousarray(W, dtype=np.float32)
    R, C = W.shape
    assert C % 16 == 0
    q = np.empty((R, C // 2), dtype=np.uint8)
    s16 = np.empty((R, C // 16), dtype=np.uint8)
    st = np.zeros(1, dtype=np.float32)
    lib().synth_quant_nvfp4(_ptr(W), R, C, _ptr(q), _ptr(s16), _ptr(st))
    return q, s16, float(st[0])


def quant_mxfp4(W: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """W [R][C] -> (packed e2m1 [R][C/2], E8M0 scale codes [R][C/32])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    R, C = W.shape
    assert C % 32 == 0
    q = np.empty((R, C // 2), dtype=np.uint8)
    s = np.empty((R, C // 32), dtype=np.uint8)
    lib().synth_quant_mxfp4(_ptr(W), R, C, _ptr(q), _ptr(s))
    return q, s


# --------------------------------------------------------------------------
# Layer configurations (the five synthetic workloads).
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class LayerConfig:
    name: str
    d: int
    E: int
    k: int
    I: int
    wdtype: str           # "f32" | "bf16" | "fp8" | "nvfp4" | "mxfp4"
    has_shared: int
    S: int                # slots in the HBM pool
    bias: str             # "none" | "uniform" | "zero" | "zipf"
    T: Tuple[int, ...]    # token counts the layer is run at
    trace_steps: int = 1  # >1: a decode trace with fresh hidden states per step
    lru: bool = False     # True: the S slots are an LRU cache over E experts in host memory

    @property
    def act_dtype(self) -> str:
        return "f32" if self.wdtype == "f32" else "bf16"


CONFIGS: Dict[str, LayerConfig] = {
    "tiny": LayerConfig("tiny", d=256, E=8, k=2, I=512, wdtype="f32", has_shared=0, S=8,
                        bias="none", T=(16,)),
    "35b_decode": LayerConfig("35b_decode", d=2048, E=128, k=8, I=768, wdtype="bf16", has_shared=0,
                              S=128, bias="uniform", T=(1, 8, 32, 64)),
    "35b_prefill": LayerConfig("35b_prefill", d=2048, E=128, k=8, I=768, wdtype="bf16", has_shared=0,
                               S=128, bias="zero", T=(8192,)),
    "284b_trace": LayerConfig("284b_trace", d=4096, E=256, k=6, I=2048, wdtype="fp8", has_shared=1,
                              S=64, bias="zipf", T=(32,), trace_steps=256, lru=True),
    "753b_nvfp4": LayerConfig("753b_nvfp4", d=6144, E=160, k=8, I=2048, wdtype="nvfp4", has_shared=1,
                              S=160, bias="zero", T=(16, 16384)),
    # the same layer with MXFP4 weights (pomoai.com FreeToken hub, checkpoint
    # list: MXFP4 next to NVFP4, FP8 and BF16); router, bias and hidden states
    # are those of the NVFP4 layer
    "753b_mxfp4": LayerConfig("753b_mxfp4", d=6144, E=160, k=8, I=2048, wdtype="mxfp4", has_shared=1,
                              S=160, bias="zero", T=(16, 16384)),
}

# configurations whose router and hidden states (hence redraw tables) are another's
REDRAWS_OF = {"753b_mxfp4": "753b_nvfp4"}


def scaled(cfg: LayerConfig, **kw) -> LayerConfig:
    """A smaller layer of the same kind (tests): override any field."""
    d = dict(cfg.__dict__)
    d.update(kw)
    return LayerConfig(**d)


@dataclass
class ExpertWeights:
    """One expert in storage form.  For f32/bf16: gate/up [I][d], down [d][I]
    (float32 or bf16 bits).  fp8: (q, s) per matrix.  nvfp4: (q_packed, s16, s_t).
    mxfp4: (q_packed, s32) per matrix (E8M0 codes, one per 32 elements)."""
    gate: object
    up: object
    down: object


class Layer:
    """Weights and hidden states of one synthetic layer, drawn lazily."""

    def __init__(self, cfg: LayerConfig, seed: int = 0, redraws: Optional[Dict[Tuple[int, int], int]] = None):
        self.cfg = cfg
        self.seed = seed
        self.redraws = dict(redraws or {})
        self._experts: Dict[int, ExpertWeights] = {}

    # ---- router -----------------------------------------------------------
    def router_f32(self) -> np.ndarray:
        c = self.cfg
        w = normal(self.seed, TAG_ROUTER, 0, 0, 0, c.E * c.d, WEIGHT_SIGMA).reshape(c.E, c.d)
        if c.act_dtype == "bf16":
            w = bf16_to_f32(bf16_bits(w))
        return w

    def router_storage(self) -> np.ndarray:
        w = self.router_f32()
        return bf16_bits(w) if self.cfg.act_dtype == "bf16" else w

    def zipf_order(self) -> np.ndarray:
        return permutation(self.seed, TAG_ZIPF, self.cfg.E)

    def bias(self) -> Optional[np.ndarray]:
        c = self.cfg
        if c.bias == "none":
            return None
        if c.bias == "zero":
            return np.zeros(c.E, dtype=np.float32)
        if c.bias == "uniform":
            return uniform(self.seed, TAG_BIAS, 0, 0, 0, c.E, -0.5, 0.5)
        if c.bias == "zipf":
            # rank r (1-based) holds expert order[r-1]; b = ln p_r, p_r ~ r^-1.1
            r = np.arange(1, c.E + 1, dtype=np.float64)
            p = r ** -1.1
            p /= p.sum()
            b = np.empty(c.E, dtype=np.float32)
            b[self.zipf_order()] = np.log(p).astype(np.float32)
            return b
        raise ValueError(c.bias)

    # ---- experts ----------------------------------------------------------
    def expert_f32(self, e: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """Drawn fp32 values before storage rounding (e == E: shared expert)."""
        c = self.cfg
        g = normal(self.seed, TAG_EXPERT, e, 0, 0, c.I * c.d, WEIGHT_SIGMA).reshape(c.I, c.d)
        u = normal(self.seed, TAG_EXPERT, e, 1, 0, c.I * c.d, WEIGHT_SIGMA).reshape(c.I, c.d)
        dn = normal(self.seed, TAG_EXPERT, e, 2, 0, c.d * c.I, WEIGHT_SIGMA).reshape(c.d, c.I)
        return g, u, dn

    def expert(self, e: int, cache: bool = False) -> ExpertWeights:
        if e in self._experts:
            return self._experts[e]
        g, u, dn = self.expert_f32(e)
        w = self.cfg.wdtype
        if w == "f32":
            ew = ExpertWeights(g, u, dn)
        elif w == "bf16":
            ew = ExpertWeights(bf16_bits(g), bf16_bits(u), bf16_bits(dn))
        elif w == "fp8":
            ew = ExpertWeights(quant_fp8_b128(g), quant_fp8_b128(u), quant_fp8_b128(dn))
        elif w == "nvfp4":
            ew = ExpertWeights(quant_nvfp4(g), quant_nvfp4(u), quant_nvfp4(dn))
        elif w == "mxfp4":
            ew = ExpertWeights(quant_mxfp4(g), quant_mxfp4(u), quant_mxfp4(dn))
        else:
            raise ValueError(w)
        if cache:
            self._experts[e] = ew
        return ew

    def slot_of_expert(self) -> np.ndarray:
        """Resident layers: expert e lives in slot perm[e] (identity shuffled by seed)."""
        return permutation(self.seed, TAG_SLOTS, self.cfg.E)

    # ---- hidden states ----------------------------------------------------
    def hidden_row_f32(self, step: int, row: int, attempt: int) -> np.ndarray:
        x = normal(self.seed, TAG_HIDDEN, step, row, attempt, self.cfg.d, 1.0)
        if self.cfg.act_dtype == "bf16":
            x = bf16_to_f32(bf16_bits(x))
        return x

    def hidden_f32(self, T: int, step: int = 0, attempts: Optional[np.ndarray] = None) -> np.ndarray:
        x = np.empty((T, self.cfg.d), dtype=np.float32)
        for r in range(T):
            a = int(attempts[r]) if attempts is not None else self.redraws.get((step, r), 0)
            x[r] = self.hidden_row_f32(step, r, a)
        return x

    def hidden_storage(self, T: int, step: int = 0) -> np.ndarray:
        x = self.hidden_f32(T, step)
        return bf16_bits(x) if self.cfg.act_dtype == "bf16" else x


# --------------------------------------------------------------------------
# Redraw tables: which hidden rows were redrawn to keep a top-k logit margin.
# --------------------------------------------------------------------------

GOLDEN = os.path.join(os.path.dirname(_HERE), "tests", "golden")


def redraw_path(name: str, T: int) -> str:
    return os.path.join(GOLDEN, f"redraws_{name}_T{T}.json")


def load_redraws(name: str, T: int) -> Optional[Dict[Tuple[int, int], int]]:
    p = redraw_path(REDRAWS_OF.get(name, name), T)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    return {(int(s), int(r)): int(a) for s, r, a in d["redraws"]}


def screen_hidden(layer: Layer, T: int, steps: int, margin_ok) -> Dict[Tuple[int, int], int]:
    """Draw each step's T rows; rows whose router margin fails (margin_ok is a
    callback returning a bool per row) are redrawn with the next attempt index
    until all pass.  Returns {(step, row): attempt} for redrawn rows."""
    table: Dict[Tuple[int, int], int] = {}
    for s in range(steps):
        att = np.zeros(T, dtype=np.int64)
        x = layer.hidden_f32(T, s, att)
        while True:
            ok = np.asarray(margin_ok(x), dtype=bool)
            bad = np.nonzero(~ok)[0]
            if bad.size == 0:
                break
            for r in bad:
                att[r] += 1
                x[r] = layer.hidden_row_f32(s, int(r), int(att[r]))
        for r in np.nonzero(att)[0]:
            table[(s, int(r))] = int(att[r])
    return table
