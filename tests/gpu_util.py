"""Helpers of the GPU parity tests: run the C ABI on a staged layer and build the
oracle's expected values from the same seeded inputs."""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from synth.device import DeviceLayer, Workspace

TOL = {"f32": 2e-2, "bf16": 2e-2, "fp8": 5e-2, "nvfp4": 5e-2, "mxfp4": 5e-2}
TOL_F32_SIMT = 1e-4


def gate_rtol(d: int, sigma_x: float = 1.0, sigma_w: float = 0.02) -> float:
    """Relative tolerance of the gates against the oracle, from the arithmetic.
    A logit is d exact products accumulated in fp32 (unit roundoff u = 2^-24);
    its partial sums random-walk with step sigma_x * sigma_w, so the rounding
    error has standard deviation about u * sigma_x * sigma_w * d / sqrt(2).  A
    gate is the softmax of the k picked logits: its relative error is at most
    twice the largest logit error.  Six standard deviations, and never below
    1e-5 (the bar for the widths where fp32 rounding is far smaller)."""
    u = 2.0 ** -24
    return max(1e-5, 2 * 6 * u * sigma_x * sigma_w * d / np.sqrt(2.0))


def screened_layer(cfg: synth.LayerConfig, T: int, steps: int = 1, seed: int = 0, slot_perm=None) -> DeviceLayer:
    """A device layer whose hidden rows are screened for the top-k margin by the oracle."""
    base = synth.Layer(cfg, seed)
    Wr = base.router_f32()
    b = base.bias()
    table = synth.screen_hidden(base, T, steps,
                                lambda x: oracle.margin_ok(oracle.router_logits(x, Wr, b), cfg.k, synth.MARGIN))
    return DeviceLayer(cfg, seed, redraws=table, slot_perm=slot_perm)


def storage_to_f32(dl: DeviceLayer, arr: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f32(arr) if dl.cfg.act_dtype == "bf16" else np.asarray(arr, np.float32)


def oracle_route(dl: DeviceLayer, T: int, step: int = 0):
    x = storage_to_f32(dl, dl.layer.hidden_storage(T, step))
    Wr = storage_to_f32(dl, dl.layer.router_storage())
    ids, g, lg = oracle.route(x, Wr, dl.layer.bias(), dl.cfg.k)
    return x, ids, g


def to_np_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def run_layer(dl: DeviceLayer, x_dev: torch.Tensor, T: int, cache: bool = False) -> torch.Tensor:
    out = torch.empty((T, dl.cfg.d), dtype=dl.out_dtype(), device=x_dev.device)
    ws = Workspace(ftm.ftm_workspace_bytes(dl.desc, T))
    copy_stream = torch.cuda.Stream() if cache else None
    ftm.ftm_moe_layer_forward(dl.desc, dl.weights(), dl.cache if cache else None, x_dev, T, out, ws.ptr, ws.nbytes,
                              None, copy_stream)
    torch.cuda.synchronize()
    assert ftm.ftm_device_status(True) == 0
    return out


def oracle_rows(dl: DeviceLayer, x: np.ndarray, ids: np.ndarray, g: np.ndarray, rows: Sequence[int],
                cache: Optional[Dict] = None) -> np.ndarray:
    return oracle.moe_rows(dl.layer, x, rows, ids, g, weight_cache=cache)


def assert_rows_close(got: np.ndarray, want: np.ndarray, frac: float, what: str = ""):
    """max-abs error per token row <= frac * max |oracle row|."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    err = np.abs(got - want).max(axis=1)
    scale = np.abs(want).max(axis=1)
    bad = np.nonzero(err > frac * scale)[0]
    worst = float((err / np.maximum(scale, 1e-30)).max()) if len(err) else 0.0
    assert bad.size == 0, f"{what}: {bad.size} rows exceed {frac} (worst ratio {worst:.3g}, rows {bad[:8]})"
    return worst


def group_edge_rows(ids: np.ndarray, E: int, T: int, n: int = 512, seed: int = 0):
    """Token rows to check on a large batch: the tokens of the first and the
    last pair of every expert group (the ragged edges of the GEMM tiles), the
    first and last token, and seeded random tokens up to n rows."""
    counts, offsets, perm, _ = oracle.permute(ids, E)
    k = ids.shape[1]
    rows = {0, T - 1}
    for e in range(E):
        if counts[e]:
            rows.add(int(perm[offsets[e]]) // k)
            rows.add(int(perm[offsets[e + 1] - 1]) // k)
    rng = np.random.default_rng(seed)
    while len(rows) < min(n, T):
        rows.add(int(rng.integers(T)))
    return sorted(rows)
