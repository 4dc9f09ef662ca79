"""NVFP4 layers (e2m1 weights, e4m3 scale per 16, fp32 per-tensor scale; block-
scaled tcgen05 MMA): parity with the oracle in its activation-quantised mode
(x and H quantised to NVFP4 with 16-element groups), bar 5e-2 of the row max."""
import numpy as np
import pytest

import oracle
import synth
from synth.device import DeviceLayer
from tests.gpu_util import (TOL, assert_rows_close, group_edge_rows, oracle_route, oracle_rows, run_layer,
                            screened_layer, to_np_f32)

pytestmark = pytest.mark.gpu

SMALL_FP4 = synth.scaled(synth.CONFIGS["753b_nvfp4"], name="small_nvfp4", d=256, I=256, E=16, k=4, S=16,
                         has_shared=1, bias="uniform", T=(300,))


def _check(dl, T, rows=None):
    x_dev = dl.hidden(T)
    out = to_np_f32(run_layer(dl, x_dev, T))
    x, ids, g = oracle_route(dl, T)
    rows = list(range(T)) if rows is None else list(rows)
    want = oracle_rows(dl, x, ids, g, rows)
    worst = assert_rows_close(out[rows], want, TOL["nvfp4"], f"{dl.cfg.name} T={T}")
    return out, x, ids, g, rows, worst


@pytest.mark.parametrize("T", [1, 20, 300, 700, 1100])   # token tiles of 32, 32, 64, 128 rows; CTA pairs
def test_small_nvfp4_layer(T):
    dl = screened_layer(SMALL_FP4, T)
    out, x, ids, g, rows, worst = _check(dl, T)
    # against the oracle without activation quantisation (W4A4 error is expected to be larger)
    plain = oracle.moe_rows(dl.layer, x, rows, ids, g, qa=oracle.QA_NONE)
    assert_rows_close(out[rows], plain, 0.35, "nvfp4 vs unquantised activations")


def test_nvfp4_pair_tiles_multi_stage():
    # >= 192 rows per expert on average: both GEMMs on CTA pairs (224-token
    # tiles), several K stages in each GEMM, ragged groups and a shared expert
    cfg = synth.scaled(SMALL_FP4, name="small_nvfp4_pairs", d=768, I=512, E=12, k=4, S=12)
    dl = screened_layer(cfg, 900)
    _check(dl, 900)


def test_small_nvfp4_no_shared_expert():
    cfg = synth.scaled(SMALL_FP4, name="small_nvfp4_ns", has_shared=0, E=24, k=3, S=32)
    dl = screened_layer(cfg, 45)
    _check(dl, 45)


@pytest.fixture(scope="module")
def dl_753b():
    return DeviceLayer(synth.CONFIGS["753b_nvfp4"])


def test_753b_nvfp4_decode_layer(dl_753b):
    _check(dl_753b, 16)


def test_753b_nvfp4_prefill_layer_512_rows(dl_753b):
    """512 token rows of the 16384-token prefill, including the tokens of the
    first and last pair of every expert group (the ragged 224-token tile edges)."""
    T = 16384
    _, ids, _ = oracle_route(dl_753b, T)
    rows = group_edge_rows(ids, dl_753b.cfg.E, T, 512, seed=1)
    assert len(rows) >= 512
    _check(dl_753b, T, rows)
