"""MXFP4 layers (e2m1 weights with one E8M0 scale per 32 elements, OCP MX;
block-scaled tcgen05 MMA with 32-element blocks): parity with the oracle in
its MXFP4 activation mode (x and H quantised per 32-group with E8M0 scales),
bar 5e-2 of the row max, like the other 4-bit format."""
import pytest

import oracle
import synth
from synth.device import DeviceLayer
from tests.gpu_util import (TOL, assert_rows_close, group_edge_rows, oracle_route, oracle_rows, run_layer,
                            screened_layer, to_np_f32)

pytestmark = pytest.mark.gpu

SMALL_MX = synth.scaled(synth.CONFIGS["753b_mxfp4"], name="small_mxfp4", d=256, I=256, E=16, k=4, S=16,
                        has_shared=1, bias="uniform", T=(300,))


def _check(dl, T, rows=None):
    x_dev = dl.hidden(T)
    out = to_np_f32(run_layer(dl, x_dev, T))
    x, ids, g = oracle_route(dl, T)
    rows = list(range(T)) if rows is None else list(rows)
    want = oracle_rows(dl, x, ids, g, rows)
    assert_rows_close(out[rows], want, TOL["nvfp4"], f"{dl.cfg.name} T={T}")
    return out, x, ids, g, rows


@pytest.mark.parametrize("T", [1, 20, 300, 700, 1100])   # token tiles of 32, 32, 64, 128 rows; CTA pairs
def test_small_mxfp4_layer(T):
    dl = screened_layer(SMALL_MX, T)
    out, x, ids, g, rows = _check(dl, T)
    # against the oracle without activation quantisation: the W4A4 error itself.
    # E8M0 scales put a block's amax between 4 and 8 units of its scale, so
    # values above 6 saturate: a looser bound than NVFP4's e4m3 scales need
    plain = oracle.moe_rows(dl.layer, x, rows, ids, g, qa=oracle.QA_NONE)
    assert_rows_close(out[rows], plain, 0.5, "mxfp4 vs unquantised activations")


def test_mxfp4_pair_tiles_multi_stage():
    cfg = synth.scaled(SMALL_MX, name="small_mxfp4_pairs", d=768, I=512, E=12, k=4, S=12)
    dl = screened_layer(cfg, 900)
    _check(dl, 900)


def test_small_mxfp4_no_shared_expert():
    cfg = synth.scaled(SMALL_MX, name="small_mxfp4_ns", has_shared=0, E=24, k=3, S=32)
    dl = screened_layer(cfg, 45)
    _check(dl, 45)


@pytest.fixture(scope="module")
def dl_753b_mx():
    return DeviceLayer(synth.CONFIGS["753b_mxfp4"])


def test_753b_mxfp4_decode_layer(dl_753b_mx):
    _check(dl_753b_mx, 16)


def test_753b_mxfp4_prefill_layer_512_rows(dl_753b_mx):
    T = 16384
    _, ids, _ = oracle_route(dl_753b_mx, T)
    rows = group_edge_rows(ids, dl_753b_mx.cfg.E, T, 512, seed=2)
    _check(dl_753b_mx, T, rows)
