"""NVFP4 activation global scales (the per-tensor activation scale an NVFP4
checkpoint's calibration supplies): small activations, which the scale-1
quantiser sends to zero, stay within the NVFP4 bar once the caller passes
calibrated scales; scale (1, 1) is the default path bit for bit."""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from synth.device import DeviceLayer, Workspace, to_device_storage
from tests.gpu_util import TOL, assert_rows_close, run_layer, screened_layer, to_np_f32

pytestmark = pytest.mark.gpu

CFG = synth.scaled(synth.CONFIGS["753b_nvfp4"], name="small_nvfp4_scales", d=512, I=256, E=16, k=4, S=16,
                   has_shared=1, bias="uniform", T=(96,))


def _ffn(dl, x_dev, T, ids, act):
    cfg = dl.cfg
    counts, offsets, perm, inv = oracle.permute(ids, cfg.E)
    P = T * cfg.k
    y = torch.empty((P + T, cfg.d), dtype=torch.bfloat16, device="cuda")
    ws = Workspace(ftm.ftm_ffn_workspace_bytes(dl.desc, T))
    ftm.ftm_expert_ffn(dl.desc, x_dev, T, torch.from_numpy(offsets).cuda(), torch.from_numpy(perm).cuda(),
                       dl.slot_of_expert, dl.pool, dl.shared_bank, y, ws.ptr, ws.nbytes, act_scale=act)
    torch.cuda.synchronize()
    assert ftm.ftm_device_status(True) == 0
    return to_np_f32(y), perm


def _oracle_pairs(dl, x, ids, perm, act, qa=oracle.QA_NVFP4):
    """Unweighted FFN output of every permuted pair and of the shared expert."""
    cfg = dl.cfg
    T = x.shape[0]
    want = np.zeros((T * cfg.k + T, cfg.d), np.float32)
    for e in range(cfg.E + 1):
        W = oracle.expert_weights_f32(dl.layer, e)
        if e == cfg.E:
            want[T * cfg.k:] = oracle.expert_ffn(x, *W, qa, act)
            continue
        pos = [p for p in range(T * cfg.k) if ids.ravel()[perm[p]] == e]
        if pos:
            want[pos] = oracle.expert_ffn(x[[perm[p] // cfg.k for p in pos]], *W, qa, act)
    return want


def test_small_activations_with_calibrated_global_scales():
    dl = DeviceLayer(CFG)
    T, cfg = 96, CFG
    x = oracle.bf16_to_f32(synth.bf16_bits(dl.layer.hidden_f32(T) * np.float32(1e-2)))   # x ~ N(0, 1e-4)
    rng = np.random.default_rng(3)
    ids = np.stack([rng.choice(cfg.E, size=cfg.k, replace=False) for _ in range(T)]).astype(np.int32)
    x_dev = to_device_storage(synth.bf16_bits(x), "bf16")
    # calibration: amax of x and of the (unquantised) SwiGLU output over this batch
    hmax = 0.0
    for e in range(cfg.E + 1):
        Wg, Wu, _ = oracle.expert_weights_f32(dl.layer, e)
        g, u = x.astype(np.float64) @ Wg.T.astype(np.float64), x.astype(np.float64) @ Wu.T.astype(np.float64)
        hmax = max(hmax, float(np.abs(g / (1 + np.exp(-g)) * u).max()))
    gx, gh = float(np.abs(x).max()) / (6 * 448), hmax / (6 * 448)
    act = torch.tensor([gx, gh], dtype=torch.float32, device="cuda")
    got, perm = _ffn(dl, x_dev, T, ids, act)
    want = _oracle_pairs(dl, x, ids, perm, (gx, gh))
    assert_rows_close(got, want, TOL["nvfp4"], "calibrated global scales")
    plain = _oracle_pairs(dl, x, ids, perm, None, qa=oracle.QA_NONE)
    assert_rows_close(got, plain, 0.35, "vs unquantised activations")
    # with global scales 1 the same batch quantises h to zero: the edge the scales fix
    got1, _ = _ffn(dl, x_dev, T, ids, None)
    want1 = _oracle_pairs(dl, x, ids, perm, None)
    assert np.abs(want1).max() == 0.0 and np.abs(got1).max() == 0.0


def test_unit_global_scales_are_the_default_path():
    T = 300
    dl = screened_layer(CFG, T)
    x = dl.hidden(T)
    a = run_layer(dl, x, T)
    ones = torch.ones(2, dtype=torch.float32, device="cuda")
    w = dl.weights()
    w.act_scale = ones.data_ptr()
    out = torch.empty_like(a)
    ws = Workspace(ftm.ftm_workspace_bytes(dl.desc, T))
    ftm.ftm_moe_layer_forward(dl.desc, w, None, x, T, out, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert torch.equal(a, out)
