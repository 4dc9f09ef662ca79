"""Bit-exact routing and permutation at the full size of every configuration
(router on its real shape: the tensor-core router at 35B prefill and 753B
prefill, the 284B and 753B routers at decode sizes, every step of a stretch
of the 284B trace), checked against the oracle's router and permutation."""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from synth.device import Workspace, to_device_storage
from tests.gpu_util import gate_rtol

pytestmark = pytest.mark.gpu


def _route_permute_case(cfg, T, step=0):
    layer = synth.Layer(cfg, 0, synth.load_redraws(cfg.name, max(cfg.T)) or {})
    desc = ftm.desc_for(cfg)
    x_st = layer.hidden_storage(T, step)
    wr_st = layer.router_storage()
    b = layer.bias()
    x = to_device_storage(x_st, cfg.act_dtype)
    wr = to_device_storage(wr_st, cfg.act_dtype)
    bias = None if b is None else torch.from_numpy(b).cuda()
    P = T * cfg.k
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(P, dtype=torch.int32, device="cuda")
    inv = torch.empty(P, dtype=torch.int32, device="cuda")
    ws = Workspace(ftm.ftm_permute_workspace_bytes(desc, T))
    ftm.ftm_route(desc, x, T, wr, bias, ids, gw)
    ftm.ftm_permute(desc, ids, T, counts, offsets, perm, inv, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert ftm.ftm_device_status(True) == 0
    to32 = oracle.bf16_to_f32 if cfg.act_dtype == "bf16" else (lambda a: np.asarray(a, np.float32))
    rid, rg, _ = oracle.route(to32(x_st), to32(wr_st), b, cfg.k)
    assert np.array_equal(ids.cpu().numpy(), rid), f"{cfg.name} T={T} step {step}: routing ids differ"
    g = gw.cpu().numpy()
    rel = float((np.abs(g - rg) / np.abs(rg)).max())
    assert np.allclose(g, rg, rtol=gate_rtol(cfg.d), atol=1e-6), f"worst gate relative error {rel:.3g}"
    rc, ro, rp, ri = oracle.permute(rid, cfg.E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)
    return rc


@pytest.mark.parametrize("name,T", [("35b_prefill", 8192), ("753b_nvfp4", 16), ("753b_nvfp4", 16384),
                                    ("35b_decode", 32), ("284b_trace", 32)])
def test_route_and_permute_full_size(name, T):
    counts = _route_permute_case(synth.CONFIGS[name], T)
    if name == "35b_prefill":
        assert (counts > 0).all()            # near-uniform routing: every expert receives tokens


def test_route_and_permute_284b_trace_steps():
    cfg = synth.CONFIGS["284b_trace"]
    for step in range(16):
        _route_permute_case(cfg, cfg.T[0], step)
