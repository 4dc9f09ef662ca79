"""FP8 (e4m3, 128x128 block scales) layers: parity with the oracle in its
activation-quantised mode (x and H quantised per 1x128 group), bar 5e-2 of the
row max; and the 284B-class slot-cache decode trace, with the LRU state checked
bit-exactly after every step."""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from synth.device import DeviceLayer, Workspace
from tests.gpu_util import TOL, assert_rows_close, oracle_route, oracle_rows, run_layer, screened_layer, to_np_f32

pytestmark = pytest.mark.gpu

SMALL_FP8 = synth.scaled(synth.CONFIGS["284b_trace"], name="small_fp8", d=256, I=256, E=16, k=4, S=16,
                         has_shared=1, lru=False, bias="uniform", T=(300,), trace_steps=1)


@pytest.mark.parametrize("T", [1, 24, 300])
def test_small_fp8_layer(T):
    dl = screened_layer(SMALL_FP8, T)
    x_dev = dl.hidden(T)
    out = to_np_f32(run_layer(dl, x_dev, T))
    x, ids, g = oracle_route(dl, T)
    want = oracle_rows(dl, x, ids, g, range(T))
    assert_rows_close(out, want, TOL["fp8"], f"fp8 T={T}")
    # against the oracle without activation quantisation the error stays moderate
    plain = oracle.moe_rows(dl.layer, x, range(T), ids, g, qa=oracle.QA_NONE)
    assert_rows_close(out, plain, 0.15, "fp8 vs unquantised activations")


def test_284b_trace_slot_cache():
    """256 decode steps of T=32 over 64 HBM slots and 256 experts in pinned
    host memory.  Slot table, reverse table and last-use stamps must equal the
    oracle's LRU after every step; sampled outputs within 5e-2."""
    cfg = synth.CONFIGS["284b_trace"]
    dl = DeviceLayer(cfg)
    T = cfg.T[0]
    ref = oracle.LRUState(cfg.E, cfg.S)
    Wr = oracle.bf16_to_f32(dl.layer.router_storage())
    b = dl.layer.bias()
    ws = Workspace(ftm.ftm_workspace_bytes(dl.desc, T))
    out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    copy_stream = torch.cuda.Stream()
    check_steps = {0, 1, 2, cfg.trace_steps - 1} | set(range(3, cfg.trace_steps, 8))   # 35 steps
    cache = {}
    hits = distinct = 0
    for s in range(cfg.trace_steps):
        x_dev = dl.hidden(T, step=s)
        ftm.ftm_moe_layer_forward(dl.desc, dl.weights(), dl.cache, x_dev, T, out, ws.ptr, ws.nbytes, None,
                                  copy_stream)
        torch.cuda.synchronize()
        x = oracle.bf16_to_f32(dl.layer.hidden_storage(T, s))
        ids, g, _ = oracle.route(x, Wr, b, cfg.k)
        rc, misses, nd, nh = ref.update(ids)
        assert rc == 0
        hits += nh
        distinct += nd
        assert dl.cache.step == ref.step
        assert np.array_equal(dl.slot_of_expert.cpu().numpy(), ref.slot_of_expert), f"step {s}"
        assert np.array_equal(dl.expert_of_slot.cpu().numpy(), ref.expert_of_slot), f"step {s}"
        assert np.array_equal(dl.last_use.cpu().numpy(), ref.last_use), f"step {s}"
        assert (dl.cache.last_hits, dl.cache.last_misses) == (nh, len(misses))
        if s in check_steps:
            rows = [0, 11, 21, T - 1]
            want = oracle.moe_rows(dl.layer, x, rows, ids, g, weight_cache=cache)
            assert_rows_close(to_np_f32(out)[rows], want, TOL["fp8"], f"trace step {s}")
            if len(cache) > 24:
                cache.clear()
    assert len(check_steps) >= 32
    assert ftm.ftm_device_status(True) == 0
    hit_rate = hits / distinct
    assert 0.5 < hit_rate < 0.95, hit_rate
