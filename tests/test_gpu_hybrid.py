"""The layer with the bandwidth-adaptive miss split (ftm_moe_layer_forward_hybrid)
on the GPU, through the C ABI, against the oracle.

Every step of a decode trace over an LRU cache: the split (m, q and the host's
experts) equals orc_hybrid_split's on the oracle's routing and the oracle cache
state before the step; the slot table, reverse table and last-use stamps equal
the oracle LRU after a step that requested only the GPU's experts (hits and
the q copied misses), bit for bit; every output row is within the dtype's bar
of the oracle layer.  Bh = 0 reduces to the plain cache step: outputs and
state bit-identical to ftm_moe_layer_forward.  Bp = 0 computes every miss on
the host and leaves the cache as the hits found it.
"""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from synth.device import Workspace
from tests.gpu_util import TOL, assert_rows_close, oracle_route, screened_layer, to_np_f32

pytestmark = pytest.mark.gpu

HYB = {
    "fp8": synth.scaled(synth.CONFIGS["284b_trace"], name="hyb_fp8", d=256, I=256, E=32, k=4, S=10, has_shared=1,
                        T=(16,), trace_steps=10),
    "bf16": synth.scaled(synth.CONFIGS["35b_decode"], name="hyb_bf16", d=256, I=256, E=32, k=4, S=10,
                         bias="zipf", T=(16,), trace_steps=10, lru=True),
    "nvfp4": synth.scaled(synth.CONFIGS["753b_nvfp4"], name="hyb_nvfp4", d=256, I=256, E=32, k=4, S=10,
                          bias="zipf", T=(16,), trace_steps=10, lru=True),
    "mxfp4": synth.scaled(synth.CONFIGS["753b_mxfp4"], name="hyb_mxfp4", d=256, I=256, E=32, k=4, S=10,
                          bias="zipf", T=(16,), trace_steps=10, lru=True),
}


def _hybrid(desc, T, bp, bh, threads=4):
    nb = ftm.ftm_hybrid_host_bytes(desc, T)
    buf = torch.empty(nb, dtype=torch.uint8, pin_memory=True)
    h = ftm.Hybrid(bp, bh, threads, 0, 0, 0, 0.0, buf.data_ptr(), nb)
    return h, buf


def _state(dl):
    return (dl.slot_of_expert.cpu().numpy().copy(), dl.expert_of_slot.cpu().numpy().copy(),
            dl.last_use.cpu().numpy().copy())


def _run_trace(wdtype, bp, bh):
    cfg = HYB[wdtype]
    T = cfg.T[0]
    dl = screened_layer(cfg, T, steps=cfg.trace_steps)
    ref = oracle.LRUState(cfg.E, cfg.S)
    ws = Workspace(ftm.ftm_hybrid_workspace_bytes(dl.desc, T))
    out = torch.empty((T, cfg.d), dtype=dl.out_dtype(), device="cuda")
    copy_stream = torch.cuda.Stream()
    h, hbuf = _hybrid(dl.desc, T, bp, bh)
    wcache = {}
    totals = [0, 0]
    for s in range(cfg.trace_steps):
        x_dev = dl.hidden(T, step=s)
        ftm.ftm_moe_layer_forward_hybrid(dl.desc, dl.weights(), dl.cache, h, x_dev, T, out, ws.ptr, ws.nbytes, None,
                                         copy_stream)
        torch.cuda.synchronize()
        x, ids, g = oracle_route(dl, T, s)
        counts = oracle.permute(ids, cfg.E)[0]
        m, q, host = oracle.hybrid_split(counts, ref.slot_of_expert >= 0, bp, bh)
        assert (h.last_misses, h.last_host, h.last_host_rows) == (m, m - q, int(sum(counts[e] for e in host))), s
        gpu_ids = ids[~np.isin(ids, host)]
        rc, misses, nd, nh = ref.update(gpu_ids)
        assert rc == 0 and len(misses) == q
        soe, eos, lu = _state(dl)
        assert np.array_equal(soe, ref.slot_of_expert), f"step {s}"
        assert np.array_equal(eos, ref.expert_of_slot), f"step {s}"
        assert np.array_equal(lu, ref.last_use), f"step {s}"
        assert (dl.cache.last_hits, dl.cache.last_misses) == (nh, q)
        want = oracle.moe_rows(dl.layer, x, range(T), ids, g, weight_cache=wcache)
        assert_rows_close(to_np_f32(out), want, TOL[wdtype], f"{wdtype} hybrid step {s}")
        totals[0] += m
        totals[1] += m - q
    assert ftm.ftm_device_status(True) == 0
    del hbuf
    return totals


@pytest.mark.parametrize("wdtype,bp,bh", [("fp8", 1.0, 1.0), ("fp8", 52.7, 77.3), ("fp8", 3.0, 1.0),
                                          ("bf16", 1.0, 1.0), ("bf16", 52.7, 77.3), ("nvfp4", 1.0, 1.0),
                                          ("mxfp4", 1.0, 1.0)])
def test_hybrid_trace_matches_oracle(wdtype, bp, bh):
    m, host = _run_trace(wdtype, bp, bh)
    assert m > 0 and host > 0     # the split really sent work both ways


def test_hybrid_every_miss_on_the_host():
    m, host = _run_trace("fp8", 0.0, 1.0)
    assert m == host > 0


def test_hybrid_without_host_bandwidth_is_the_plain_cache_step():
    cfg = HYB["fp8"]
    T = cfg.T[0]
    a = screened_layer(cfg, T, steps=cfg.trace_steps)
    b = screened_layer(cfg, T, steps=cfg.trace_steps)
    ws_a = Workspace(ftm.ftm_workspace_bytes(a.desc, T))
    ws_b = Workspace(ftm.ftm_hybrid_workspace_bytes(b.desc, T))
    out_a = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    out_b = torch.empty_like(out_a)
    cs = torch.cuda.Stream()
    h, hbuf = _hybrid(b.desc, T, 1.0, 0.0)
    for s in range(cfg.trace_steps):
        ftm.ftm_moe_layer_forward(a.desc, a.weights(), a.cache, a.hidden(T, s), T, out_a, ws_a.ptr, ws_a.nbytes, None,
                                  cs)
        ftm.ftm_moe_layer_forward_hybrid(b.desc, b.weights(), b.cache, h, b.hidden(T, s), T, out_b, ws_b.ptr,
                                         ws_b.nbytes, None, cs)
        torch.cuda.synchronize()
        assert h.last_host == 0
        assert torch.equal(out_a, out_b), f"step {s}"
        for u, v in zip(_state(a), _state(b)):
            assert np.array_equal(u, v), f"step {s}"
    assert ftm.ftm_device_status(True) == 0
    del hbuf


def _step(dl, h, ws, out, cs, s, T):
    ftm.ftm_moe_layer_forward_hybrid(dl.desc, dl.weights(), dl.cache, h, dl.hidden(T, s), T, out, ws.ptr, ws.nbytes,
                                     None, cs)
    torch.cuda.synchronize()


def test_hybrid_capacity_refused_with_state_unchanged():
    """Two slots: a cold step whose GPU share needs more than two copies is
    refused with the state untouched; the same step with every miss on the host
    (Bp = 0) needs no slot and matches the oracle."""
    cfg = synth.scaled(HYB["fp8"], name="hyb_fp8_s2", S=2)
    T = cfg.T[0]
    dl = screened_layer(cfg, T, steps=1)
    ws = Workspace(ftm.ftm_hybrid_workspace_bytes(dl.desc, T))
    out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    cs = torch.cuda.Stream()
    x, ids, g = oracle_route(dl, T, 0)
    m, q, _ = oracle.hybrid_split(oracle.permute(ids, cfg.E)[0], np.zeros(cfg.E, np.int32), 1.0, 0.0)
    assert q == m > cfg.S
    h, hbuf = _hybrid(dl.desc, T, 1.0, 0.0)
    before = _state(dl)
    with pytest.raises(ftm.FtmError) as ei:
        _step(dl, h, ws, out, cs, 0, T)
    assert ei.value.status == ftm.binding.FTM_ERR_CAPACITY and dl.cache.step == 0
    assert all(np.array_equal(u, v) for u, v in zip(before, _state(dl)))
    h.pcie_gbs, h.host_gbs = 0.0, 1.0
    _step(dl, h, ws, out, cs, 0, T)
    assert (h.last_misses, h.last_host) == (m, m) and dl.cache.step == 1
    assert all(np.array_equal(u, v) for u, v in zip(before, _state(dl)))   # nothing inserted, nothing touched
    want = oracle.moe_rows(dl.layer, x, range(T), ids, g)
    assert_rows_close(to_np_f32(out), want, TOL["fp8"], "all misses on the host")
    assert ftm.ftm_device_status(True) == 0
    del hbuf


def test_hybrid_copy_failure_rolls_back_then_the_step_succeeds():
    """A step whose first miss copy cannot be issued (the library's test hook)
    fails with FTM_ERR_CUDA and leaves the cache as it was; the same step then
    runs and matches the oracle's split, LRU state and outputs."""
    cfg = HYB["fp8"]
    T = cfg.T[0]
    dl = screened_layer(cfg, T, steps=1)
    ws = Workspace(ftm.ftm_hybrid_workspace_bytes(dl.desc, T))
    out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    cs = torch.cuda.Stream()
    h, hbuf = _hybrid(dl.desc, T, 1.0, 1.0)
    before = _state(dl)
    dl.cache.fail_before_copy = 1
    with pytest.raises(ftm.FtmError) as ei:
        _step(dl, h, ws, out, cs, 0, T)
    assert ei.value.status == ftm.binding.FTM_ERR_CUDA and dl.cache.step == 0 and dl.cache.fail_before_copy == 0
    assert all(np.array_equal(u, v) for u, v in zip(before, _state(dl)))
    _step(dl, h, ws, out, cs, 0, T)
    x, ids, g = oracle_route(dl, T, 0)
    counts = oracle.permute(ids, cfg.E)[0]
    ref = oracle.LRUState(cfg.E, cfg.S)
    m, q, host = oracle.hybrid_split(counts, ref.slot_of_expert >= 0, 1.0, 1.0)
    assert q > 0 and (h.last_misses, h.last_host) == (m, m - q)
    assert ref.update(ids[~np.isin(ids, host)])[0] == 0
    for u, v in zip(_state(dl), (ref.slot_of_expert, ref.expert_of_slot, ref.last_use)):
        assert np.array_equal(u, v)
    assert_rows_close(to_np_f32(out), oracle.moe_rows(dl.layer, x, range(T), ids, g), TOL["fp8"], "after rollback")
    assert ftm.ftm_device_status(True) == 0
    del hbuf
