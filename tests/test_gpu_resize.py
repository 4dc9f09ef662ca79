"""Elastic slot-pool resize on the GPU: the new slot table, reverse table and
last-use stamps equal the oracle's bit for bit, every kept bank is moved
intact, the cache keeps following the LRU rule afterwards, and a layer run on
the resized cache matches the oracle."""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from tests.gpu_util import TOL, Workspace, assert_rows_close, screened_layer, to_np_f32

pytestmark = pytest.mark.gpu


def _cache_arrays(E, S, bank_bytes, fill=7):
    soe = torch.full((E,), fill, dtype=torch.int32, device="cuda")     # garbage: every entry must be written
    eos = torch.full((S,), fill, dtype=torch.int32, device="cuda")
    lu = torch.full((S,), fill, dtype=torch.int64, device="cuda")
    pool = torch.zeros(S * bank_bytes, dtype=torch.uint8, device="cuda")
    return soe, eos, lu, pool


def _zipf_ids(rng, E, n, order):
    z = 1.0 / np.arange(1, E + 1) ** 1.1
    return order[rng.choice(E, size=n, p=z / z.sum())].astype(np.int32)


@pytest.mark.parametrize("E,S,S_new", [(64, 16, 6), (64, 16, 16), (64, 16, 40), (16, 4, 1), (300, 200, 150)])
def test_slot_resize_bit_exact(E, S, S_new):
    cfg = synth.LayerConfig("lru_resize", d=128, E=E, k=6, I=128, wdtype="bf16", has_shared=0, S=S, bias="zipf",
                            T=(1,), lru=True)
    desc = ftm.desc_for(cfg)
    bb = ftm.ftm_get_bank_layout(desc).bank_bytes
    host_pool = torch.empty(E * bb, dtype=torch.uint8, pin_memory=True)
    host_pool.copy_(torch.arange(E, dtype=torch.int32).repeat_interleave(bb // 4).view(torch.uint8))
    soe, eos, lu, pool = _cache_arrays(E, S, bb, fill=-1)
    scratch = torch.zeros(ftm.ftm_slot_host_scratch_ints(desc), dtype=torch.int32, pin_memory=True)
    cache = ftm.SlotCache(soe.data_ptr(), eos.data_ptr(), lu.data_ptr(), 0, pool.data_ptr(), host_pool.data_ptr(),
                          scratch.data_ptr(), 0, 0, 0, 0)
    ws = Workspace(ftm.ftm_slot_workspace_bytes(desc))
    ref = oracle.LRUState(E, S)
    rng = np.random.default_rng(E + S + S_new)
    order = rng.permutation(E)
    copy_stream = torch.cuda.Stream()
    n = 6                                                               # one token of k = 6 picks
    for _ in range(40):
        ids = _zipf_ids(rng, E, n, order)
        rc, _, _, _ = ref.update(ids)
        if rc != 0:                                                     # S = 4 < 6 distinct: skipped on both
            continue
        ftm.ftm_slot_lookup_update(desc, cache, torch.from_numpy(ids).cuda(), 1, ws.ptr, ws.nbytes, None,
                                   copy_stream)
    torch.cuda.synchronize()
    assert np.array_equal(eos.cpu().numpy(), ref.expert_of_slot)

    soe2, eos2, lu2, pool2 = _cache_arrays(E, S_new, bb)
    new = ftm.SlotCache(soe2.data_ptr(), eos2.data_ptr(), lu2.data_ptr(), 0, pool2.data_ptr(), host_pool.data_ptr(),
                        scratch.data_ptr(), 0, 0, 0, 0)
    ftm.ftm_slot_resize(desc, cache, S_new, new, ws.ptr, ws.nbytes, None)
    torch.cuda.synchronize()
    nref, move_from = ref.resize(S_new)
    assert np.array_equal(soe2.cpu().numpy(), nref.slot_of_expert)
    assert np.array_equal(eos2.cpu().numpy(), nref.expert_of_slot)
    assert np.array_equal(lu2.cpu().numpy(), nref.last_use)
    assert new.step == ref.step
    old_banks, new_banks = pool.view(S, bb), pool2.view(S_new, bb)
    for i, j in enumerate(move_from.tolist()):
        assert torch.equal(new_banks[i], old_banks[j]), (i, j)
    assert ftm.ftm_device_status(True) == 0

    # the resized cache keeps following the LRU rule
    desc2 = ftm.desc_for(cfg)
    desc2.S = S_new
    ws2 = Workspace(ftm.ftm_slot_workspace_bytes(desc2))
    for step in range(40):
        ids = _zipf_ids(rng, E, 6, order)                               # one token of k = 6 picks
        rc, misses, nd, nh = nref.update(ids)
        d_ids = torch.from_numpy(ids).cuda()
        if rc != 0:                                                     # more distinct experts than slots
            with pytest.raises(ftm.FtmError) as ei:
                ftm.ftm_slot_lookup_update(desc2, new, d_ids, 1, ws2.ptr, ws2.nbytes, None, copy_stream)
            assert ei.value.status == 3
            continue
        ftm.ftm_slot_lookup_update(desc2, new, d_ids, 1, ws2.ptr, ws2.nbytes, None, copy_stream)
        torch.cuda.synchronize()
        assert np.array_equal(soe2.cpu().numpy(), nref.slot_of_expert), step
        assert np.array_equal(eos2.cpu().numpy(), nref.expert_of_slot), step
        assert np.array_equal(lu2.cpu().numpy(), nref.last_use), step
        assert new.step == nref.step and new.last_misses == len(misses)
    banks = pool2.view(S_new, -1)[:, :4].contiguous().view(torch.int32).cpu().numpy()[:, 0]
    e_of_s = eos2.cpu().numpy()
    for s in range(S_new):
        if e_of_s[s] >= 0:
            assert banks[s] == e_of_s[s]


def test_layer_after_resize_matches_oracle():
    """A small FP8 slot-cache layer with a shared expert: run decode steps, shrink
    the pool, run more steps on the resized cache; outputs stay within the FP8 bar
    and the state follows the oracle."""
    # T = 2 tokens of k = 4 picks: at most 8 distinct experts, which fit both pools
    cfg = synth.scaled(synth.CONFIGS["284b_trace"], name="small_trace_resize", d=256, I=256, E=32, k=4, S=16,
                       T=(2,), trace_steps=24)
    T = cfg.T[0]
    dl = screened_layer(cfg, T, steps=cfg.trace_steps)
    Wr = oracle.bf16_to_f32(dl.layer.router_storage())
    b = dl.layer.bias()
    ref = oracle.LRUState(cfg.E, cfg.S)
    ws = Workspace(ftm.ftm_workspace_bytes(dl.desc, T))
    out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    copy_stream = torch.cuda.Stream()

    def step(desc, weights, cache, s, ref, ws):
        ftm.ftm_moe_layer_forward(desc, weights, cache, dl.hidden(T, step=s), T, out, ws.ptr, ws.nbytes, None,
                                  copy_stream)
        torch.cuda.synchronize()
        x = oracle.bf16_to_f32(dl.layer.hidden_storage(T, s))
        ids, g, _ = oracle.route(x, Wr, b, cfg.k)
        assert ref.update(ids)[0] == 0
        return x, ids, g

    for s in range(12):
        step(dl.desc, dl.weights(), dl.cache, s, ref, ws)
    S_new = 10
    bb = dl.bl.bank_bytes
    soe2, eos2, lu2, pool2 = _cache_arrays(cfg.E, S_new, bb)
    new = ftm.SlotCache(soe2.data_ptr(), eos2.data_ptr(), lu2.data_ptr(), 0, pool2.data_ptr(),
                        dl.host_pool.data_ptr(), dl.host_scratch.data_ptr(), 0, 0, 0, 0)
    ftm.ftm_slot_resize(dl.desc, dl.cache, S_new, new, ws.ptr, ws.nbytes, None)
    ref, _ = ref.resize(S_new)
    desc2 = ftm.desc_for(cfg)
    desc2.S = S_new
    ws2 = Workspace(ftm.ftm_workspace_bytes(desc2, T))
    w2 = ftm.LayerWeights(dl.w_router.data_ptr(), None if dl.bias is None else dl.bias.data_ptr(), pool2.data_ptr(),
                          soe2.data_ptr(), dl.shared_bank.data_ptr())
    for s in range(12, cfg.trace_steps):
        x, ids, g = step(desc2, w2, new, s, ref, ws2)
        assert np.array_equal(soe2.cpu().numpy(), ref.slot_of_expert), s
        assert np.array_equal(eos2.cpu().numpy(), ref.expert_of_slot), s
        assert np.array_equal(lu2.cpu().numpy(), ref.last_use), s
        rows = list(range(T))
        want = oracle.moe_rows(dl.layer, x, rows, ids, g)
        assert_rows_close(to_np_f32(out)[rows], want, TOL["fp8"], f"after resize, step {s}")
    assert ftm.ftm_device_status(True) == 0
