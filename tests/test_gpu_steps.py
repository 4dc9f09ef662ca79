"""Per-step parity of the CUDA kernels (through the C ABI) with the oracle:
routing ids / permutation / slot state bit-exact, gates within 1e-5."""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from tests.gpu_util import Workspace, gate_rtol, oracle_route, screened_layer

pytestmark = pytest.mark.gpu


def _route_case(cfg, T):
    dl = screened_layer(cfg, T)
    x = dl.hidden(T)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    ftm.ftm_route(dl.desc, x, T, dl.w_router, dl.bias, ids, gw)
    torch.cuda.synchronize()
    _, rid, rg = oracle_route(dl, T)
    return ids.cpu().numpy(), gw.cpu().numpy(), rid, rg


@pytest.mark.parametrize("name,T", [("tiny", 16), ("35b_decode", 1), ("35b_decode", 8), ("35b_decode", 64)])
def test_route_configs(name, T):
    ids, gw, rid, rg = _route_case(synth.CONFIGS[name], T)
    assert np.array_equal(ids, rid)
    assert np.allclose(gw, rg, rtol=gate_rtol(synth.CONFIGS[name].d), atol=1e-6)


@pytest.mark.parametrize("E,k,d,T,dt", [(37, 1, 128, 5, "bf16"), (16, 16, 128, 3, "bf16"), (300, 7, 256, 33, "bf16"),
                                        (8, 8, 128, 9, "f32"), (512, 16, 128, 17, "bf16"), (1, 1, 128, 4, "f32"),
                                        # cluster router at medium batches
                                        (120, 4, 256, 300, "bf16"), (200, 6, 128, 333, "bf16"),
                                        # tensor-core router (T >= 2048): 128-token tiles, experts on the
                                        # MMA N side padded to 16 (N = 48 .. 256), ragged last tiles, k = 16
                                        (37, 3, 128, 2049, "bf16"), (120, 4, 256, 2100, "bf16"),
                                        (200, 6, 128, 2500, "bf16"), (256, 16, 256, 3000, "bf16"),
                                        (128, 8, 256, 10000, "bf16"), (160, 8, 256, 9601, "bf16"),
                                        (64, 2, 128, 2048, "bf16"), (96, 1, 128, 2100, "bf16")])
def test_route_shapes(E, k, d, T, dt):
    cfg = synth.LayerConfig("route_case", d=d, E=E, k=k, I=128, wdtype=dt, has_shared=0, S=E, bias="uniform", T=(T,))
    ids, gw, rid, rg = _route_case(cfg, T)
    assert np.array_equal(ids, rid)
    assert np.allclose(gw, rg, rtol=gate_rtol(d), atol=1e-6)
    assert np.allclose(gw.sum(1), 1.0, atol=1e-5)


@pytest.mark.parametrize("k", [1, 2, 5, 8, 16])
def test_route_tc_ties(k):
    """Tensor-core router on exact ties: zero tokens make every logit its bias, which repeats in threes, so
    each pick list must order equal logits by ascending expert id like the oracle; the other tokens are
    random.  k = 2 and 8 take the single-scan selection, 1, 5 and 16 the pass-based one."""
    T, E, d = 2048, 64, 128
    rng = np.random.default_rng(40 + k)
    x = rng.standard_normal((T, d)).astype(np.float32)
    x[: T // 2] = 0.0
    wr = (0.02 * rng.standard_normal((E, d))).astype(np.float32)
    bias = np.ascontiguousarray(0.5 * ((E - 1 - np.arange(E)) // 3), dtype=np.float32)   # 0 alone, then threes
    xb = torch.from_numpy(x).to(torch.bfloat16).cuda()
    wb = torch.from_numpy(wr).to(torch.bfloat16).cuda()
    cfg = synth.LayerConfig("route_ties", d=d, E=E, k=k, I=128, wdtype="bf16", has_shared=0, S=E, bias="uniform",
                            T=(T,))
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ftm.ftm_route(ftm.desc_for(cfg), xb, T, wb, torch.from_numpy(bias).cuda(), ids, gw)
    torch.cuda.synchronize()
    rid, rg, _ = oracle.route(xb.float().cpu().numpy(), wb.float().cpu().numpy(), bias, k)
    assert np.array_equal(ids.cpu().numpy()[: T // 2], rid[: T // 2])
    assert (ids.cpu().numpy()[: T // 2, 0] == 0).all()
    assert np.allclose(gw.cpu().numpy(), rg, rtol=gate_rtol(d), atol=1e-6)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (5, 2, 8), (64, 8, 128), (37, 3, 300), (600, 8, 128),
                                   (9000, 8, 128), (16384, 8, 160), (2000, 6, 512)])
def test_permute_bit_exact(T, k, E):
    rng = np.random.default_rng(T + 7 * E)
    # skewed expert popularity, some experts empty
    p = rng.dirichlet(np.full(E, 0.3))
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    desc = ftm.LayerDesc(128, E, k, 128, 0, E, ftm.FTM_BF16, 0)
    P = T * k
    d_ids = torch.from_numpy(ids).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(P, dtype=torch.int32, device="cuda")
    inv = torch.empty(P, dtype=torch.int32, device="cuda")
    ws = Workspace(ftm.ftm_permute_workspace_bytes(desc, T))
    ftm.ftm_permute(desc, d_ids, T, counts, offsets, perm, inv, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    rc, ro, rp, ri = oracle.permute(ids, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    assert np.array_equal(inv.cpu().numpy(), ri)


def test_permute_empty():
    desc = ftm.LayerDesc(128, 8, 2, 128, 0, 8, ftm.FTM_BF16, 0)
    counts = torch.full((8,), 7, dtype=torch.int32, device="cuda")
    offsets = torch.full((9,), 7, dtype=torch.int32, device="cuda")
    ftm.ftm_permute(desc, None, 0, counts, offsets, None, None, None, 0)
    torch.cuda.synchronize()
    assert counts.cpu().tolist() == [0] * 8 and offsets.cpu().tolist() == [0] * 9


def _lru_setup(E, S):
    cfg = synth.LayerConfig("lru_case", d=128, E=E, k=6, I=128, wdtype="bf16", has_shared=0, S=S, bias="zipf",
                            T=(32,), lru=True)
    desc = ftm.desc_for(cfg)
    bl = ftm.ftm_get_bank_layout(desc)
    host_pool = torch.empty(E * bl.bank_bytes, dtype=torch.uint8, pin_memory=True)
    host_pool.copy_(torch.arange(E, dtype=torch.int32).repeat_interleave(bl.bank_bytes // 4).view(torch.uint8))
    pool = torch.zeros(S * bl.bank_bytes, dtype=torch.uint8, device="cuda")
    soe = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    eos = torch.full((S,), -1, dtype=torch.int32, device="cuda")
    lu = torch.full((S,), -1, dtype=torch.int64, device="cuda")
    scratch = torch.zeros(ftm.ftm_slot_host_scratch_ints(desc), dtype=torch.int32, pin_memory=True)
    cache = ftm.SlotCache(soe.data_ptr(), eos.data_ptr(), lu.data_ptr(), 0, pool.data_ptr(), host_pool.data_ptr(),
                          scratch.data_ptr(), 0, 0, 0, 0)
    ws = Workspace(ftm.ftm_slot_workspace_bytes(desc))
    return desc, bl, cache, (soe, eos, lu, pool), ws


@pytest.mark.parametrize("E,S,n", [(256, 64, 32 * 6), (16, 4, 6), (100, 100, 42)])
def test_lru_trace_bit_exact(E, S, n):
    desc, bl, cache, (soe, eos, lu, pool), ws = _lru_setup(E, S)
    ref = oracle.LRUState(E, S)
    rng = np.random.default_rng(E + S)
    z = 1.0 / np.arange(1, E + 1) ** 1.1
    z /= z.sum()
    order = rng.permutation(E)
    copy_stream = torch.cuda.Stream()
    for step in range(60):
        ids = order[rng.choice(E, size=n, p=z)].astype(np.int32)
        d_ids = torch.from_numpy(ids).cuda()
        rc, misses, nd, nh = ref.update(ids)
        # the n ids are T = n/k tokens of k picks
        if rc != 0:
            with pytest.raises(ftm.FtmError) as ei:
                ftm.ftm_slot_lookup_update(desc, cache, d_ids, n // desc.k, ws.ptr, ws.nbytes, None, copy_stream)
            assert ei.value.status == 3
            continue
        ftm.ftm_slot_lookup_update(desc, cache, d_ids, n // desc.k, ws.ptr, ws.nbytes, None, copy_stream)
        torch.cuda.synchronize()
        assert np.array_equal(soe.cpu().numpy(), ref.slot_of_expert), step
        assert np.array_equal(eos.cpu().numpy(), ref.expert_of_slot), step
        assert np.array_equal(lu.cpu().numpy(), ref.last_use), step
        assert cache.step == ref.step and cache.last_misses == len(misses) and cache.last_hits == nh
    # every resident slot holds the bytes of its expert (banks were filled with the expert id)
    banks = pool.view(S, -1)[:, :4].contiguous().view(torch.int32).cpu().numpy()[:, 0]
    e_of_s = eos.cpu().numpy()
    for s in range(S):
        if e_of_s[s] >= 0:
            assert banks[s] == e_of_s[s]


def test_lru_capacity_and_rollback():
    E, S = 16, 4
    desc, bl, cache, (soe, eos, lu, pool), ws = _lru_setup(E, S)
    copy_stream = torch.cuda.Stream()
    ids = torch.tensor([[0, 1, 2, 3, 4, 5]], dtype=torch.int32, device="cuda")   # 6 distinct > 4 slots
    before = (soe.clone(), eos.clone(), lu.clone())
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_slot_lookup_update(desc, cache, ids, 1, ws.ptr, ws.nbytes, None, copy_stream)
    assert ei.value.status == 3
    assert all(torch.equal(a, b) for a, b in zip(before, (soe, eos, lu))) and cache.step == 0
    ok_ids = torch.tensor([[0, 1, 2, 0, 1, 2]], dtype=torch.int32, device="cuda")
    ftm.ftm_slot_lookup_update(desc, cache, ok_ids, 1, ws.ptr, ws.nbytes, None, copy_stream)
    torch.cuda.synchronize()
    snap = (soe.clone(), eos.clone(), lu.clone())
    cache.fail_before_copy = 1
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_slot_lookup_update(desc, cache, torch.tensor([[7, 8, 0, 7, 8, 0]], dtype=torch.int32, device="cuda"),
                                   1, ws.ptr, ws.nbytes, None, copy_stream)
    assert ei.value.status == 4
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(snap, (soe, eos, lu))) and cache.step == 1


def test_combine_hand_example():
    desc = ftm.LayerDesc(128, 4, 2, 128, 1, 4, ftm.FTM_F32, 0)
    T, k, d = 2, 2, 128
    y = torch.arange((T * k + T) * d, dtype=torch.float32, device="cuda").view(T * k + T, d) / 100
    inv = torch.tensor([3, 0, 1, 2], dtype=torch.int32, device="cuda")
    gw = torch.tensor([[0.25, 0.75], [0.5, 0.5]], dtype=torch.float32, device="cuda")
    out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ftm.ftm_combine(desc, y, inv, gw, T, out)
    torch.cuda.synchronize()
    yc = y.cpu().numpy().astype(np.float64)
    want = np.stack([0.25 * yc[3] + 0.75 * yc[0] + yc[4], 0.5 * yc[1] + 0.5 * yc[2] + yc[5]])
    assert np.allclose(out.cpu().numpy(), want, rtol=1e-6)


def test_lru_rollback_after_partial_copies():
    """A copy failure after some copies were issued: slots whose copy was issued
    come back empty with their old experts unmapped; everything else is rolled
    back; the cache keeps working from that state like the oracle's LRU."""
    E, S = 16, 4
    desc, bl, cache, (soe, eos, lu, pool), ws = _lru_setup(E, S)
    copy_stream = torch.cuda.Stream()

    def step(ids):
        t = torch.tensor([ids], dtype=torch.int32, device="cuda")
        ftm.ftm_slot_lookup_update(desc, cache, t, 1, ws.ptr, ws.nbytes, None, copy_stream)

    desc.k = 2
    step([0, 1])
    step([2, 3])           # slots 0..3 hold experts 0..3, last_use 0, 0, 1, 1
    step([0, 1])           # slots 0, 1 used again at step 2
    torch.cuda.synchronize()
    assert eos.cpu().tolist() == [0, 1, 2, 3] and lu.cpu().tolist() == [2, 2, 1, 1]
    # step 3 misses 7 and 8: victims in (last_use, slot) order are slots 2 and 3;
    # the second copy fails, after the first (7 -> slot 2) was issued
    cache.fail_before_copy = 2
    with pytest.raises(ftm.FtmError) as ei:
        step([7, 8])
    assert ei.value.status == 4 and cache.fail_before_copy == 0
    torch.cuda.synchronize()
    assert cache.step == 3
    assert eos.cpu().tolist() == [0, 1, -1, 3]             # slot 2 may hold part of bank 7: empty
    assert lu.cpu().tolist() == [2, 2, -1, 1]
    want_soe = [-1] * E
    want_soe[0], want_soe[1], want_soe[3] = 0, 1, 3         # expert 2 unmapped; 7 never mapped
    assert soe.cpu().tolist() == want_soe
    banks = pool.view(S, -1)[:, :4].contiguous().view(torch.int32).cpu().numpy()[:, 0]
    assert banks[0] == 0 and banks[1] == 1 and banks[3] == 3  # untouched slots keep their banks
    # later steps behave like the oracle's LRU started from the rolled-back state
    ref = oracle.LRUState(E, S)
    ref.slot_of_expert[:] = want_soe
    ref.expert_of_slot[:] = [0, 1, -1, 3]
    ref.last_use[:] = [2, 2, -1, 1]
    ref.step = 3
    for ids in ([7, 8], [2, 7], [9, 0], [3, 2]):
        ref.update(np.array(ids, np.int32))
        step(ids)
        torch.cuda.synchronize()
        assert soe.cpu().tolist() == ref.slot_of_expert.tolist()
        assert eos.cpu().tolist() == ref.expert_of_slot.tolist()
        assert lu.cpu().tolist() == ref.last_use.tolist()
    banks = pool.view(S, -1)[:, :4].contiguous().view(torch.int32).cpu().numpy()[:, 0]
    for s, e in enumerate(eos.cpu().tolist()):
        if e >= 0:
            assert banks[s] == e


def test_lru_rejects_out_of_range_ids():
    E, S = 16, 4
    desc, bl, cache, (soe, eos, lu, pool), ws = _lru_setup(E, S)
    desc.k = 2
    copy_stream = torch.cuda.Stream()
    assert ftm.ftm_device_status(True) == 0
    before = (soe.clone(), eos.clone(), lu.clone())
    for bad in (E, -1):
        t = torch.tensor([[1, bad]], dtype=torch.int32, device="cuda")
        with pytest.raises(ftm.FtmError) as ei:
            ftm.ftm_slot_lookup_update(desc, cache, t, 1, ws.ptr, ws.nbytes, None, copy_stream)
        assert ei.value.status == 1 and cache.step == 0
        assert all(torch.equal(a, b) for a, b in zip(before, (soe, eos, lu)))
        assert ftm.ftm_device_status(True) == 2


@pytest.mark.parametrize("T", [40, 700])     # one-block and three-pass permutation
def test_permute_skips_out_of_range_ids(T):
    E, k = 12, 3
    rng = np.random.default_rng(T)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    ids[3, 1] = E
    ids[T - 1, 0] = -5
    desc = ftm.LayerDesc(128, E, k, 128, 0, E, ftm.FTM_BF16, 0)
    P = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((P,), 123, dtype=torch.int32, device="cuda")
    inv = torch.full((P,), 123, dtype=torch.int32, device="cuda")
    ws = Workspace(ftm.ftm_permute_workspace_bytes(desc, T))
    assert ftm.ftm_device_status(True) == 0
    ftm.ftm_permute(desc, torch.from_numpy(ids).cuda(), T, counts, offsets, perm, inv, ws.ptr, ws.nbytes)
    torch.cuda.synchronize()
    assert ftm.ftm_device_status(True) == 2
    flat = ids.ravel()
    ok = (flat >= 0) & (flat < E)
    want_counts = np.bincount(flat[ok], minlength=E)
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    assert np.array_equal(offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(want_counts)]))
    order = sorted(np.nonzero(ok)[0].tolist(), key=lambda q: (flat[q], q))
    pm, iv = perm.cpu().numpy(), inv.cpu().numpy()
    assert pm[:len(order)].tolist() == order and (pm[len(order):] == -1).all()
    assert (iv[~ok] == -1).all() and all(iv[q] == pos for pos, q in enumerate(order))


def test_combine_skips_unplaced_pairs():
    desc = ftm.LayerDesc(128, 4, 2, 128, 0, 4, ftm.FTM_F32, 0)
    T, k, d = 2, 2, 128
    y = torch.arange(T * k * d, dtype=torch.float32, device="cuda").view(T * k, d) / 100
    inv = torch.tensor([3, -1, 1, 2], dtype=torch.int32, device="cuda")
    gw = torch.tensor([[0.25, 0.75], [0.5, 0.5]], dtype=torch.float32, device="cuda")
    out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    assert ftm.ftm_device_status(True) == 0
    ftm.ftm_combine(desc, y, inv, gw, T, out)
    torch.cuda.synchronize()
    assert ftm.ftm_device_status(True) == 2
    yc = y.cpu().numpy().astype(np.float64)
    want = np.stack([0.25 * yc[3], 0.5 * yc[1] + 0.5 * yc[2]])
    assert np.allclose(out.cpu().numpy(), want, rtol=1e-6)


def test_bounded_wait_gives_up_and_context_survives():
    """A wait on a barrier that nothing completes gives up after its limit, reports status 1 (timeout), and
    the context stays usable: a layer computed afterwards still matches the oracle."""
    ftm.ftm_device_status(True)
    assert ftm.ftm_selftest_bounded_wait() == 1
    assert ftm.ftm_device_status(True) == 0
    cfg = synth.CONFIGS["tiny"]
    ids, gw, rid, rg = _route_case(cfg, 16)
    assert np.array_equal(ids, rid)
    assert ftm.ftm_device_status(True) == 0
