"""The bandwidth-adaptive miss split (the pages' q* policy), on the CPU.

Oracle pins (orc_hybrid_split), from outside the oracle:
  - the hand-worked case of the docstring example below;
  - q against a brute-force search over every q' in [0, m] for the one that
    balances the two sides best (|q'(Bp + Bh) - m Bp| smallest, halves to the
    larger q');
  - the endpoints Bh = 0 (every miss over PCIe) and Bp = 0 (every miss on the
    host) and the invariants of the choice: host experts are misses, the host's
    (pairs, id) all precede the GPU misses', in that order.
Library against the oracle, no GPU needed: ftm_hybrid_split's q, and the
host expert FFN (ftm_host_expert_ffn) for every weight dtype (fp32, bf16, FP8,
NVFP4 with unit and non-unit activation global scales, MXFP4) against the
oracle's expert FFN in the same activation mode.
"""
import itertools

import numpy as np
import pytest

import expert_offloaded_edge_b200 as ftm
import oracle
import synth
from expert_offloaded_edge_b200.layout import pack_bank


def test_split_hand_worked():
    # experts 0..5 with 3, 0, 1, 2, 1, 5 pairs; expert 3 is cached.  Misses:
    # 0 (3 pairs), 2 (1), 4 (1), 5 (5): m = 4.  Bp = Bh: q = floor(2 + 0.5) = 2,
    # the host takes the two with the fewest pairs: 2 and 4 (1 pair each, the
    # lower id first).  Bp = 52.7, Bh = 77.3 (the pages' `ft bench bw` example):
    # 4 * 52.7 / 130 = 1.62 -> q = 2.  Bp = 3 Bh: 3 -> q = 3, host = [2].
    counts = np.array([3, 0, 1, 2, 1, 5])
    resident = np.array([0, 0, 0, 1, 0, 0])
    assert oracle.hybrid_split(counts, resident, 1.0, 1.0) == (4, 2, [2, 4])
    assert oracle.hybrid_split(counts, resident, 52.7, 77.3) == (4, 2, [2, 4])
    assert oracle.hybrid_split(counts, resident, 3.0, 1.0) == (4, 3, [2])
    # Bh = 0: all over PCIe; Bp = 0: all on the host, fewest pairs first
    assert oracle.hybrid_split(counts, resident, 1.0, 0.0) == (4, 4, [])
    assert oracle.hybrid_split(counts, resident, 0.0, 1.0) == (4, 0, [2, 4, 0, 5])


def _brute_q(m, bp, bh):
    best, bq = None, None
    for q in range(m + 1):
        dev = abs(q * (bp + bh) - m * bp)
        if best is None or dev < best - 1e-12 or (abs(dev - best) <= 1e-12 and q > bq):
            best, bq = dev, q
    return bq


def test_split_q_balances_the_two_sides_brute_force():
    rng = np.random.default_rng(1)
    for _ in range(400):
        E = int(rng.integers(1, 40))
        counts = rng.integers(0, 5, size=E)
        resident = rng.integers(0, 2, size=E)
        bp, bh = (float(v) for v in rng.uniform(0.0, 100.0, size=2))
        m, q, host = oracle.hybrid_split(counts, resident, bp, bh)
        assert m == int(np.sum((counts > 0) & (resident == 0)))
        assert q == _brute_q(m, bp, bh), (m, bp, bh, q)
        assert len(host) == m - q
        # the library's split takes the same decision in the same precision
        assert ftm.ftm_hybrid_split(m, bp, bh) == q


def test_split_choice_invariants_and_brute_force():
    rng = np.random.default_rng(2)
    for _ in range(200):
        E = int(rng.integers(1, 9))
        counts = rng.integers(0, 4, size=E)
        resident = rng.integers(0, 2, size=E)
        bp, bh = (float(v) for v in rng.uniform(0.0, 10.0, size=2))
        m, q, host = oracle.hybrid_split(counts, resident, bp, bh)
        misses = [e for e in range(E) if counts[e] > 0 and not resident[e]]
        assert set(host) <= set(misses) and len(set(host)) == len(host)
        gpu = [e for e in misses if e not in host]
        key = lambda e: (int(counts[e]), e)   # noqa: E731
        assert [key(e) for e in host] == sorted(key(e) for e in host)
        if host and gpu:
            assert max(key(e) for e in host) < min(key(e) for e in gpu)
        # brute force: of every subset of m - q misses, the host's has the fewest
        # pairs, and among those the smallest sorted id list
        best = min(itertools.combinations(misses, m - q), key=lambda c: (sum(int(counts[e]) for e in c), sorted(c)))
        assert sorted(host) == sorted(best)


def test_library_split_endpoints_and_errors():
    assert ftm.ftm_hybrid_split(7, 1.0, 0.0) == 7
    assert ftm.ftm_hybrid_split(7, 0.0, 1.0) == 0
    assert ftm.ftm_hybrid_split(0, 1.0, 1.0) == 0
    assert ftm.ftm_hybrid_split(5, 1.0, 1.0) == 3   # 2.5 rounds half up
    for bad in ((3, 0.0, 0.0), (3, -1.0, 1.0), (3, float("nan"), 1.0), (3, float("inf"), 1.0), (-1, 1.0, 1.0)):
        assert ftm.ftm_hybrid_split(*bad) == -1


def _aligned(nbytes, align=64):
    buf = np.zeros(nbytes + align, dtype=np.uint8)
    off = (-buf.ctypes.data) % align
    return buf[off:off + nbytes]


HOST_CFGS = {
    "f32": synth.scaled(synth.CONFIGS["tiny"], name="host_f32", d=128, I=128, E=4, k=2, S=4, has_shared=0),
    "bf16": synth.scaled(synth.CONFIGS["35b_decode"], name="host_bf16", d=256, I=128, E=4, k=2, S=4, has_shared=0),
    "fp8": synth.scaled(synth.CONFIGS["284b_trace"], name="host_fp8", d=256, I=256, E=4, k=2, S=4, has_shared=0,
                        lru=False, bias="uniform", T=(8,), trace_steps=1),
    "nvfp4": synth.scaled(synth.CONFIGS["753b_nvfp4"], name="host_nvfp4", d=256, I=512, E=4, k=2, S=4, has_shared=0,
                          T=(8,)),
    "mxfp4": synth.scaled(synth.CONFIGS["753b_mxfp4"], name="host_mxfp4", d=512, I=256, E=4, k=2, S=4, has_shared=0,
                          T=(8,)),
}
HOST_TOL = {"f32": 1e-4, "bf16": 2e-2, "fp8": 5e-2, "nvfp4": 5e-2, "mxfp4": 5e-2}


@pytest.mark.parametrize("wdtype,act_scale", [("f32", None), ("bf16", None), ("fp8", None), ("nvfp4", None),
                                              ("nvfp4", (0.5, 3.0)), ("mxfp4", None)])
@pytest.mark.parametrize("n", [1, 5])
def test_host_expert_ffn_matches_oracle(wdtype, act_scale, n):
    cfg = HOST_CFGS[wdtype]
    layer = synth.Layer(cfg, 0)
    desc = ftm.desc_for(cfg)
    bl = ftm.ftm_get_bank_layout(desc)
    e = 2
    bank = _aligned(bl.bank_bytes)
    pack_bank(desc, layer.expert(e), bl, out=bank)
    xs = layer.hidden_storage(n, 0)                  # bf16 bits, or fp32 for f32 layers
    x = np.ascontiguousarray(xs)
    y = np.zeros_like(x)
    nb = ftm.ftm_host_ffn_scratch_bytes(desc, n)
    scratch = _aligned(nb)
    gs = None if act_scale is None else np.array(act_scale, dtype=np.float32)
    ftm.ftm_host_expert_ffn(desc, bank, x, n, y, scratch, nb, threads=3, act_scale=gs)
    xf = x.astype(np.float32) if wdtype == "f32" else oracle.bf16_to_f32(x)
    yf = y.astype(np.float32) if wdtype == "f32" else oracle.bf16_to_f32(y)
    Wg, Wu, Wd = oracle.expert_weights_f32(layer, e)
    want = oracle.expert_ffn(xf, Wg, Wu, Wd, oracle.qa_mode(wdtype), act_scale)
    for r in range(n):
        err = float(np.max(np.abs(yf[r] - want[r])))
        scale = float(np.max(np.abs(want[r])))
        assert err <= HOST_TOL[wdtype] * scale, (wdtype, r, err, scale)
    if wdtype in ("fp8", "nvfp4", "mxfp4"):
        # the activation quantisation is applied: without it the result moves by
        # more than the host's distance to the quantised oracle
        plain = oracle.expert_ffn(xf, Wg, Wu, Wd, oracle.QA_NONE)
        assert np.abs(yf - want).max() < np.abs(plain - want).max()
    # the thread count does not change a value (each output element is one thread's sum)
    y1 = np.zeros_like(x)
    ftm.ftm_host_expert_ffn(desc, bank, x, n, y1, scratch, nb, threads=1, act_scale=gs)
    assert np.array_equal(y, y1)


def test_host_ffn_rejects_short_scratch_and_bad_bandwidths():
    cfg = HOST_CFGS["bf16"]
    desc = ftm.desc_for(cfg)
    nb = ftm.ftm_host_ffn_scratch_bytes(desc, 2)
    assert nb == 2 * (cfg.d + cfg.I) * 4
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_host_expert_ffn(desc, 64, 64, 2, 64, 64, nb - 1)
    assert ei.value.status == ftm.binding.FTM_ERR_INVALID_ARG
    # the layer entry point refuses fp32 layers (their SIMT GPU FFN computes
    # every row, the host's too) and bad bandwidths before any device call
    f32 = ftm.desc_for(HOST_CFGS["f32"])
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_moe_layer_forward_hybrid(f32, ftm.LayerWeights(16), ftm.SlotCache(), ftm.Hybrid(1.0, 1.0, 0), 16, 1,
                                         16, 16, 0, 1, 1)
    assert ei.value.status == ftm.binding.FTM_ERR_UNSUPPORTED
    h = ftm.Hybrid(0.0, 0.0, 0)
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_moe_layer_forward_hybrid(desc, ftm.LayerWeights(16), ftm.SlotCache(), h, 16, 1, 16, 16, 0, 1, 1)
    assert ei.value.status == ftm.binding.FTM_ERR_INVALID_ARG


def test_host_ffn_concurrent_callers_match_sequential_results():
    """The host FFN's thread pool is shared by the process: calls from several
    host threads at once (ctypes releases the GIL) must each get the result a
    call on its own gets."""
    import threading

    cfg = HOST_CFGS["fp8"]
    layer = synth.Layer(cfg, 0)
    desc = ftm.desc_for(cfg)
    bl = ftm.ftm_get_bank_layout(desc)
    n = 3
    jobs = []
    for e in range(4):
        bank = _aligned(bl.bank_bytes)
        pack_bank(desc, layer.expert(e), bl, out=bank)
        x = np.ascontiguousarray(layer.hidden_storage(n, e))
        nb = ftm.ftm_host_ffn_scratch_bytes(desc, n)
        want = np.zeros_like(x)
        ftm.ftm_host_expert_ffn(desc, bank, x, n, want, _aligned(nb), nb, threads=4)
        jobs.append((bank, x, want, nb))
    errors = []

    def worker(j):
        bank, x, want, nb = jobs[j % 4]
        for _ in range(5):
            y = np.zeros_like(x)
            ftm.ftm_host_expert_ffn(desc, bank, x, n, y, _aligned(nb), nb, threads=4)
            if not np.array_equal(y, want):
                errors.append(j)

    threads = [threading.Thread(target=worker, args=(j,)) for j in range(8)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors


def test_split_workspace_queries():
    for name in ("284b_trace", "35b_decode", "753b_nvfp4"):
        desc = ftm.desc_for(synth.CONFIGS[name])
        prev_d = prev_h = 0
        for T in (1, 16, 64, 512):
            wd = ftm.ftm_hybrid_workspace_bytes(desc, T)
            wh = ftm.ftm_hybrid_host_bytes(desc, T)
            assert wd >= ftm.ftm_workspace_bytes(desc, T) > 0
            assert wd >= prev_d and wh > prev_h
            # the host FFN scratch for every pair is part of the host buffer
            assert wh >= ftm.ftm_host_ffn_scratch_bytes(desc, T * desc.k)
            prev_d, prev_h = wd, wh
    bad = ftm.LayerDesc(100, 8, 2, 128, 0, 8, ftm.FTM_BF16, 0)   # d not a multiple of 128
    assert ftm.ftm_hybrid_workspace_bytes(bad, 16) == 0 and ftm.ftm_hybrid_host_bytes(bad, 16) == 0
    assert ftm.ftm_host_ffn_scratch_bytes(bad, 4) == 0
