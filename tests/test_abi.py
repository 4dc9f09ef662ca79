"""CPU checks of the C ABI: the library loads, exports every symbol the header
declares, and rejects out-of-contract arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np

import pytest

import expert_offloaded_edge_b200 as ftm
import synth

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ftm.h")


def declared_symbols():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ftm_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 14
    lib = ftm.library()
    for n in names:
        assert hasattr(lib, n), n


def test_bank_layouts():
    want = {
        "tiny": 3 * 256 * 512 * 4,
        "35b_decode": 3 * 2048 * 768 * 2,
        "284b_trace": 3 * 4096 * 2048 + (2 * 2048 // 128) * (4096 // 128) * 4 + (4096 // 128) * (2048 // 128) * 4,
        "753b_nvfp4": 3 * 6144 * 2048 // 2 + 3 * 6144 * 2048 // 16 + 256,
    }
    for name, nbytes in want.items():
        bl = ftm.ftm_get_bank_layout(ftm.desc_for(synth.CONFIGS[name]))
        assert bl.bank_bytes % 256 == 0
        assert nbytes <= bl.bank_bytes < nbytes + 5 * 256, name
        assert bl.w_gu_off == 0 and bl.w_d_off >= bl.w_gu_bytes
    bl = ftm.ftm_get_bank_layout(ftm.desc_for(synth.CONFIGS["284b_trace"]))
    assert bl.bank_bytes == 25171968           # 25.17 MB per FP8 expert incl. 6,144 B of block scales
    mx = ftm.ftm_get_bank_layout(ftm.desc_for(synth.CONFIGS["753b_mxfp4"]))
    d, I = 6144, 2048
    assert (mx.w_gu_bytes, mx.w_d_bytes, mx.s_gu_bytes, mx.s_d_bytes, mx.s_t_bytes) == \
        (2 * I * d // 2, d * I // 2, 2 * I * d // 32, d * I // 32, 0)


@pytest.mark.parametrize("field,value", [("d", 100), ("d", 0), ("I", 96), ("k", 0), ("k", 9), ("E", 0),
                                         ("E", 600), ("S", 0), ("wdtype", 7), ("reserved", 1), ("has_shared", 2)])
def test_invalid_desc_rejected_without_gpu(field, value):
    d = ftm.desc_for(synth.CONFIGS["35b_decode"])
    if field == "k" and value == 9:
        d.E = 8
    setattr(d, field, value)
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_get_bank_layout(d)
    assert ei.value.status == 1
    assert ftm.ftm_last_error()


def test_invalid_calls_rejected_without_gpu():
    d = ftm.desc_for(synth.CONFIGS["35b_decode"])
    lib = ftm.library()
    assert lib.ftm_route(None, None, 1, None, None, None, None, None) == 1
    assert lib.ftm_route(ctypes.byref(d), None, -1, None, None, None, None, None) == 1
    assert lib.ftm_route(ctypes.byref(d), None, 4, None, None, None, None, None) == 1
    assert lib.ftm_route(ctypes.byref(d), None, 0, None, None, None, None, None) == 0      # T = 0: no-op
    # workspace too small / misaligned
    assert lib.ftm_permute(ctypes.byref(d), 16, 9000, 16, 16, 16, 16, None, 0, None) == 1
    assert lib.ftm_moe_layer_forward(ctypes.byref(d), None, None, None, 4, None, None, 0, None, None) == 1
    assert lib.ftm_combine(ctypes.byref(d), None, None, None, 3, None, None) == 1
    assert "NULL" in ftm.ftm_last_error()


def test_workspace_sizes_monotone():
    for name in synth.CONFIGS:
        d = ftm.desc_for(synth.CONFIGS[name])
        sizes = [ftm.ftm_workspace_bytes(d, T) for T in (0, 1, 16, 1024, 16384)]
        assert sizes == sorted(sizes) and sizes[1] > 0
        assert ftm.ftm_ffn_workspace_bytes(d, 16) <= ftm.ftm_workspace_bytes(d, 16)


def test_nvfp4_scale_chunk_packing_brute_force():
    from expert_offloaded_edge_b200.layout import nvfp4_scale_chunks
    rng = np.random.default_rng(0)
    R, G16 = 256, 24
    s16 = rng.integers(0, 256, size=(R, G16), dtype=np.uint8)
    packed = nvfp4_scale_chunks(s16)
    assert packed.size == s16.size
    for r in range(R):
        for g in range(G16):
            rb, kb, rl, j = r // 128, g // 4, r % 128, g % 4
            off = (rb * (G16 // 4) + kb) * 512 + (rl % 32) * 16 + (rl // 32) * 4 + j
            assert packed[off] == s16[r, g]


def test_gate_up_paired_rows_brute_force():
    from expert_offloaded_edge_b200.layout import gate_up_paired_rows
    rng = np.random.default_rng(1)
    I, C = 192, 5
    gate = rng.integers(0, 256, size=(I, C), dtype=np.uint8)
    up = rng.integers(0, 256, size=(I, C), dtype=np.uint8)
    paired = gate_up_paired_rows(gate, up)
    assert paired.shape == (2 * I, C)
    for r in range(2 * I):
        b, rl = r // 128, r % 128
        want = gate[64 * b + rl] if rl < 64 else up[64 * b + rl - 64]
        assert (paired[r] == want).all()


def test_slot_resize_rejected_without_gpu():
    cfg = synth.CONFIGS["284b_trace"]
    d = ftm.desc_for(cfg)
    bb = ftm.ftm_get_bank_layout(d).bank_bytes
    lib = ftm.library()
    # fake, never dereferenced device addresses: the checks fail before any launch
    old = ftm.SlotCache(0x100000, 0x200000, 0x300000, 7, 0x10_0000_0000, 0x4000_0000, 0x5000_0000, 0, 0, 0, 0)
    new_pool = 0x10_0000_0000 + bb * cfg.S          # right after the old pool: no overlap
    new = ftm.SlotCache(0x600000, 0x700000, 0x800000, 0, new_pool, 0x4000_0000, 0x5000_0000, 0, 0, 0, 0)
    ws = 0x9000_0000
    nbytes = ftm.ftm_slot_workspace_bytes(d)
    assert lib.ftm_slot_resize(None, ctypes.byref(old), 8, ctypes.byref(new), ws, nbytes, None) == 1
    assert lib.ftm_slot_resize(ctypes.byref(d), ctypes.byref(old), 0, ctypes.byref(new), ws, nbytes, None) == 1
    assert lib.ftm_slot_resize(ctypes.byref(d), ctypes.byref(old), 5000, ctypes.byref(new), ws, nbytes, None) == 2
    bad = ftm.SlotCache(0x600000, 0x700000, 0x800000, 0, 0x10_0000_0000 + bb, 0, 0, 0, 0, 0, 0)  # overlaps
    assert lib.ftm_slot_resize(ctypes.byref(d), ctypes.byref(old), 8, ctypes.byref(bad), ws, nbytes, None) == 1
    assert "overlap" in ftm.ftm_last_error()
    same = ftm.SlotCache(0x100000, 0x700000, 0x800000, 0, new_pool, 0, 0, 0, 0, 0, 0)            # shared state array
    assert lib.ftm_slot_resize(ctypes.byref(d), ctypes.byref(old), 8, ctypes.byref(same), ws, nbytes, None) == 1
    assert lib.ftm_slot_resize(ctypes.byref(d), ctypes.byref(old), 8, ctypes.byref(new), ws, nbytes - 8, None) == 1
    assert lib.ftm_slot_resize(ctypes.byref(d), ctypes.byref(old), 8, ctypes.byref(new), None, nbytes, None) == 1


def _layers_call(S, overlap, n_layers=3, n_keys=None, T=0):
    """ftm_moe_layers_forward on fake, never dereferenced addresses: at T = 0 the
    call validates, settles the overlap rule and returns before any launch."""
    cfg = synth.scaled(synth.CONFIGS["35b_decode"], S=S, E=8, k=2, d=256, I=256)
    d = ftm.desc_for(cfg)
    lib = ftm.library()
    cache = ftm.SlotCache(0x100000, 0x200000, 0x300000, 0, 0x10_0000_0000, 0x4000_0000, 0x5000_0000, 0, 0, 0, 0,
                          n_layers * cfg.E if n_keys is None else n_keys, 0)
    W = (ftm.LayerWeights * n_layers)(*[ftm.LayerWeights(0x7000_0000, None, None, None, None)
                                        for _ in range(n_layers)])
    X = (ctypes.c_void_p * n_layers)(*[0x8000_0000] * n_layers)
    O = (ctypes.c_void_p * n_layers)(*[0x9000_0000] * n_layers)
    used = ctypes.c_int32(-1)
    ws = np.zeros(ftm.ftm_workspace_bytes(d, T) + 512, dtype=np.uint8)
    wp = ws.ctypes.data + (-ws.ctypes.data) % 256
    st = lib.ftm_moe_layers_forward(ctypes.byref(d), n_layers, W, ctypes.byref(cache), X, T, O, int(overlap),
                                    ctypes.byref(used), wp, ws.nbytes - 256, None, None)
    return st, used.value


def test_layers_overlap_rule_without_gpu():
    # the copy/compute overlap needs room for two whole layers of experts (S >= 2E)
    st, used = _layers_call(S=16, overlap=True)
    assert st == 0 and used == 1 and ftm.ftm_last_warning() == ""
    st, used = _layers_call(S=15, overlap=True)
    assert st == 0 and used == 0
    w = ftm.ftm_last_warning()
    assert w.startswith("WARNING Disabling MoE prefill overlap") and "two whole layers" in w
    st, used = _layers_call(S=40, overlap=False)
    assert st == 0 and used == 0 and ftm.ftm_last_warning() == ""


def test_layers_rejected_without_gpu():
    st, _ = _layers_call(S=16, overlap=True, n_keys=8)             # 3 layers x 8 experts need 24 keys
    assert st == 1 and "keys" in ftm.ftm_last_error()
    st, _ = _layers_call(S=16, overlap=True, n_layers=0)
    assert st == 1
