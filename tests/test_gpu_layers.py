"""Several layers over one shared slot cache with full-layer staging: layer
outputs against the oracle, the cache state against the oracle's staging
steps, banks in their slots, and the overlap switched off (with a warning)
when the cache cannot hold two whole layers."""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
from expert_offloaded_edge_b200.layout import pack_bank
import oracle
import synth
from synth.device import Workspace, to_device_storage
from tests.gpu_util import TOL, assert_rows_close, to_np_f32

pytestmark = pytest.mark.gpu

BASE = synth.scaled(synth.CONFIGS["35b_decode"], name="pipe", d=256, I=256, E=8, k=2, S=16, has_shared=1,
                    bias="uniform", T=(96,))


class Stack:
    """n layers of one shape, each with its own seed, staged through one cache."""

    def __init__(self, cfg, n, S, T):
        self.cfg, self.n, self.T = cfg, n, T
        self.desc = ftm.desc_for(synth.scaled(cfg, S=S))
        self.bl = ftm.ftm_get_bank_layout(self.desc)
        bb = self.bl.bank_bytes
        self.layers, self.x, self.w_router, self.bias, self.shared = [], [], [], [], []
        self.host_pool = torch.empty(n * cfg.E * bb, dtype=torch.uint8, pin_memory=True)
        hp = self.host_pool.numpy()
        for l in range(n):
            base = synth.Layer(cfg, seed=l)
            Wr, b = base.router_f32(), base.bias()
            table = synth.screen_hidden(base, T, 1, lambda xx: oracle.margin_ok(oracle.router_logits(xx, Wr, b),
                                                                                cfg.k, synth.MARGIN))
            layer = synth.Layer(cfg, seed=l, redraws=table)
            self.layers.append(layer)
            self.x.append(to_device_storage(layer.hidden_storage(T), cfg.act_dtype))
            self.w_router.append(to_device_storage(layer.router_storage(), cfg.act_dtype))
            self.bias.append(torch.from_numpy(b).cuda())
            self.shared.append(torch.from_numpy(pack_bank(self.desc, layer.expert(cfg.E), self.bl)).cuda())
            for e in range(cfg.E):
                k = l * cfg.E + e
                pack_bank(self.desc, layer.expert(e), self.bl, out=hp[k * bb:(k + 1) * bb])
        self.pool = torch.zeros(S * bb, dtype=torch.uint8, device="cuda")
        self.soe = torch.full((n * cfg.E,), -1, dtype=torch.int32, device="cuda")
        self.eos = torch.full((S,), -1, dtype=torch.int32, device="cuda")
        self.lu = torch.full((S,), -1, dtype=torch.int64, device="cuda")
        self.scratch = torch.zeros(ftm.ftm_slot_host_scratch_ints(self.desc), dtype=torch.int32, pin_memory=True)
        self.cache = ftm.SlotCache(self.soe.data_ptr(), self.eos.data_ptr(), self.lu.data_ptr(), 0,
                                   self.pool.data_ptr(), self.host_pool.data_ptr(), self.scratch.data_ptr(),
                                   0, 0, 0, 0, n * cfg.E, 0)
        self.weights = [ftm.LayerWeights(self.w_router[l].data_ptr(), self.bias[l].data_ptr(), None, None,
                                         self.shared[l].data_ptr()) for l in range(n)]
        self.ws = Workspace(ftm.ftm_workspace_bytes(self.desc, T))
        self.outs = [torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        self.copy_stream = torch.cuda.Stream()

    def run(self, overlap):
        used = ftm.ftm_moe_layers_forward(self.desc, self.weights, self.cache, self.x, self.T, self.outs, overlap,
                                          self.ws.ptr, self.ws.nbytes, None, self.copy_stream)
        torch.cuda.synchronize()
        assert ftm.ftm_device_status(True) == 0
        return used

    def check_outputs(self):
        for l in range(self.n):
            layer = self.layers[l]
            x = oracle.bf16_to_f32(layer.hidden_storage(self.T))
            Wr = oracle.bf16_to_f32(layer.router_storage())
            ids, g, _ = oracle.route(x, Wr, layer.bias(), self.cfg.k)
            want = oracle.moe_rows(layer, x, range(self.T), ids, g)
            assert_rows_close(to_np_f32(self.outs[l]), want, TOL["bf16"], f"layer {l}")

    def check_state(self, ref):
        assert self.cache.step == ref.step
        assert np.array_equal(self.soe.cpu().numpy(), ref.slot_of_expert)
        assert np.array_equal(self.eos.cpu().numpy(), ref.expert_of_slot)
        assert np.array_equal(self.lu.cpu().numpy(), ref.last_use)
        bb = self.bl.bank_bytes
        pool = self.pool.view(-1, bb).cpu()
        host = self.host_pool.view(-1, bb)
        for s, key in enumerate(self.eos.cpu().tolist()):
            if key >= 0:
                assert torch.equal(pool[s], host[key]), f"slot {s} does not hold the bank of key {key}"


def _replay(n, E, S, overlap_used, calls=1):
    ref = oracle.LRUState(n * E, S)
    for _ in range(calls):
        for l in range(n):
            rc = ref.stage_layer(l, E, overlap=overlap_used and l > 0)[0]
            assert rc == 0
    return ref


@pytest.mark.parametrize("S,overlap", [(16, True), (24, True), (16, False)])
def test_layers_staged_through_one_cache(S, overlap):
    st = Stack(BASE, 4, S, 96)
    used = st.run(overlap)
    assert used == overlap
    assert ftm.ftm_last_warning() == ""
    st.check_outputs()
    st.check_state(_replay(4, BASE.E, S, used))
    # a second pass continues from that state (some of layer 0's experts may
    # still be resident) and gives the same outputs
    first = [o.clone() for o in st.outs]
    st.run(overlap)
    assert all(torch.equal(a, b) for a, b in zip(first, st.outs))
    st.check_state(_replay(4, BASE.E, S, used, calls=2))


def test_overlap_off_when_two_layers_do_not_fit():
    st = Stack(BASE, 3, 12, 96)                        # 12 < 2 x 8 slots
    used = st.run(True)
    assert used is False
    assert "Disabling MoE prefill overlap" in ftm.ftm_last_warning()
    st.check_outputs()
    st.check_state(_replay(3, BASE.E, 12, False))


def test_overlap_and_serial_staging_give_identical_outputs():
    a = Stack(BASE, 3, 16, 200)
    b = Stack(BASE, 3, 16, 200)
    a.run(True)
    b.run(False)
    assert all(torch.equal(x, y) for x, y in zip(a.outs, b.outs))


def test_layers_forward_rejects_too_few_keys():
    st = Stack(BASE, 2, 16, 8)
    st.cache.n_keys = BASE.E                           # one layer's keys only
    with pytest.raises(ftm.FtmError) as ei:
        st.run(True)
    assert ei.value.status == 1
