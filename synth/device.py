"""Stage a synthetic layer on the GPU in the library's layout (tests, bench, smoke).

Uploads the generator's weights and hidden states; no layer arithmetic here.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

import expert_offloaded_edge_b200 as ftm
from expert_offloaded_edge_b200.layout import pack_bank

from . import Layer, LayerConfig, load_redraws


def to_device_storage(arr: np.ndarray, act_dtype: str, device="cuda") -> torch.Tensor:
    """fp32 arrays stay fp32; bf16 bit patterns (uint16) become torch.bfloat16."""
    if act_dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


class DeviceLayer:
    """Weights of one synthetic layer on the device.

    Resident layers (lru=False): every expert e lives in slot slot_of_expert[e]
    of a device pool of S banks.  Cache layers (lru=True): all E banks live in a
    pinned host pool and the device pool of S slots starts empty."""

    def __init__(self, cfg: LayerConfig, seed: int = 0, device: str = "cuda", T_redraw: Optional[int] = None,
                 redraws=None, slot_perm: Optional[np.ndarray] = None, banks: Optional[np.ndarray] = None):
        """banks: optional [E + has_shared][bank_bytes] uint8, the packed banks of
        this layer (row E = the shared expert), e.g. from pack_banks() saved
        earlier; when absent they are drawn and packed here."""
        self.cfg = cfg
        self.device = device
        if redraws is None:
            redraws = load_redraws(cfg.name, T_redraw or max(cfg.T)) or {}
        self.layer = Layer(cfg, seed, redraws)
        self.desc = ftm.desc_for(cfg)
        self.bl = ftm.ftm_get_bank_layout(self.desc)
        bb = self.bl.bank_bytes
        L = self.layer
        if banks is not None:
            assert banks.shape == (cfg.E + cfg.has_shared, bb), banks.shape

        def bank(e):
            return banks[e] if banks is not None else pack_bank(self.desc, L.expert(e), self.bl)

        self.w_router = to_device_storage(L.router_storage(), cfg.act_dtype, device)
        b = L.bias()
        self.bias = None if b is None else torch.from_numpy(b).to(device)
        self.shared_bank = None
        if cfg.has_shared:
            self.shared_bank = torch.from_numpy(np.ascontiguousarray(bank(cfg.E))).to(device)
        if cfg.lru:
            self.host_pool = torch.empty(cfg.E * bb, dtype=torch.uint8, pin_memory=True)
            hp = self.host_pool.numpy()
            for e in range(cfg.E):
                if banks is not None:
                    hp[e * bb:(e + 1) * bb] = banks[e]
                else:
                    pack_bank(self.desc, L.expert(e), self.bl, out=hp[e * bb:(e + 1) * bb])
            self.pool = torch.zeros(cfg.S * bb, dtype=torch.uint8, device=device)
            self.slot_of_expert_np = None
            self.slot_of_expert = torch.full((cfg.E,), -1, dtype=torch.int32, device=device)
            self.expert_of_slot = torch.full((cfg.S,), -1, dtype=torch.int32, device=device)
            self.last_use = torch.full((cfg.S,), -1, dtype=torch.int64, device=device)
            self.host_scratch = torch.zeros(ftm.ftm_slot_host_scratch_ints(self.desc), dtype=torch.int32,
                                            pin_memory=True)
            self.cache = ftm.SlotCache(self.slot_of_expert.data_ptr(), self.expert_of_slot.data_ptr(),
                                       self.last_use.data_ptr(), 0, self.pool.data_ptr(), self.host_pool.data_ptr(),
                                       self.host_scratch.data_ptr(), 0, 0, 0, 0)
        else:
            assert cfg.S >= cfg.E
            soe = L.slot_of_expert() if slot_perm is None else slot_perm
            self.slot_of_expert_np = soe.astype(np.int32)
            self.slot_of_expert = torch.from_numpy(self.slot_of_expert_np).to(device)
            self.pool = torch.zeros(cfg.S * bb, dtype=torch.uint8, device=device)
            for e in range(cfg.E):
                s = int(soe[e])
                self.pool[s * bb:(s + 1) * bb].copy_(torch.from_numpy(np.ascontiguousarray(bank(e))))
            self.cache = None

    def weights(self) -> ftm.LayerWeights:
        return ftm.LayerWeights(self.w_router.data_ptr(), None if self.bias is None else self.bias.data_ptr(),
                                self.pool.data_ptr(), self.slot_of_expert.data_ptr(),
                                None if self.shared_bank is None else self.shared_bank.data_ptr())

    def hidden(self, T: int, step: int = 0) -> torch.Tensor:
        return to_device_storage(self.layer.hidden_storage(T, step), self.cfg.act_dtype, self.device)

    def out_dtype(self):
        return torch.float32 if self.cfg.act_dtype == "f32" else torch.bfloat16


def pack_banks(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """All banks of a layer, [E + has_shared][bank_bytes] uint8 (row E = shared)."""
    layer = Layer(cfg, seed)
    desc = ftm.desc_for(cfg)
    bl = ftm.ftm_get_bank_layout(desc)
    out = np.zeros((cfg.E + cfg.has_shared, bl.bank_bytes), dtype=np.uint8)
    for e in range(cfg.E + cfg.has_shared):
        pack_bank(desc, layer.expert(e), bl, out=out[e])
    return out


class Workspace:
    """A 256-byte aligned device scratch buffer of at least nbytes."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.ptr = self.buf.data_ptr() + off
