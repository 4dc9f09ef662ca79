"""Host-side packing of one expert's weights into the library's bank layout.

A bank is the contiguous byte range of one expert (gate rows, then up rows,
then down, then block scales), so a cache miss is one host-to-device copy.
Offsets come from ``ftm_get_bank_layout``; this module only places bytes.
"""
from __future__ import annotations

import numpy as np

from .binding import FTM_BF16, FTM_F32, FTM_FP8_E4M3_B128, FTM_MXFP4, FTM_NVFP4, BankLayout, LayerDesc, ftm_get_bank_layout


def nvfp4_scale_chunks(s16: np.ndarray) -> np.ndarray:
    """Block scales [R][G] (G groups per row: C/16 for NVFP4, C/32 for MXFP4)
    -> the MMA chunk layout: one 512-byte chunk per (128-row block rb, block
    kb of four groups), chunks ordered [rb][kb]; inside a chunk the scale of
    local row r and group j of the block is byte (r%32)*16 + (r//32)*4 + j."""
    R, G16 = s16.shape
    assert R % 128 == 0 and G16 % 4 == 0
    a = np.ascontiguousarray(s16, dtype=np.uint8).reshape(R // 128, 4, 32, G16 // 4, 4)
    return np.ascontiguousarray(a.transpose(0, 3, 2, 1, 4)).ravel()


def gate_up_paired_rows(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    """[I][C] gate and up rows -> [2I][C] in paired order: 64 gate rows, then
    the same 64 up rows, and so on (the row order of the NVFP4 gate/up scale
    chunks, so one 128-row chunk covers the gate and up rows of 64 intermediate
    indices)."""
    I, C = gate.shape
    assert up.shape == (I, C) and I % 64 == 0
    return np.stack([gate.reshape(I // 64, 64, C), up.reshape(I // 64, 64, C)], axis=1).reshape(2 * I, C)


def _put(bank: np.ndarray, off: int, arr: np.ndarray, nbytes: int):
    b = np.ascontiguousarray(arr).view(np.uint8).ravel()
    assert b.size == nbytes, (b.size, nbytes)
    bank[off:off + nbytes] = b


def pack_bank(desc: LayerDesc, ew, bl: BankLayout = None, out: np.ndarray = None) -> np.ndarray:
    """ew: an expert in storage form with .gate/.up/.down
    f32/bf16: arrays [I][d], [I][d], [d][I] (float32 or bf16 bits as uint16);
    fp8: (q uint8, s float32 [R/128][C/128]) per matrix;
    nvfp4: (q packed uint8 [R][C/2], s16 uint8 [R][C/16], s_t float) per matrix;
    mxfp4: (q packed uint8 [R][C/2], s32 E8M0 codes uint8 [R][C/32]) per matrix."""
    bl = bl or ftm_get_bank_layout(desc)
    bank = out if out is not None else np.zeros(bl.bank_bytes, dtype=np.uint8)
    w = desc.wdtype
    if w in (FTM_F32, FTM_BF16):
        _put(bank, bl.w_gu_off, np.concatenate([ew.gate, ew.up], axis=0), bl.w_gu_bytes)
        _put(bank, bl.w_d_off, ew.down, bl.w_d_bytes)
    elif w == FTM_FP8_E4M3_B128:
        _put(bank, bl.w_gu_off, np.concatenate([ew.gate[0], ew.up[0]], axis=0), bl.w_gu_bytes)
        _put(bank, bl.w_d_off, ew.down[0], bl.w_d_bytes)
        _put(bank, bl.s_gu_off, np.concatenate([ew.gate[1], ew.up[1]], axis=0).astype(np.float32), bl.s_gu_bytes)
        _put(bank, bl.s_d_off, ew.down[1].astype(np.float32), bl.s_d_bytes)
    elif w == FTM_NVFP4:
        _put(bank, bl.w_gu_off, np.concatenate([ew.gate[0], ew.up[0]], axis=0), bl.w_gu_bytes)
        _put(bank, bl.w_d_off, ew.down[0], bl.w_d_bytes)
        _put(bank, bl.s_gu_off, nvfp4_scale_chunks(gate_up_paired_rows(ew.gate[1], ew.up[1])), bl.s_gu_bytes)
        _put(bank, bl.s_d_off, nvfp4_scale_chunks(ew.down[1]), bl.s_d_bytes)
        _put(bank, bl.s_t_off, np.array([ew.gate[2], ew.up[2], ew.down[2], 0.0], dtype=np.float32), bl.s_t_bytes)
    elif w == FTM_MXFP4:
        _put(bank, bl.w_gu_off, np.concatenate([ew.gate[0], ew.up[0]], axis=0), bl.w_gu_bytes)
        _put(bank, bl.w_d_off, ew.down[0], bl.w_d_bytes)
        _put(bank, bl.s_gu_off, nvfp4_scale_chunks(gate_up_paired_rows(ew.gate[1], ew.up[1])), bl.s_gu_bytes)
        _put(bank, bl.s_d_off, nvfp4_scale_chunks(ew.down[1]), bl.s_d_bytes)
    else:
        raise ValueError(w)
    return bank
