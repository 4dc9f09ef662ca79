"""The allocation-free whole-layer entry point.

Some callers cannot allocate device memory (code running during CUDA-graph
capture, allocator-free embedded runtimes, engines that reserve all memory up
front).  ftm_moe_layer_forward_noalloc serves them with a static scratch array
inside the library.  This file is collected last so that a run stopping at the
first failure has already run every other test; it passes alone in a fresh
process and after the other tests.
"""
import numpy as np
import pytest
import torch

import expert_offloaded_edge_b200 as ftm
import synth
from synth.device import DeviceLayer
from tests.gpu_util import TOL, assert_rows_close, run_layer, to_np_f32

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_twice():
    cfg = synth.CONFIGS["35b_decode"]
    dl = DeviceLayer(cfg)
    lib = ftm.library()
    for T in (64, 8):                       # two calls in a row, different batch sizes
        x = dl.hidden(T)
        want_t = run_layer(dl, x, T)                     # existing entry point, torch-allocated workspace
        want = to_np_f32(want_t)
        out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
        w = dl.weights()
        st = lib.ftm_moe_layer_forward_noalloc(ftm.binding.ctypes.byref(dl.desc), ftm.binding.ctypes.byref(w),
                                               x.data_ptr(), T, out.data_ptr(),
                                               torch.cuda.current_stream().cuda_stream)
        assert st == 0, ftm.ftm_last_error()
        torch.cuda.synchronize()
        assert ftm.ftm_device_status(True) == 0
        # the same kernels on the same inputs: bit-identical (a stale byte left in
        # the shared scratch by the previous call would show here), and so also
        # within the bf16 tolerance of the layer
        assert torch.equal(out, want_t), f"noalloc T={T} differs from the workspace entry point"
        assert_rows_close(to_np_f32(out), want, TOL["bf16"], f"noalloc T={T}")


def test_noalloc_rejects_batches_beyond_the_static_scratch():
    cfg = synth.CONFIGS["35b_decode"]
    dl = DeviceLayer(cfg)
    T = 4096                                  # needs far more than 16 MiB of scratch
    x = torch.zeros((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(ftm.FtmError) as ei:
        ftm.ftm_moe_layer_forward_noalloc(dl.desc, dl.weights(), x, T, out)
    assert ei.value.status == 1 and "static limit" in str(ei.value)
