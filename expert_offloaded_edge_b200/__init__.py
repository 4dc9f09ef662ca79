"""B200-native routed-MoE layer over a slot-indexed expert cache.

Python binding of the C ABI in ``include/ftm.h`` (argument marshalling only;
every step runs in the sm_100a kernels of ``libftm.so``).  Function names match
the C entry points.  Tensors are torch tensors on the CUDA device (or pinned
host tensors where the header says host); streams default to torch's current
stream.
"""
from .binding import (  # noqa: F401
    FTM_BF16,
    FTM_F32,
    FTM_FP8_E4M3_B128,
    FTM_MXFP4,
    FTM_NVFP4,
    BankLayout,
    FtmError,
    Hybrid,
    LayerDesc,
    LayerWeights,
    SlotCache,
    desc_for,
    ftm_combine,
    ftm_device_status,
    ftm_expert_ffn,
    ftm_ffn_workspace_bytes,
    ftm_get_bank_layout,
    ftm_host_expert_ffn,
    ftm_host_ffn_scratch_bytes,
    ftm_hybrid_host_bytes,
    ftm_hybrid_split,
    ftm_hybrid_workspace_bytes,
    ftm_kernel_launches,
    ftm_selftest_bounded_wait,
    ftm_last_error,
    ftm_moe_layer_forward,
    ftm_moe_layer_forward_hybrid,
    ftm_moe_layer_forward_noalloc,
    ftm_moe_layers_forward,
    ftm_last_warning,
    ftm_permute,
    ftm_permute_workspace_bytes,
    ftm_route,
    ftm_set_profile_events,
    KERNEL_NAMES,
    ftm_slot_host_scratch_ints,
    ftm_slot_lookup_update,
    ftm_slot_resize,
    ftm_slot_stage_layer,
    ftm_slot_workspace_bytes,
    ftm_workspace_bytes,
    library,
)
