"""COAT FP8 optimizer-state step and activation quantizers for B200 (sm_100a).

The compute lives in libcoat.so (hand-written CUDA, C ABI in include/coat.h);
this package is its thin ctypes binding plus helpers for sharding and
synthetic inputs.  The library is loaded on first use and a missing library
raises -- there is no CPU path.
"""
from ._lib import (  # noqa: F401
    COAT_E4M3,
    COAT_E5M2,
    COAT_FORCE_K1,
    COAT_NOALLOC_MAX_GROUPS,
    CoatError,
    PackTable,
    coat_adamw_fp8_step,
    coat_adamw_fp8_step_peers,
    coat_count_nonfinite_bf16,
    coat_dequant,
    coat_enable_peer_access,
    coat_fp8_encode,
    coat_group_quant_1xG,
    coat_group_scaling_quant_pertensor,
    coat_group_scaling_quant_pertensor_noalloc,
    coat_group_scaling_workspace_bytes,
    coat_norm_group_amax,
    coat_pack_bf16,
    coat_quantize_state,
    coat_state_stats,
    coat_status_string,
    coat_swiglu_group_amax,
    coat_unpack_bf16,
    coat_version,
    load,
)

__version__ = "0.1.0"
