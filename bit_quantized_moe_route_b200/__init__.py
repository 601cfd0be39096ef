"""B200-native routed low-bit MoE FFN layer.

The compute lives in ``libmoe_lowbit.so`` (hand-written CUDA for sm_100a,
C ABI in ``include/moe_lowbit.h``); this package is its thin Python binding.
"""
from ._lib import (  # noqa: F401
    FFN_AUTO,
    FFN_DECODE_FUSED,
    FFN_GEMV,
    FFN_TENSOR_CORE,
    FMT_AFFINE,
    FMT_MXFP4,
    LIB_PATH,
    Dims,
    MoEError,
    QMatC,
    alloc_workspace,
    combine,
    dequant_mxfp8,
    expert_ffn,
    expert_ffn_noalloc,
    forward,
    forward_host,
    forward_partial,
    hc_sinkhorn_mix,
    load_library,
    make_dims,
    permute,
    qmat,
    read_device_error,
    read_noalloc_error,
    route,
    set_ffn_path,
    set_timing_events,
    status_string,
    timing_labels,
    workspace_size,
)
from .layer import MoELayer, expert_range  # noqa: F401
