"""B200-native (sm_100a) fused per-row-scaled gated activation + MXFP8 quantization.

The computation lives in ``libmoeact.so`` (hand-written CUDA kernels behind the
C ABI of ``include/moeact.h``); ``ops`` wraps it for PyTorch tensors and
``workloads`` draws the seeded synthetic inputs.  Importing this package does
not load the library; the first call does, and fails loudly if it is missing.
"""
from .ops import (  # noqa: F401
    COLWISE,
    MXFP8,
    ROWWISE,
    Backward,
    bwd_workspace_bytes,
    grouped_scaled_clamped_swiglu_mxfp8_bwd,
    grouped_scaled_clamped_swiglu_mxfp8_fwd,
    grouped_scaled_srelu_mxfp8_bwd,
    grouped_scaled_srelu_mxfp8_fwd,
    grouped_scaled_swiglu_mxfp8_fc2,
    grouped_scaled_swiglu_mxfp8_bwd,
    grouped_scaled_swiglu_mxfp8_fwd,
    clamped_sigmoid_table,
    init,
    init_clamped,
    scaled_clamped_swiglu_mxfp8_bwd,
    scaled_clamped_swiglu_mxfp8_fwd,
    scaled_srelu_mxfp8_bwd,
    scaled_srelu_mxfp8_fwd,
    scaled_swiglu_mxfp8_bwd,
    scaled_swiglu_mxfp8_fwd,
    sigmoid_table,
    splits_to_offsets,
)
