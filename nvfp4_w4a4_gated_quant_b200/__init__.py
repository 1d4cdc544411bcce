"""NVFP4 W4A4 Gated DeltaNet layer forward for B200 (sm_100a).

The compute path is the C-ABI library ``libgdn.so`` built from ``csrc/``
(hand-written sm_100a kernels); ``_lib`` is its thin ctypes binding.  PyTorch
supplies device memory and streams only.  Importing this package does not load
the library; the first call does, and raises if it is missing.
"""
from ._lib import (  # noqa: F401
    GdnError,
    QuantizedLayerWeights,
    gdn_delta_rule_fwd,
    gdn_delta_rule_step,
    gdn_gates,
    gdn_gemm_nvfp4,
    gdn_layer_fwd,
    gdn_layer_workspace_offsets,
    gdn_layer_workspace_size,
    gdn_quantize_nvfp4,
    gemm_bf16,
    layer_cfg,
    lib,
    stream_check,
)
