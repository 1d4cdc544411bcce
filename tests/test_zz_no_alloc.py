"""The allocation-free layer entry point (gdn_layer_fwd_static_ws).

It serves callers that cannot allocate device memory -- plugins that are handed
only their input and output tensors, and real-time paths whose memory budget
is fixed up front: its scratch is a static device array inside the library
instead of a caller workspace.  It runs the same kernels in the same order as
gdn_layer_fwd, which is deterministic, so its results must be bit-identical
to the workspace entry point's; two calls in a row check that nothing stale
in the shared array leaks into the second call.  This file sorts last so that
a run stopping at the first failure has already run every other test; it also
passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib, inputs

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_entry_point_twice():
    d = inputs.tiny_layer()
    H, dk, dv = d["H"], d["dk"], d["dv"]
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], H, dk, dv)
    x = torch.from_numpy(d["x"]).cuda().to(torch.bfloat16)
    S0 = torch.from_numpy(np.random.default_rng(1).standard_normal((1, H, dk, dv)).astype(np.float32) * 0.1).cuda()
    y_ref, S_ref, _ = _lib.gdn_layer_fwd(lw, x, S0=S0)
    _lib.stream_check()
    for _ in range(2):      # the shared array keeps the last call's contents
        y, S_T = _lib.gdn_layer_fwd_static_ws(lw, x, S0=S0)
        _lib.stream_check()
        assert torch.equal(y, y_ref)
        assert torch.equal(S_T, S_ref)


def test_static_scratch_rejects_oversized_workspace():
    cfg = _lib.layer_cfg(4, 8192, 5120, 32, 128, 128)
    assert _lib.gdn_layer_workspace_size(cfg) > _lib.LAYER_STATIC_WS_BYTES
    d = inputs.tiny_layer()
    lw = _lib.QuantizedLayerWeights(d["W"], d["A_log"], d["dt_bias"], d["H"], d["dk"], d["dv"])
    # a tiny-layer-shaped call with enough tokens to overflow the array
    T = _lib.LAYER_STATIC_WS_BYTES // 400
    x = torch.zeros((1, T, d["d_model"]), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.GdnError, match="exceeds"):
        _lib.gdn_layer_fwd_static_ws(lw, x)
