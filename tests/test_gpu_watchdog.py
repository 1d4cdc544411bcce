"""The bounded device waits report a timeout instead of hanging.

A one-warp kernel waits (a bounded number of polls) on an mbarrier that
nothing arrives on -- the same wait loop the pipelined GEMM uses -- and must
leave GDN_ERR_TIMEOUT in the device status word; reading it clears it, and the
context stays usable for the next call.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest
import torch

from nvfp4_w4a4_gated_quant_b200 import _lib
from tests._helpers import f32_cuda, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    L = _lib.lib()
    stream = torch.cuda.current_stream()
    assert L.gdn_stream_check(_lib._stream()) == 0
    assert L.gdn_selftest_bounded_wait(2000, _lib._stream()) == 0
    assert L.gdn_stream_check(_lib._stream()) == 5          # GDN_ERR_TIMEOUT
    assert L.gdn_stream_check(_lib._stream()) == 0          # read and cleared
    # the context is still healthy: a normal call runs and is correct
    a = np.zeros((4, 2), np.float32)
    la, be = _lib.gdn_gates(f32_cuda(a), f32_cuda(a), f32_cuda(np.zeros(2, np.float32)),
                            f32_cuda(np.zeros(2, np.float32)))
    _lib.stream_check()
    np.testing.assert_allclose(np.exp(to_np(la).astype(np.float64)), 0.5, rtol=1e-6)
    stream.synchronize()
