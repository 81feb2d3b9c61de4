"""Failure reporting on the GPU without faulting it: a bounded device wait that
is made to run out (a barrier nothing arrives at) must come back as
NVFP4_ERR_TIMEOUT through the status word, leave the context usable, and argument
errors must come back before any launch."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(oracle):
    assert nv.last_device_status() == nv.OK
    assert nv.lib().nvfp4_debug_wait_timeout(50_000, nv._stream()) == nv.OK   # 50 ms budget
    assert nv.last_device_status() == nv.ERR_TIMEOUT
    assert nv.last_device_status() == nv.OK                                   # cleared
    x = W.random_bf16((64, 128), seed=1).cuda()
    p, s, g = nv.nvfp4_quantize(x)
    op, os_, og = oracle.quantize(W.to_u16(x.cpu()))
    assert np.array_equal(p.cpu().numpy(), op)


def test_device_argument_errors():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.nvfp4_quantize(x[:, 8:].contiguous()[:, :48].contiguous(), rotate_group=32)
    assert e.value.status == nv.ERR_SHAPE
    bad = torch.zeros(4 * 64 + 8, dtype=torch.bfloat16, device="cuda")[1:257].view(4, 64)
    with pytest.raises(nv.NVFP4Error) as e:
        nv.nvfp4_quantize(bad)
    assert e.value.status == nv.ERR_ALIGN
