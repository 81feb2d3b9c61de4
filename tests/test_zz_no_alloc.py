"""nvfp4_linear_fixed_scratch: the linear with the library's own fixed device
scratch instead of a caller workspace, checked through the C ABI against
nvfp4_linear on the same inputs.  Both run the same kernels on the same inputs, so
the outputs must agree bit for bit; two calls in a row with different shapes, then a
repeat of the first, so that a stale or misplaced scratch byte would show.
This file is collected last on purpose: it must pass both in a fresh process and
after every other test has used the device.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_17_b200 as nv
from nvfp4_block_scaled_17_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def make_case(M, N, K, group, seed):
    x = W.with_outliers((M, K), 0.01, 20.0, W._gen(seed, "cpu"), "cpu").to(DEV)
    w = W.normal((N, K), 0.02, W._gen(seed + 1, "cpu"), "cpu").to(torch.bfloat16).to(DEV)
    b = W.normal((N,), 0.01, W._gen(seed + 2, "cpu"), "cpu").to(torch.bfloat16).to(DEV)
    wp, wsf, gw = nv.pack_weight(w, group)
    return x, wp, wsf, gw, b


def reference(case, N, group, gsf_x):
    x, wp, wsf, gw, b = case
    return nv.nvfp4_linear(x, wp, wsf, gw, N, bias=b, gsf_x=gsf_x, rotate_group=group)


def fixed(case, N, group, gsf_x):
    x, wp, wsf, gw, b = case
    out = torch.full((x.shape[0], N), float("nan"), dtype=torch.bfloat16, device=DEV)
    return nv.nvfp4_linear_fixed_scratch(x, wp, wsf, gw, N, out, bias=b, gsf_x=gsf_x,
                                         rotate_group=group)


def check(y, y_ref, what):
    torch.cuda.synchronize()
    assert nv.last_device_status() == nv.OK
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), what


@pytest.mark.parametrize("group", [0, 128])
def test_two_calls_in_a_row_match_nvfp4_linear(group):
    # first a ragged shape, then one tile of the ViT block at the largest K it takes
    shapes = [(300, 520, 512, 11), (4096, 1024, 1024, 12)]
    cases = [make_case(M, N, K, group, seed) for M, N, K, seed in shapes]
    refs = [reference(c, s[1], group, None) for c, s in zip(cases, shapes)]
    outs = [fixed(c, s[1], group, None) for c, s in zip(cases, shapes)]
    for y, r, s in zip(outs, refs, shapes):
        check(y, r, f"fixed scratch {s[:3]} g={group}")
    # and again, now after the larger call left its bytes in the scratch
    y = fixed(cases[0], shapes[0][1], group, None)
    check(y, refs[0], f"fixed scratch repeat {shapes[0][:3]} g={group}")


def test_static_scale_matches_nvfp4_linear():
    M, N, K = 1000, 768, 1024
    case = make_case(M, N, K, 64, 21)
    gsf_x = torch.tensor([2688.0 / 40.0], dtype=torch.float32, device=DEV)
    for _ in range(2):
        check(fixed(case, N, 64, gsf_x), reference(case, N, 64, gsf_x), "fixed scratch static")


def test_largest_fitting_and_too_large_sizes():
    K = 1024
    cap = nv.FIXED_SCRATCH_BYTES
    M_fit = max(m for m in range(128, 16384, 128) if nv.nvfp4_linear_workspace_bytes(m, K) <= cap)
    case = make_case(M_fit, 256, K, 128, 31)
    check(fixed(case, 256, 128, None), reference(case, 256, 128, None), f"fixed M={M_fit}")

    M_big = M_fit + 128
    assert nv.nvfp4_linear_workspace_bytes(M_big, K) > cap
    x, wp, wsf, gw, b = make_case(M_big, 256, K, 128, 32)
    out = torch.zeros(M_big, 256, dtype=torch.bfloat16, device=DEV)
    st = nv.lib().nvfp4_linear_fixed_scratch(
        x.data_ptr(), M_big, K, wp.data_ptr(), wsf.data_ptr(), gw.data_ptr(), 256, b.data_ptr(),
        None, 128, out.data_ptr(), None)
    assert st == nv.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not out.any(), "a rejected call must launch nothing"
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_linear_fixed_scratch(x, wp, wsf, gw, 256, out, bias=b, rotate_group=128)
    assert np.isfinite(out.float().cpu().numpy()).all()
