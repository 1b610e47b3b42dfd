"""The allocation-free decode step (ssd_decode_step_noalloc) against the workspace one.

Some callers cannot allocate device memory or pass a workspace (an engine's enqueue hook
that owns all device memory, code recorded during CUDA graph capture, serving loops that
forbid allocation after start-up).  For them the library keeps the decode step's scratch
in its own file-scope device array.  This test calls that entry point through the C ABI
twice in a row (the second call reuses the scratch the first one left behind) and checks
y, the SSM state and the conv window against ssd_decode_step with a caller workspace,
at the same tolerance the other decode tests use.  It is collected last and passes both
alone in a fresh process (where its first call does the per-device set-up) and after the
rest of the suite.
"""
import numpy as np
import pytest
import torch

from ssd_inputs import make_decode
from tests.helpers import bf16_tensor, check, f32_tensor

pytestmark = pytest.mark.gpu

ssd = pytest.importorskip("state_space_model_04_b200")


def _dev(d):
    return dict(h=f32_tensor(d.h), cs=f32_tensor(d.conv_state), xbc=bf16_tensor(d.xbc_bits),
                dt=f32_tensor(d.dt), A=f32_tensor(d.A), D=f32_tensor(d.D), w=f32_tensor(d.conv_w),
                b=f32_tensor(d.conv_b))


def test_noalloc_decode_matches_workspace_decode_two_calls():
    d = make_decode(layers=3, b=2, H=8, P=64, N=128, G=2, ring=2, seed=61)
    ref, got = _dev(d), _dev(d)
    ws = torch.empty(ssd.decode_workspace_size(3, 2, 2), dtype=torch.uint8, device="cuda")
    for s in range(2):
        y_ref = ssd.decode_step(ref["h"], ref["cs"], ref["xbc"][s], ref["dt"][s], ref["A"], ref["D"], ref["w"],
                                ref["b"], G=2, workspace=ws)
        y = torch.empty_like(y_ref)
        ssd.decode_step_noalloc(got["h"], got["cs"], got["xbc"][s], got["dt"][s], got["A"], got["D"], got["w"],
                                got["b"], y, G=2)
        torch.cuda.synchronize()
        check(y.float().cpu().numpy(), y_ref.float().cpu().numpy(), "bf16", "y call %d" % s)
        check(got["h"].cpu().numpy(), ref["h"].cpu().numpy(), "bf16", "h call %d" % s)
        np.testing.assert_array_equal(got["cs"].cpu().numpy(), ref["cs"].cpu().numpy())


def test_noalloc_decode_rejects_sizes_beyond_its_scratch():
    limit = 65536  # SSD_DECODE_NOALLOC_MAX_COUNTERS in include/ssd.h
    d = make_decode(layers=1, b=1, H=8, P=64, N=128, G=1, ring=1, seed=62)
    t = _dev(d)
    y = torch.empty((1, 1, 8, 64), dtype=torch.bfloat16, device="cuda")
    L = ssd.lib()
    st = L.ssd_decode_step_noalloc(limit + 1, 1, 8, 64, 128, 1, 4, 1, 1, t["h"].data_ptr(), t["cs"].data_ptr(),
                                   t["xbc"].data_ptr(), t["dt"].data_ptr(), t["A"].data_ptr(), t["D"].data_ptr(),
                                   t["w"].data_ptr(), t["b"].data_ptr(), y.data_ptr(), None)
    assert st == 1 and "exceeds" in ssd.last_error()
