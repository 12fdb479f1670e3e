"""The forward entry point that allocates no device memory.

For callers that cannot call cudaMalloc (fixed memory plans such as graph
capture, allocators that own all device memory, embedded callers), the
library keeps the layer's scratch in a fixed 32 MiB device array.  Its output
must match the regular workspace entry point within the tolerance used by
every Y check here, call after call: the array keeps the previous call's
contents, so the second call checks that nothing stale leaks into it.  This
file is collected last so that a failure here cannot stop the other tests."""
import numpy as np
import pytest

import synth
from dq_case import Case, assert_y_close, bf16_bits_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    import video_diffusion_w4a4_b200 as dq
    return dq, torch


def _wl(name, T, H, W, Ci, Co, r, cube):
    grid = (T, max(1, -(-H // 4)), max(1, -(-W // 4)))
    return synth.Workload(name, T, H, W, Ci, Co, r, cube, grid, (0.01, 50.0), (0.01, 20.0))


@pytest.mark.parametrize("wl", [synth.WORKLOADS["tiny"], _wl("ragged", 3, 10, 37, 512, 512, 32, (1, 2, 2))],
                         ids=["tiny", "ragged"])
def test_no_alloc_matches_workspace_entry_point(env, wl):
    dq, torch = env
    case = Case(wl)
    ref = case.run_gpu(dq, torch)          # dq_linear_forward_ex with a caller workspace
    assert ref["status"] == 0
    y_ref = bf16_bits_to_f64(ref["Y"])
    t, h, w = case.cube
    packed, L1m, L2s, _ = dq.dq_pack_weight_factors(case.Wb, case.L1, case.L2)
    dev = torch.device("cuda")
    Xd = torch.from_numpy(case.X.view(np.int16)).to(dev)
    Pd, L1d, L2d = (torch.from_numpy(a).to(dev) for a in (packed, L1m.view(np.int16), L2s.view(np.int16)))
    st = torch.cuda.current_stream()
    for _ in range(2):
        Yd = torch.full((wl.N, wl.Co), 0x7FC0, dtype=torch.int16, device=dev)   # NaN-filled output
        dq.dq_linear_forward_noalloc(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, st)
        torch.cuda.synchronize()
        assert_y_close(Yd.cpu().numpy().view(np.uint16), y_ref, what="no-alloc Y")


def test_no_alloc_refuses_layers_beyond_its_array(env):
    dq, torch = env
    wl = synth.WORKLOADS["wan480p_proj"]
    t, h, w = wl.cube
    assert dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank) > (32 << 20)
    rc = dq._lib.dq_linear_forward_noalloc(0x10000, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, 0x20000,
                                           0x30000, 0x40000, 0x50000, None)
    assert rc == dq.DQ_ERR_WORKSPACE_TOO_SMALL
