"""The forward entry point that allocates no device memory.

Some callers cannot call cudaMalloc: code running under a fixed memory plan
(graph capture), processes whose allocator owns every device byte, embedded
callers that may not grow their footprint.  For them the library keeps the
layer's scratch in a fixed 32 MiB device array.  The same kernels run on the
same carve-up as with a caller workspace, so the output must equal the
workspace entry point's bit for bit, and the oracle's within the Y tolerance
used everywhere here.  The array keeps the previous call's contents: between
two calls of one layer a different layer (another shape, other inputs) goes
through it, and the second call must still give the same bits.  The status
word of the array is read back after every call.  This file is collected
last so that a failure here cannot stop the other tests."""
import numpy as np
import pytest

import synth
from dq_case import Case, assert_y_close

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


LAYERS = [synth.WORKLOADS["tiny"], _wl("ragged", 3, 10, 37, 512, 512, 32, (1, 2, 2)),
          _wl("cube_222", 5, 9, 21, 768, 256, 16, (2, 2, 2))]


def _device_inputs(dq, torch, case):
    packed, L1m, L2s, _ = dq.dq_pack_weight_factors(case.Wb, case.L1, case.L2)
    dev = torch.device("cuda")
    return tuple(torch.from_numpy(a).to(dev) for a in (case.X.view(np.int16), packed, L1m.view(np.int16),
                                                        L2s.view(np.int16)))


def _run_no_alloc(dq, torch, case, inputs):
    wl, (t, h, w) = case.wl, case.cube
    Xd, Pd, L1d, L2d = inputs
    st = torch.cuda.current_stream()
    Yd = torch.full((wl.N, wl.Co), 0x7FC0, dtype=torch.int16, device=Xd.device)   # NaN-filled output
    dq.dq_linear_forward_noalloc(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, st)
    torch.cuda.synchronize()
    assert dq.dq_read_device_status(dq.DQ_NOALLOC_WORKSPACE, st, clear=True) == 0
    return Yd.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("i", range(len(LAYERS)), ids=[wl.name for wl in LAYERS])
def test_no_alloc_matches_workspace_entry_point(env, i):
    dq, torch = env
    case = Case(LAYERS[i])
    other = Case(LAYERS[(i + 1) % len(LAYERS)], seed=77)
    ref = case.run_gpu(dq, torch)          # dq_linear_forward_ex with a caller workspace
    assert ref["status"] == 0
    act, wq = case.run_oracle()
    y_oracle = case.oracle_rows(act, wq, np.arange(case.wl.N))
    mine, theirs = _device_inputs(dq, torch, case), _device_inputs(dq, torch, other)
    for _ in range(2):
        y = _run_no_alloc(dq, torch, case, mine)
        assert np.array_equal(y, ref["Y"]), "no-alloc Y differs from the workspace entry point's"
        assert_y_close(y, y_oracle, what="no-alloc Y")
        # another layer through the shared array before the next call
        _run_no_alloc(dq, torch, other, theirs)


def test_no_alloc_reports_a_bad_packed_weight(env):
    """A device-side error of a no-alloc call is readable from the array's status
    word, and the next good call clears it."""
    dq, torch = env
    case = Case(LAYERS[0])
    Xd, Pd, L1d, L2d = _device_inputs(dq, torch, case)
    bad = Pd.clone()
    bad[0] ^= 0xFF            # magic
    wl, (t, h, w) = case.wl, case.cube
    st = torch.cuda.current_stream()
    Yd = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=Xd.device)
    dq.dq_linear_forward_noalloc(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, bad, L1d, L2d, Yd, st)
    assert dq.dq_read_device_status(dq.DQ_NOALLOC_WORKSPACE, st) == dq.DQ_ERR_BAD_PACKED_WEIGHT
    _run_no_alloc(dq, torch, case, (Xd, Pd, L1d, L2d))


def test_no_alloc_refuses_layers_beyond_its_array(env):
    dq, torch = env
    wl = synth.WORKLOADS["wan480p_proj"]
    t, h, w = wl.cube
    assert dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank) > (32 << 20)
    rc = dq._lib.dq_linear_forward_noalloc(0x10000, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, 0x20000,
                                           0x30000, 0x40000, 0x50000, None)
    assert rc == dq.DQ_ERR_WORKSPACE_TOO_SMALL
