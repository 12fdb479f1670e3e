"""Cube-sharded layer: the slab partition, the all-reduce of the one exchanged
scalar (two gloo ranks on CPU, with the library's calls recorded by a stand-in),
and, on the GPU, two slabs run one after the other giving the unsharded Y bit
for bit."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from video_diffusion_w4a4_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("T,t,world", [(21, 1, 2), (21, 1, 8), (21, 2, 3), (9, 4, 3), (8, 2, 4), (5, 5, 1)])
def test_slabs_cover_whole_cube_layers(T, t, world):
    spans = [shard.slab_frames(T, t, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == T
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    assert all(s0 % t == 0 and s1 > s0 for s0, s1 in spans)
    layers = [-(-(s1 - s0) // t) for s0, s1 in spans]
    assert max(layers) - min(layers) <= 1


def test_more_ranks_than_cube_layers_is_refused():
    with pytest.raises(ValueError):
        shard.slab_frames(4, 2, 3, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import video_diffusion_w4a4_b200 as dq
    from video_diffusion_w4a4_b200 import shard as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T, H, W, cube, Ci, Co, r = 6, 4, 4, (1, 2, 2), 256, 256, 16
        t0, t1 = sh.slab_frames(T, cube[0], world, rank)
        lay = dq.dq_workspace_layout_get(t1 - t0, H, W, *cube, Ci, Co, r)
        ws = torch.zeros(lay.total_bytes, dtype=torch.uint8)
        calls = []
        local_amax = [3.5, 7.25][rank]

        def fake_forward(*a):
            mask = a[16]
            calls.append(mask)
            if mask == dq.DQ_STAGE_STATS:   # the statistics pass leaves this slab's max |delta|
                ws[lay.off_scalars:lay.off_scalars + 4].view(torch.float32)[0] = local_amax
            else:
                seen = float(ws[lay.off_scalars:lay.off_scalars + 4].view(torch.float32)[0])
                calls.append(seen)

        real = dq.dq_linear_forward_ex
        dq.dq_linear_forward_ex = fake_forward
        try:
            sh.forward_sharded(None, t1 - t0, H, W, cube, Ci, Co, r, None, None, None, None, ws,
                               lambda v: dist.all_reduce(v, op=dist.ReduceOp.MAX))
        finally:
            dq.dq_linear_forward_ex = real
        out.put((rank, calls))
    finally:
        dist.destroy_process_group()


def test_two_ranks_exchange_only_the_largest_delta():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    import video_diffusion_w4a4_b200 as dq
    for rank, calls in sorted(q.get() for _ in range(world)):
        rest = dq.DQ_STAGE_ENCODE | dq.DQ_STAGE_KERNEL_GEMM | dq.DQ_STAGE_MAIN_GEMM
        assert calls == [dq.DQ_STAGE_STATS, rest, 7.25], (rank, calls)


@pytest.mark.gpu
@pytest.mark.parametrize("name,slabs", [("ragged_122", 2), ("cube_414_r128", 3), ("ragged_222", 2),
                                        ("wan480p_proj", 3)])
def test_sharded_equals_unsharded_on_one_gpu(name, slabs):
    """The slabs run one after the other on one GPU, the host taking the maximum that the
    all-reduce would: Y of every row bit-identical to the unsharded layer (small ragged
    lattices, and the 480p projection in three slabs of 7 frames)."""
    import torch
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import synth
    import video_diffusion_w4a4_b200 as dq
    from dq_case import Case
    from test_gpu_parity import SMALL
    wl = dict(SMALL).get(name) or synth.WORKLOADS[name]
    case = Case(wl)
    full = case.run_gpu(dq, torch)
    t, h, w = case.cube
    packed, L1m, L2s, _ = dq.dq_pack_weight_factors(case.Wb, case.L1, case.L2)
    dev = torch.device("cuda")
    Pd, L1d, L2d = (torch.from_numpy(a).to(dev) for a in (packed, L1m.view(np.int16), L2s.view(np.int16)))
    HW = wl.H * wl.W
    X = torch.from_numpy(case.X.view(np.int16)).to(dev)
    Y = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=dev)
    spans = [shard.slab_frames(wl.T, t, slabs, r) for r in range(slabs)]
    wss, lays = [], []
    st = torch.cuda.current_stream()
    for t0, t1 in spans:
        ts = shard.slab_cube(case.cube, t1 - t0)[0]
        lay = dq.dq_workspace_layout_get(t1 - t0, wl.H, wl.W, ts, h, w, wl.Ci, wl.Co, wl.rank)
        ws = torch.zeros(lay.total_bytes, dtype=torch.uint8, device=dev)
        dq.dq_linear_forward_ex(X[t0 * HW:t1 * HW], t1 - t0, wl.H, wl.W, ts, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d,
                                L2d, Y[t0 * HW:t1 * HW], ws, lay.total_bytes, dq.DQ_STAGE_STATS, None, st)
        wss.append(ws)
        lays.append(lay)
    amaxes = [ws[l.off_scalars:l.off_scalars + 4].view(torch.float32) for ws, l in zip(wss, lays)]
    top = torch.stack([a[0] for a in amaxes]).max()
    for a in amaxes:
        a.fill_(top)
    for (t0, t1), ws, lay in zip(spans, wss, lays):
        ts = shard.slab_cube(case.cube, t1 - t0)[0]
        dq.dq_linear_forward_ex(X[t0 * HW:t1 * HW], t1 - t0, wl.H, wl.W, ts, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d,
                                L2d, Y[t0 * HW:t1 * HW], ws, lay.total_bytes,
                                dq.DQ_STAGE_ENCODE | dq.DQ_STAGE_KERNEL_GEMM | dq.DQ_STAGE_MAIN_GEMM, None, st)
    torch.cuda.synchronize()
    for ws in wss:
        assert dq.dq_read_device_status(ws, st, clear=True) == 0
    assert float(top) == float(np.float32(full["amax_delta"]))
    assert np.array_equal(Y.cpu().numpy().view(np.uint16), full["Y"])


def test_last_slab_cube_is_the_ragged_layer():
    assert shard.slab_cube((4, 2, 8), 1) == (1, 2, 8)
    assert shard.slab_cube((4, 2, 8), 4) == (4, 2, 8)
