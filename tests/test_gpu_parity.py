"""GPU parity of the DeltaQuant layer against the CPU oracle, through the C ABI.

Small shapes that span several tiles in every kernel and leave ragged edges
(partial cubes, a partial last M tile, boxes that overhang the lattice),
every cube shape the layer supports, and the degenerate 1x1x1 cube.  Every
quantised tensor must be bit-exact; Y within max(1 BF16 ulp, 1e-3 RMS)."""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from dq_case import Case, assert_kernel_term_close, assert_y_close, compare_quantised

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    import video_diffusion_w4a4_b200 as dq
    return dq, torch


def _wl(name, T, H, W, Ci, Co, r, cube, gelu=False):
    grid = (T, max(1, -(-H // 4)), max(1, -(-W // 4)))
    return synth.Workload(name, T, H, W, Ci, Co, r, cube, grid, (0.01, 50.0) if not gelu else (0.005, 80.0),
                          (0.01, 20.0), gelu=gelu)


def test_device_format_conversions(env):
    dq, torch = env
    mags2 = oracle.e2m1_value(np.arange(8))
    mags8 = oracle.e4m3_value(np.arange(127))
    pts = np.concatenate([mags2, (mags2[:-1] + mags2[1:]) / 2, mags8, (mags8[:-1] + mags8[1:]) / 2,
                          [448.0, 464.0, 500.0, 1e9, 7.0, 6.5, 2.0 ** -10, 2.0 ** -11, 0.0]]).astype(np.float32)
    pts = np.concatenate([pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rng = np.random.default_rng(0)
    sweep = np.exp(rng.uniform(np.log(1e-6), np.log(1000.0), 400000)).astype(np.float32)
    v = np.concatenate([pts, sweep])
    v = np.concatenate([v, -v]).astype(np.float32)
    n = v.size
    dev = torch.device("cuda")
    vin = torch.from_numpy(v).to(dev)
    e2 = torch.empty(n, dtype=torch.uint8, device=dev)
    e4 = torch.empty(n, dtype=torch.uint8, device=dev)
    back = torch.empty(n, dtype=torch.float32, device=dev)
    dq.dq_selftest_convert(vin, n, e2, e4, back, torch.cuda.current_stream())
    torch.cuda.synchronize()
    g2, g4, gb = e2.cpu().numpy(), e4.cpu().numpy(), back.cpu().numpy()
    w2, w4 = oracle.e2m1_encode(v), oracle.e4m3_encode(v)
    bad2 = np.flatnonzero(g2 != w2)
    bad4 = np.flatnonzero(g4 != w4)
    assert bad2.size == 0, ("E2M1", v[bad2[:8]], g2[bad2[:8]], w2[bad2[:8]])
    assert bad4.size == 0, ("E4M3", v[bad4[:8]], g4[bad4[:8]], w4[bad4[:8]])
    assert np.array_equal(gb.astype(np.float64), oracle.e4m3_value(g4))


SMALL = [
    ("tiny", None),
    ("ragged_122", _wl("ragged_122", 3, 10, 37, 512, 512, 32, (1, 2, 2))),
    ("ragged_222", _wl("ragged_222", 5, 9, 21, 768, 256, 16, (2, 2, 2))),
    ("unit_cube", _wl("unit_cube", 2, 7, 19, 256, 512, 16, (1, 1, 1))),
    ("cube_244", _wl("cube_244", 4, 9, 18, 512, 256, 48, (2, 4, 4))),
    ("cube_418", _wl("cube_418", 6, 5, 20, 256, 256, 16, (4, 1, 8))),
    ("gelu_122", _wl("gelu_122", 2, 12, 40, 1024, 512, 64, (1, 2, 2), gelu=True)),
    # the note's own operating point: 64-token cubes 4x1x4 and 4x2x8, low-rank branch of rank 128
    ("cube_414_r128", _wl("cube_414_r128", 9, 6, 22, 512, 256, 128, (4, 1, 4))),
    ("cube_428", _wl("cube_428", 8, 7, 27, 256, 512, 32, (4, 2, 8))),
    # cubes of more than 128 tokens: kernel tokens from the means kernel, boxes are row segments
    ("global", _wl("global", 3, 10, 37, 512, 256, 16, (3, 10, 37))),
    ("big_cube", _wl("big_cube", 5, 18, 21, 256, 256, 16, (2, 8, 16))),
    ("wide_cube", _wl("wide_cube", 2, 3, 200, 256, 256, 16, (1, 2, 150))),
]


@pytest.mark.parametrize("name,wl", SMALL, ids=[s[0] for s in SMALL])
def test_parity_small(env, name, wl):
    dq, torch = env
    wl = wl or synth.WORKLOADS["tiny"]
    case = Case(wl)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K))
    y_ref = case.oracle_rows(act, wq, np.arange(wl.N))
    assert_y_close(g["Y"], y_ref)


@pytest.mark.parametrize("name,kernel_group", [("ragged_122", 0), ("unit_cube", 0), ("global", 0),
                                                ("ragged_122", 64), ("cube_428", 64)])
def test_parity_bias(env, name, kernel_group):
    """A bias in the packed weight: every quantised tensor unchanged and bit-exact,
    Y = the oracle's x W^T + b within tolerance, for a ragged lattice, the
    one-token cube (P' per token), the whole-lattice cube (one P' row), and with
    group-64 kernel scales (P' without a per-row scale)."""
    dq, torch = env
    wl = dict(SMALL)[name]
    case = Case(wl, kernel_group=kernel_group)
    b = synth.normal_bf16((wl.Co,), sd=4.0, seed=21)
    g = case.run_gpu(dq, torch, bias=b)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K), bias=b,
                             extra_rel=2.0 ** -16 if kernel_group else 0.0)
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N), bias=b))
    # clearing the bias again gives the no-bias layer bit for bit
    g0 = case.run_gpu(dq, torch)
    g1 = case.run_gpu(dq, torch, packed_override=lambda p: dq.dq_pack_bias(dq.dq_pack_bias(p.copy(), b), None))
    assert np.array_equal(g0["Y"], g1["Y"])


@pytest.mark.parametrize("name", ["tiny", "ragged_122", "unit_cube", "cube_414_r128", "cube_428", "global",
                                  "wide_cube"])
def test_parity_group64_kernel_scales(env, name):
    """One FP8 scale per 64 channels of each kernel token: codes and the
    K x Ci/64 scales bit-exact, the hi + lo product operand within 2^-16, Y
    within tolerance; across small and big cubes and ragged lattices."""
    dq, torch = env
    wl = dict(SMALL)[name] or synth.WORKLOADS["tiny"]
    case = Case(wl, kernel_group=64)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    assert g["s8"].shape == act["s8"].shape
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K), extra_rel=2.0 ** -16)
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N)))


@pytest.mark.parametrize("name", ["tiny", "ragged_122", "ragged_222", "unit_cube", "cube_414_r128", "cube_428",
                                  "global", "wide_cube"])
def test_parity_fp8_kernel_product(env, name):
    """The FP8-rate kernel-token product on restricted-scale (C2) weights: the packed
    weight, every quantised tensor and S_delta bit-exact, P' within the fp32
    accumulation bound of the oracle's kernel term, Y within tolerance of the
    oracle's fp64 product with the same C2 weights; small and big cubes, ragged
    lattices, partial last tiles."""
    dq, torch = env
    wl = dict(SMALL)[name] or synth.WORKLOADS["tiny"]
    case = Case(wl, fp8_product=True)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K))
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N)))


def test_fp8_kernel_product_with_bias(env):
    dq, torch = env
    wl = dict(SMALL)["ragged_122"]
    case = Case(wl, fp8_product=True)
    b = synth.normal_bf16((wl.Co,), sd=4.0, seed=22)
    g = case.run_gpu(dq, torch, bias=b)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K), bias=b)
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N), bias=b))


def test_packed_weight_must_match_the_kernel_product(env):
    """A C2 weight run with the BF16 product (or a default weight with the FP8
    product) is reported in the device status word."""
    dq, torch = env
    def clear_flags(p):
        q = p.copy()
        q[28:32] = 0          # header flags word: the C2 bit cleared
        return q

    case = Case(synth.WORKLOADS["tiny"], fp8_product=True)
    out = case.run_gpu(dq, torch, packed_override=clear_flags)
    assert out["status"] == dq.DQ_ERR_BAD_PACKED_WEIGHT


@pytest.mark.parametrize("name", ["tiny", "ragged_122", "ragged_222", "unit_cube", "cube_244", "cube_418", "gelu_122",
                                  "cube_414_r128", "cube_428", "global", "big_cube", "wide_cube"])
def test_parity_single_read(env, name):
    """The single-read quantiser (power-of-two S_delta, one read of X): every
    quantised tensor bit-exact against the oracle's direct encode under the final
    power-of-two scale, S_delta too; P' and Y within tolerance; every cube shape,
    ragged lattices, big cubes whose means come from the means kernel."""
    dq, torch = env
    wl = dict(SMALL)[name] or synth.WORKLOADS["tiny"]
    case = Case(wl, pow2=True)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    assert act["pow2_scales"] and float(act["S_delta"]) == 2.0 ** round(np.log2(act["S_delta"]))
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K))
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N)))


def test_single_read_with_fp8_product(env):
    """Both options together: single-read quantiser and the FP8 kernel-token product."""
    dq, torch = env
    wl = dict(SMALL)["ragged_122"]
    case = Case(wl, pow2=True, fp8_product=True)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    assert_kernel_term_close(g["p"], act, wq, np.arange(g["layout"].K))
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N)))


def _spiky(wl, seed=5):
    """Low-amplitude activations with large outliers in the last frame's last 64 channels: every
    other 64-channel chunk's own power-of-two scale lies about 20 binades below the final one, so
    the fix-up pass must encode their groups again (E4M3's exponent field has no such headroom)."""
    x = oracle.bf16_value(synth.activations(wl, seed=seed)).astype(np.float64) * 1e-4
    last = np.arange((wl.T - 1) * wl.H * wl.W, wl.N)
    sign = np.where(np.arange(64) % 2 == 0, 1.0, -1.0)
    x[np.ix_(last, np.arange(wl.Ci - 64, wl.Ci))] = sign[None, :] * (500.0 + 7.0 * (last[:, None] % 13))
    return oracle.bf16_round_fast(x)


def test_single_read_reencodes_groups_without_headroom(env):
    """The fix-up pass's re-encode branch, forced: after the statistics pass alone,
    many groups have provisional scale codes whose exponent field is below the shift
    j + 1; after the encode stage every tensor equals the oracle's direct encode."""
    dq, torch = env
    wl = dict(SMALL)["ragged_122"]
    case = Case(wl, X=_spiky(wl), pow2=True)
    act, wq = case.run_oracle()
    g1 = case.run_gpu(dq, torch, stage_mask=dq.DQ_STAGE_STATS)
    es = int(round(np.log2(act["S_delta"])))
    prov = g1["prov"].astype(int)                              # N x Ci/64, cube-major rows
    codes = g1["dscales"].astype(int)                          # provisional, N x Ci/16
    j = es - np.repeat(prov, 4, axis=1)
    need = (np.repeat(prov, 4, axis=1) != -128) & (codes != 0) & (((codes >> 3) & 15) < j + 1)
    assert need.sum() > 100, int(need.sum())
    g = case.run_gpu(dq, torch)
    compare_quantised(g, act, wq)
    assert_y_close(g["Y"], case.oracle_rows(act, wq, np.arange(wl.N)))


def test_worked_example_through_gpu(env):
    """The hand-derived example (tests/golden) padded to 256 channels with zeros."""
    dq, torch = env
    g = json.load(open(os.path.join(HERE, "golden", "worked_cube_1x2x2.json")))
    X = np.zeros((4, 256), np.uint16)
    X[:, :16] = np.array(g["X_bf16"], np.uint16)
    wl = synth.Workload("worked", 1, 2, 2, 256, 256, 16, (1, 2, 2), (1, 1, 1), (0.0, 1.0), (0.0, 1.0))
    case = Case(wl, X=X, Wb=synth.normal_bf16((256, 256), sd=1 / 16, seed=5))
    out = case.run_gpu(dq, torch)
    assert out["status"] == 0
    assert np.array_equal(out["q8"][0, :16], np.array(g["q8"], np.uint8))
    assert not out["q8"][0, 16:].any()
    assert out["s8"][0] == np.float32(g["s8"])
    assert out["S_delta"] == np.float32(g["S_delta"])
    assert np.array_equal(out["dscales"][:, 0], np.array(g["dscales"], np.uint8))
    assert np.array_equal(out["dcodes"][:, :8], np.array(g["dcodes"], np.uint8))
    assert not out["dcodes"][:, 8:].any() and not out["dscales"][:, 1:].any()


def test_entry_points_agree(env):
    """dq_linear_forward (library workspace), _ex (caller workspace) and _host
    (host buffers, copies on the stream) give identical Y bits; two runs are
    bitwise deterministic."""
    dq, torch = env
    wl = SMALL[1][1]
    case = Case(wl)
    g = case.run_gpu(dq, torch)
    g2 = case.run_gpu(dq, torch)
    assert np.array_equal(g["Y"], g2["Y"])
    t, h, w = case.cube
    packed, L1m, L2s, _ = dq.dq_pack_weight_factors(case.Wb, case.L1, case.L2)
    dev = torch.device("cuda")
    Xd = torch.from_numpy(case.X.view(np.int16)).to(dev)
    Pd, L1d, L2d = (torch.from_numpy(a).to(dev) for a in (packed, L1m.view(np.int16), L2s.view(np.int16)))
    Yd = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=dev)
    st = torch.cuda.current_stream()
    dq.dq_linear_forward(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, st)
    torch.cuda.synchronize()
    assert dq.dq_read_device_status(None, st, clear=True) == 0
    assert np.array_equal(Yd.cpu().numpy().view(np.uint16), g["Y"])
    Xh = torch.from_numpy(case.X.view(np.int16)).pin_memory()
    Yh = torch.empty((wl.N, wl.Co), dtype=torch.int16).pin_memory()
    nbytes = dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    Xd2 = torch.empty_like(Xd)
    Yd2 = torch.empty_like(Yd)
    dq.dq_linear_forward_host(Xh, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yh, Xd2, Yd2, ws,
                              nbytes, st)
    torch.cuda.synchronize()
    assert np.array_equal(Yh.numpy().view(np.uint16), g["Y"])


@pytest.mark.parametrize("name", ["ragged_122", "ragged_222", "cube_414_r128", "cube_428", "tiny"])
def test_host_entry_point_pipeline(env, name):
    """The host-buffer entry point copies X in T-slabs overlapped with the statistics pass
    and copies finished frames of Y back while later row tiles compute: Y bit-identical to
    the device-buffer entry point's, for slabs of 1-, 2- and 4-frame cube layers, a ragged
    last layer, and a layer of one cube layer (no pipelining)."""
    dq, torch = env
    wl = dict(SMALL)[name] or synth.WORKLOADS["tiny"]
    case = Case(wl)
    g = case.run_gpu(dq, torch)
    t, h, w = case.cube
    Xd, Pd, L1d, L2d, _ = case.last_inputs
    Xh = torch.from_numpy(case.X.view(np.int16)).pin_memory()
    Yh = torch.full((wl.N, wl.Co), 0x7FC0, dtype=torch.int16).pin_memory()
    nbytes = dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=Xd.device)
    Xd2, Yd2 = torch.empty_like(Xd), torch.empty((wl.N, wl.Co), dtype=torch.int16, device=Xd.device)
    st = torch.cuda.current_stream()
    for _ in range(2):   # the second call reuses the copy streams and events
        dq.dq_linear_forward_host(Xh, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yh, Xd2, Yd2,
                                  ws, nbytes, st)
        st.synchronize()
        assert np.array_equal(Yh.numpy().view(np.uint16), g["Y"])
        assert dq.dq_read_device_status(ws, st, clear=True) == 0


def test_host_entry_point_overlapping_calls(env):
    """Back-to-back host-buffer calls with DQ_HOST_OVERLAP_PREVIOUS on one X_dev / Y_dev
    and different inputs: the second call's copy of X overlaps the first call's
    products and copy out, and each call's Y equals the device-buffer entry point's
    for its own input."""
    dq, torch = env
    wl = dict(SMALL)["ragged_122"]
    cases = [Case(wl), Case(wl, seed=99)]
    refs = [c.run_gpu(dq, torch)["Y"] for c in cases]
    t, h, w = cases[0].cube
    _, Pd, L1d, L2d, _ = cases[0].last_inputs
    Xhs = [torch.from_numpy(c.X.view(np.int16)).pin_memory() for c in cases]
    Yhs = [torch.full((wl.N, wl.Co), 0x7FC0, dtype=torch.int16).pin_memory() for _ in cases]
    nbytes = dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank)
    dev = torch.device("cuda")
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    Xd = torch.empty((wl.N, wl.Ci), dtype=torch.int16, device=dev)
    Yd = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=dev)
    st = torch.cuda.current_stream()
    for _ in range(2):
        for i in range(2):
            dq.dq_linear_forward_host_ex(Xhs[i], wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d,
                                         Yhs[i], Xd, Yd, ws, nbytes, dq.DQ_HOST_OVERLAP_PREVIOUS, st)
        st.synchronize()
        # the packed weight is the first case's; the second case's reference used its own weight, so
        # compare the second call against a device-buffer run of its X with the first case's weight
        assert np.array_equal(Yhs[0].numpy().view(np.uint16), refs[0])
        Xd2 = torch.from_numpy(cases[1].X.view(np.int16)).to(dev)
        Y2 = torch.empty_like(Yd)
        dq.dq_linear_forward_ex(Xd2, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Y2, ws, nbytes,
                                dq.DQ_STAGE_ALL, None, st)
        st.synchronize()
        assert np.array_equal(Yhs[1].numpy().view(np.uint16), Y2.cpu().numpy().view(np.uint16))
        assert dq.dq_read_device_status(ws, st, clear=True) == 0


def test_stage_mask_reuses_workspace(env):
    """Running the three stages as three calls on one workspace equals one call."""
    dq, torch = env
    wl = synth.WORKLOADS["tiny"]
    case = Case(wl)
    full = case.run_gpu(dq, torch)
    t, h, w = case.cube
    packed, L1m, L2s, _ = dq.dq_pack_weight_factors(case.Wb, case.L1, case.L2)
    dev = torch.device("cuda")
    Xd = torch.from_numpy(case.X.view(np.int16)).to(dev)
    Pd, L1d, L2d = (torch.from_numpy(a).to(dev) for a in (packed, L1m.view(np.int16), L2s.view(np.int16)))
    Yd = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=dev)
    nbytes = dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    for m in (1, 2, 4):
        dq.dq_linear_forward_ex(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws, nbytes, m,
                                None, st)
    torch.cuda.synchronize()
    assert np.array_equal(Yd.cpu().numpy().view(np.uint16), full["Y"])


def test_bad_packed_weight_is_reported(env):
    dq, torch = env
    case = Case(synth.WORKLOADS["tiny"])

    def corrupt(p):
        p = p.copy()
        p[0] ^= 0xFF          # magic
        return p

    out = case.run_gpu(dq, torch, packed_override=corrupt)
    assert out["status"] == dq.DQ_ERR_BAD_PACKED_WEIGHT


def test_bounded_wait_times_out_and_context_survives(env):
    dq, torch = env
    st = torch.cuda.current_stream()
    assert dq.dq_selftest_bounded_wait(2000, st) == dq.DQ_ERR_DEVICE_TIMEOUT
    # the context is still usable: a normal layer runs and is correct
    test_parity_small(env, "tiny", None)


def test_quotient_path_matches_ieee_division(env):
    """The quantisers' reciprocal + FMA-correction quotient equals IEEE
    division bit for bit (Markstein's correction theorem), on 2^28 pairs."""
    dq, torch = env
    bad, first = dq.dq_selftest_divide(1 << 28, seed=12345, stream=torch.cuda.current_stream())
    assert bad == 0, (bad, first)


# ------------------------------------------------------------------ feed-forward block (producer-epilogue fusion)

FFN = [
    # name, T, H, W, cube_up, cube_down, Ci, Cf, Co, rank_up, rank_down, statistics fused
    ("ragged_222_122", 3, 5, 12, (2, 2, 2), (1, 2, 2), 256, 512, 256, 32, 32, True),
    ("same_cube_122", 4, 8, 8, (1, 2, 2), (1, 2, 2), 512, 256, 512, 16, 32, True),
    ("nested_224_114", 5, 6, 16, (2, 2, 4), (1, 1, 4), 256, 256, 512, 32, 16, True),
    ("unit_cubes", 3, 7, 9, (1, 1, 1), (1, 1, 1), 256, 512, 256, 32, 32, True),
    ("cube_32_tokens", 4, 4, 16, (2, 2, 8), (2, 2, 8), 256, 256, 256, 16, 16, True),
    ("multi_tile", 6, 16, 24, (2, 2, 2), (1, 2, 2), 512, 1024, 512, 32, 32, True),
    # partitions the epilogue cannot serve: the down-projection runs its own statistics pass
    ("not_nested", 4, 8, 8, (1, 2, 2), (2, 1, 1), 256, 256, 256, 32, 32, False),
    ("straddling", 5, 7, 9, (2, 2, 2), (2, 2, 2), 256, 256, 256, 16, 16, False),
    ("cube_64_tokens", 8, 6, 16, (4, 2, 8), (4, 2, 8), 256, 256, 256, 16, 16, False),
]


@pytest.mark.parametrize("name,T,H,W,cu,cd,Ci,Cf,Co,ru,rd,fused", FFN, ids=[c[0] for c in FFN])
def test_parity_ffn_block(env, name, T, H, W, cu, cd, Ci, Cf, Co, ru, rd, fused):
    """dq_ffn_forward against the oracle: the hidden activation within the GELU-carried
    tolerance; the down-projection's cube means (formed in the up-projection's epilogue
    when `fused`), its quantised tensors bit for bit and its Y within tolerance; and
    the same Hid and Y bits as the unfused path and as the up-projection alone with
    the GELU epilogue."""
    from ffn_case import FfnCase
    dq, torch = env
    case = FfnCase(name, T, H, W, cu, cd, Ci, Cf, Co, ru, rd)
    assert case.fused_expected(dq) == fused
    g = case.run_gpu(dq, torch, gelu_layer=True)
    case.check(g)
    assert np.array_equal(g["H"], g["H_layer"]), "the GELU epilogue of the layer alone"
    s = case.run_gpu(dq, torch, ffn_flags=dq.DQ_FFN_SEPARATE_STATISTICS)
    assert s["status"] == 0 and s["status_up"] == 0
    for key in ("H", "Y", "means", "q8", "s8", "dcodes"):
        assert np.array_equal(g[key], s[key]), key


@pytest.mark.parametrize("fp8,kgroup_down", [(True, 0), (False, 64)], ids=["fp8_products", "group64_down"])
def test_parity_ffn_block_options(env, fp8, kgroup_down):
    """dq_ffn_forward_opts: the FP8 kernel-token product in both layers (restricted-scale
    weights), or one kernel scale per 64 channels in the down-projection, with the statistics
    fused; the same oracle checks, and the same bits as the unfused path."""
    from ffn_case import FfnCase
    dq, torch = env
    case = FfnCase("opts_222_122", 3, 6, 16, (2, 2, 2), (1, 2, 2), 256, 512, 256, 32, 16, fp8=fp8,
                   kgroup_down=kgroup_down)
    assert case.fused_expected(dq)
    g = case.run_gpu(dq, torch, gelu_layer=True)
    case.check(g)
    assert np.array_equal(g["H"], g["H_layer"])
    s = case.run_gpu(dq, torch, ffn_flags=dq.DQ_FFN_SEPARATE_STATISTICS)
    for key in ("H", "Y", "q8", "s8", "dcodes"):
        assert np.array_equal(g[key], s[key]), key


def test_parity_ffn_block_with_biases(env):
    """The feed-forward block with a linear bias in both layers (added once per cube in
    each layer's kernel term, so GELU sees y + b)."""
    from ffn_case import FfnCase
    dq, torch = env
    case = FfnCase("bias_222_122", 3, 6, 16, (2, 2, 2), (1, 2, 2), 256, 512, 256, 32, 16, bias=True)
    assert case.fused_expected(dq)
    g = case.run_gpu(dq, torch)
    case.check(g)


def test_forward_replays_from_a_cuda_graph(env):
    """The layer captured into a CUDA graph (every launch and memset of a call is a stream
    operation on the caller's stream): replays give the eager bits, with new inputs copied
    into the captured buffers between replays."""
    dq, torch = env
    wl = _wl("graph_122", 3, 10, 37, 512, 512, 32, (1, 2, 2))
    case = Case(wl)
    eager = case.run_gpu(dq, torch)
    Xd, Pd, L1d, L2d, Yd = case.last_inputs
    ws, lay = case.last_ws, case.last_layout
    t, h, w = case.cube
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm-up on the capture stream (first-use attribute calls)
        dq.dq_linear_forward_ex(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws,
                                lay.total_bytes, dq.DQ_STAGE_ALL, None, s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        dq.dq_linear_forward_ex(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws,
                                lay.total_bytes, dq.DQ_STAGE_ALL, None, s)
    X2 = synth.activations(wl, tau=3)
    for X_in in (X2, case.X):
        Xd.copy_(torch.from_numpy(X_in.view(np.int16)))
        Yd.zero_()
        graph.replay()
        torch.cuda.synchronize()
        if X_in is case.X:
            assert np.array_equal(Yd.cpu().numpy().view(np.uint16), eager["Y"])
    assert dq.dq_read_device_status(ws, torch.cuda.current_stream(), clear=True) == 0
    # the second replay ran on other inputs first: compare it with an eager call on them
    Xd.copy_(torch.from_numpy(X2.view(np.int16)))
    graph.replay()
    torch.cuda.synchronize()
    y_graph = Yd.cpu().numpy().copy()
    dq.dq_linear_forward_ex(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws,
                            lay.total_bytes, dq.DQ_STAGE_ALL, None, torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert np.array_equal(Yd.cpu().numpy(), y_graph)
    del graph


def test_device_gelu_error_bound(env):
    """The feed-forward epilogue's GELU (Abramowitz & Stegun 7.1.26 erfc with the hardware's
    approximate reciprocal and 2^x, in fp32) against the oracle's exact-form GELU in fp64:
    |error| <= 3e-7 max(1, |y|) over a dense grid, a wide normal sample and the extremes."""
    dq, torch = env
    rng = np.random.default_rng(11)
    y = np.concatenate([np.linspace(-12.0, 12.0, 480001), rng.normal(0.0, 8.0, 200000),
                        [0.0, -0.0, 1e-30, -1e-30, 40.0, -40.0, 1e3, -1e3, 6.5, -6.5]]).astype(np.float32)
    dev = torch.device("cuda")
    yd = torch.from_numpy(y).to(dev)
    out = torch.empty_like(yd)
    dq.dq_selftest_gelu(yd, y.size, out, torch.cuda.current_stream())
    torch.cuda.synchronize()
    h = out.cpu().numpy().astype(np.float64)
    ref = oracle.gelu_erf(y.astype(np.float64))
    err = np.abs(h - ref) / np.maximum(1.0, np.abs(y.astype(np.float64)))
    assert np.all(np.isfinite(h))
    assert err.max() <= 3e-7, (float(err.max()), float(y[np.argmax(err)]))
