"""GPU parity at the full Wan-like sizes, in the launch configuration the bench
times.  Every quantised tensor is compared in full and bit-exact: the delta
codes and scales, S_delta, the kernel tokens (E4M3 codes, their scales and
their BF16 copy), and the packed weight's residual codes, group scales (all
four per-quadrant copies of each) and S_W.  The kernel term P' (the
kernel-token product, K x Co fp32) and Y are compared on sampled cubes
(random interior cubes plus the first, last and ragged-edge cubes), which the
oracle computes one by one in fp64: P' within the fp32-accumulation bound, Y
within max(1 BF16 ulp, 1e-3 RMS).

Per-case records (errors against tolerance, and for the sweep the relative
errors) are written as JSON to the directory named by DQ_RECORD_DIR when it is
set.

The cube-size sweep on the 480p shape also records the relative Frobenius
error of Y against the unquantised product X W^T, next to plain per-token
NVFP4 (no kernel/delta split), and checks the method's claim that the split
lowers it (DeltaQuant note, key design 2 and the cube-size ablation)."""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from dq_case import Case, assert_kernel_term_close, assert_y_close, bf16_bits_to_f64, compare_quantised

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module")
def env():
    import torch
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    import video_diffusion_w4a4_b200 as dq
    return dq, torch


def sample_cubes(wl, cube, n_cubes=48, seed=0):
    """Seeded interior cubes plus the first, the last and up to eight ragged edge
    cubes, and the natural token rows they hold."""
    o = oracle.cube_order(wl.T, wl.H, wl.W, *cube)
    K = o["count"].size
    rng = np.random.default_rng(seed)
    ks = set(rng.choice(K, size=min(n_cubes, K), replace=False).tolist())
    ks |= {0, K - 1}
    ks |= set(np.flatnonzero(o["count"] < o["count"].max())[:8].tolist())   # ragged edge cubes
    ks = np.array(sorted(ks), np.int64)
    rows = np.concatenate([o["n_of_row"][o["first"][k]:o["first"][k] + o["count"][k]] for k in ks])
    return ks, np.sort(rows)


def _record(name, info):
    out = os.environ.get("DQ_RECORD_DIR")
    if not out:
        return
    os.makedirs(out, exist_ok=True)
    with open(os.path.join(out, f"parity_{name}.json"), "w") as f:
        json.dump(info, f, indent=1)


@pytest.mark.parametrize("name", ["wan480p_proj", "wan720p_ffn_up", "wan720p_ffn_down"])
def test_full_size(env, name):
    dq, torch = env
    wl = synth.WORKLOADS[name]
    case = Case(wl)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    ks, rows = sample_cubes(wl, case.cube)
    pinfo = assert_kernel_term_close(g["p"], act, wq, ks)
    info = assert_y_close(g["Y"][rows], case.oracle_rows(act, wq, rows))
    info.update(rows=int(rows.size), N=wl.N, K=int(g["layout"].K), cubes=int(ks.size),
                p_max_err_over_tol=pinfo["max_err_over_tol"], p_max_rel_err=pinfo["max_rel_err"])
    _record(name, info)


@pytest.mark.parametrize("cube", [(1, 1, 1), (1, 2, 2), (2, 2, 2), (2, 4, 4), (4, 1, 4), (4, 2, 8), (21, 30, 52)])
def test_cube_sweep(env, cube):
    dq, torch = env
    wl = synth.WORKLOADS["wan480p_cube_sweep"].with_cube(cube)
    case = Case(wl)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    ks, rows = sample_cubes(wl, cube, n_cubes=32)
    assert_kernel_term_close(g["p"], act, wq, ks)
    y_ref = case.oracle_rows(act, wq, rows)
    info = assert_y_close(g["Y"][rows], y_ref)
    # error against the unquantised product, next to plain per-token NVFP4
    x = oracle.bf16_value(case.X[rows]).astype(np.float64)
    w = oracle.bf16_value(case.Wb).astype(np.float64)
    exact = x @ w.T
    plain = oracle.quantize_plain(case.X[rows])
    plain.update(row_of_n=None, cube_of_n=None, q8=None, s8=None)
    y_plain = oracle.output_rows(plain, wq, case.X[rows], case.L1, case.L2, np.arange(rows.size), kernel=False,
                                 cube_major=False)
    rel = lambda y: float(np.linalg.norm(y - exact) / np.linalg.norm(exact))
    info.update(cube=list(cube), rel_err_gpu=rel(bf16_bits_to_f64(g["Y"][rows])), rel_err_oracle=rel(y_ref),
                rel_err_plain_nvfp4=rel(y_plain))
    # the same 512 seeded token rows for every cube, so that the errors compare across cube sizes
    fixed = np.sort(np.random.default_rng(2026).choice(wl.N, size=512, replace=False))
    xf = oracle.bf16_value(case.X[fixed]).astype(np.float64)
    exact_f = xf @ w.T
    relf = lambda y: float(np.linalg.norm(y - exact_f) / np.linalg.norm(exact_f))
    plain_f = oracle.quantize_plain(case.X[fixed])
    plain_f.update(row_of_n=None, cube_of_n=None, q8=None, s8=None)
    y_plain_f = oracle.output_rows(plain_f, wq, case.X[fixed], case.L1, case.L2, np.arange(fixed.size), kernel=False,
                                   cube_major=False)
    info.update(fixed_rows=int(fixed.size), rel_err_gpu_fixed=relf(bf16_bits_to_f64(g["Y"][fixed])),
                rel_err_plain_nvfp4_fixed=relf(y_plain_f))
    _record("sweep_%d%d%d" % cube, info)
    if cube not in ((1, 1, 1), (21, 30, 52)):
        # local cubes beat plain FP4 (the note's cube-size ablation: the global kernel loses the local structure)
        assert info["rel_err_gpu"] < info["rel_err_plain_nvfp4"], info


@pytest.mark.parametrize("cube", [(1, 2, 2), (4, 2, 8)])
def test_full_size_group64_kernel_scales(env, cube):
    """The 480p projection with one FP8 kernel scale per 64 channels (the note's
    per-group kernel quantisation), at the bench's cube and at the note's
    64-token cube."""
    dq, torch = env
    wl = synth.WORKLOADS["wan480p_cube_sweep"].with_cube(cube)
    case = Case(wl, kernel_group=64)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    ks, rows = sample_cubes(wl, cube, n_cubes=32)
    assert_kernel_term_close(g["p"], act, wq, ks, extra_rel=2.0 ** -16)
    info = assert_y_close(g["Y"][rows], case.oracle_rows(act, wq, rows))
    info.update(cube=list(cube), kernel_group=64, rows=int(rows.size))
    _record("group64_%d%d%d" % cube, info)


@pytest.mark.parametrize("name,fp8,pow2", [("wan720p_ffn_down", True, False), ("wan480p_proj", True, False),
                                           ("wan480p_proj", False, True), ("wan720p_ffn_up", True, True)],
                         ids=["ffn_down_fp8", "proj_fp8", "proj_single_read", "ffn_up_fp8_single_read"])
def test_full_size_options(env, name, fp8, pow2):
    """The layer's options at full size: the FP8-rate kernel-token product on
    restricted-scale (C2) weights and the single-read quantiser (power-of-two
    S_delta).  Every quantised tensor and the packed C2 weight bit-exact against
    the oracle's option, P' and Y on sampled cubes within tolerance."""
    dq, torch = env
    wl = synth.WORKLOADS[name]
    case = Case(wl, fp8_product=fp8, pow2=pow2)
    g = case.run_gpu(dq, torch)
    act, wq = case.run_oracle()
    compare_quantised(g, act, wq)
    ks, rows = sample_cubes(wl, case.cube, n_cubes=32)
    pinfo = assert_kernel_term_close(g["p"], act, wq, ks)
    info = assert_y_close(g["Y"][rows], case.oracle_rows(act, wq, rows))
    info.update(rows=int(rows.size), fp8_product=fp8, pow2=pow2, p_max_err_over_tol=pinfo["max_err_over_tol"])
    _record(f"options_{name}_{int(fp8)}{int(pow2)}", info)


def test_full_size_host_entry_point(env):
    """The end-to-end path the bench times, at the 720p FFN down-projection: pinned X in
    T-slabs, the statistics pass per slab, Y's finished frames back per range of row
    tiles, and a second call overlapping the first (DQ_HOST_OVERLAP_PREVIOUS); both
    calls' Y bit-identical to the device-buffer entry point's."""
    dq, torch = env
    wl = synth.WORKLOADS["wan720p_ffn_down"]
    case = Case(wl)
    g = case.run_gpu(dq, torch)
    t, h, w = case.cube
    _, Pd, L1d, L2d, _ = case.last_inputs
    dev = torch.device("cuda")
    Xh = torch.from_numpy(case.X.view(np.int16)).pin_memory()
    Yhs = [torch.empty((wl.N, wl.Co), dtype=torch.int16).pin_memory() for _ in range(2)]
    nbytes = dq.dq_workspace_bytes(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    Xd = torch.empty((wl.N, wl.Ci), dtype=torch.int16, device=dev)
    Yd = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=dev)
    st = torch.cuda.current_stream()
    for i in range(2):
        dq.dq_linear_forward_host_ex(Xh, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yhs[i], Xd,
                                     Yd, ws, nbytes, dq.DQ_HOST_OVERLAP_PREVIOUS if i else 0, st)
    st.synchronize()
    assert dq.dq_read_device_status(ws, st, clear=True) == 0
    for i in range(2):
        assert np.array_equal(Yhs[i].numpy().view(np.uint16), g["Y"]), i


def test_full_size_ffn_block(env):
    """The 720p feed-forward block (up-projection 5120 -> 13824 at cube 2x2x2, GELU,
    down-projection 13824 -> 5120 at cube 1x2x2) through dq_ffn_forward with the
    down-projection's statistics formed in the up-projection's epilogue: the hidden
    activation and Y on sampled rows against the oracle, every quantised tensor of the
    down-projection (and its cube means) in full and bit-exact, and Hid, Y and the
    down-projection's tensors bit-identical to the unfused path."""
    from ffn_case import FfnCase
    dq, torch = env
    up, down = synth.WORKLOADS["wan720p_ffn_up"], synth.WORKLOADS["wan720p_ffn_down"]
    case = FfnCase("wan720p_ffn", up.T, up.H, up.W, up.cube, down.cube, up.Ci, up.Co, down.Co, up.rank, down.rank)
    assert case.fused_expected(dq)
    g = case.run_gpu(dq, torch)
    _, rows = sample_cubes(case.up, case.up.cube, n_cubes=24)
    info = case.check(g, rows)
    s = case.run_gpu(dq, torch, ffn_flags=dq.DQ_FFN_SEPARATE_STATISTICS)
    for key in ("H", "Y", "means", "q8", "s8", "dcodes"):
        assert np.array_equal(g[key], s[key]), key
    info.update(rows=int(rows.size), N=case.up.N)
    _record("ffn_block_720p", info)
