"""Pins for the oracle's statement of the DeltaQuant layer.

Source: papernotes.org, "DeltaQuant: 4-bit Video Diffusion Models with
Spatiotemporal Delta Smoothing", key designs 2-4 (cube partition, Eq. 1
kernel/delta split, Eq. 2-3 split product with the SVD low-rank branch,
Eq. 4 quantiser).  Every check here compares the oracle with an independent
statement: closed forms, exact fp64 invariants, brute-force assembly with a
library matmul, hand-derived worked examples, or the Eckart-Young bound.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _x_f64(X):
    return oracle.bf16_value(X).astype(np.float64)


# ------------------------------------------------------------------ cube partition (design 2)

@pytest.mark.parametrize("shape,cube", [((4, 8, 8), (1, 2, 2)), ((5, 7, 9), (2, 2, 2)), ((21, 45, 80), (2, 2, 2)),
                                        ((3, 5, 6), (1, 1, 1)), ((4, 6, 10), (4, 6, 10)), ((7, 3, 5), (2, 4, 4))])
def test_cube_order_closed_form(shape, cube):
    T, H, W = shape
    t, h, w = cube
    o = oracle.cube_order(T, H, W, t, h, w)
    N = T * H * W
    assert np.array_equal(np.sort(o["row_of_n"]), np.arange(N))
    assert np.array_equal(o["n_of_row"][o["row_of_n"]], np.arange(N))
    KT, KH, KW = -(-T // t), -(-H // h), -(-W // w)
    assert o["count"].size == KT * KH * KW == oracle.num_cubes(T, H, W, t, h, w)
    # closed form for the first row of each cube and the row of each token
    for n in range(0, N, max(1, N // 997)):
        tt, hh, ww = n // (H * W), (n // W) % H, n % W
        kt, kh, kw = tt // t, hh // h, ww // w
        st, sh, sw = min(t, T - kt * t), min(h, H - kh * h), min(w, W - kw * w)
        k = (kt * KH + kh) * KW + kw
        base = kt * t * H * W + st * (kh * h * W + sh * kw * w)
        rho = base + ((tt - kt * t) * sh + (hh - kh * h)) * sw + (ww - kw * w)
        assert o["cube_of_n"][n] == k
        assert o["first"][k] == base
        assert o["row_of_n"][n] == rho
        assert o["count"][k] == st * sh * sw


# ------------------------------------------------------------------ Eq. 1

@pytest.mark.parametrize("cube", [(1, 2, 2), (2, 2, 2), (2, 4, 4)])
def test_eq1_fp64_split_is_exact_for_power_of_two_cubes(cube):
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    mean, delta = oracle.cube_split_f64(X, wl.T, wl.H, wl.W, cube)
    o = oracle.cube_order(wl.T, wl.H, wl.W, *cube)
    x = _x_f64(X)
    # kernel + delta reconstructs X exactly
    assert np.array_equal(mean[o["cube_of_n"]] + delta, x)
    # deltas sum to zero per cube, exactly (power-of-two counts)
    sums = np.zeros_like(mean)
    np.add.at(sums, o["cube_of_n"], delta)
    assert np.all(o["count"] & (o["count"] - 1) == 0)
    assert np.array_equal(sums, np.zeros_like(sums))


def test_eq1_ragged_cubes_mean_over_present_tokens():
    T, H, W = 3, 5, 7
    X = synth.normal_bf16((T * H * W, 32), sd=3.0, seed=11)
    mean, delta = oracle.cube_split_f64(X, T, H, W, (2, 2, 2))
    o = oracle.cube_order(T, H, W, 2, 2, 2)
    x = _x_f64(X)
    for k in range(o["count"].size):
        rows = o["n_of_row"][o["first"][k]:o["first"][k] + o["count"][k]]
        np.testing.assert_allclose(mean[k], x[rows].mean(axis=0), rtol=0, atol=1e-12)
        assert np.abs(delta[rows].sum(axis=0)).max() < 1e-12
    assert sorted(set(o["count"].tolist())) == [1, 2, 4, 8]


def test_fp32_means_within_rounding_of_exact():
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    m32 = oracle.cube_means(X, wl.T, wl.H, wl.W, wl.cube).astype(np.float64)
    m64, _ = oracle.cube_split_f64(X, wl.T, wl.H, wl.W, wl.cube)
    # 3 sequential adds + 1 division, each within half an ulp of its result
    bound = 4 * np.spacing(np.abs(m64).astype(np.float32).astype(np.float64) * 4 + 1e-30)
    assert np.all(np.abs(m32 - m64) <= bound)


def test_mean_is_sequential_fp32_sum_in_thw_order():
    # hand-derived: a cube whose tokens, in (t,h,w) order, carry 2^30, 1, -2^30, 1
    # in channel 0.  Summed one at a time in fp32: (0+2^30)+1 = 2^30 (the 1 is
    # below half an ulp of 2^30), then 0, then 1; mean = 1/4.  Any other order
    # or an fp64 sum would give 1/2.
    T, H, W, Ci = 1, 2, 2, 16
    vals = np.array([2.0 ** 30, 1.0, -(2.0 ** 30), 1.0])
    Xf = np.zeros((4, Ci))
    Xf[:, 0] = vals
    X = oracle.bf16_round_fast(Xf)
    m = oracle.cube_means(X, T, H, W, (1, 2, 2))
    assert m[0, 0] == np.float32(0.25)
    # the same tokens stored in another (t,h,w) arrangement change the order
    Y = X[[0, 2, 1, 3]]          # tokens now visited as 2^30, -2^30, 1, 1
    assert oracle.cube_means(Y, T, H, W, (1, 2, 2))[0, 0] == np.float32(0.5)


# ------------------------------------------------------------------ Eq. 4 quantiser

def test_fp4_reproduces_exact_grid_values():
    rng = np.random.default_rng(2)
    rows, cols = 64, 256
    S = 2.0 ** -7
    mags = oracle.e2m1_value(np.arange(8))
    e4 = oracle.e4m3_value(np.arange(1, 127))
    # each block: scale s_b on the E4M3 grid, codes anywhere, one element = +-6
    sb = rng.choice(e4[(e4 >= 2.0 ** -6) & (e4 <= 448)], size=(rows, cols // 16))
    q = rng.choice(np.concatenate([mags, -mags[1:]]), size=(rows, cols))
    q[:, ::16] = 6.0 * rng.choice([-1, 1], size=(rows, cols // 16))
    sb[0, 0] = 448.0
    Z = (q * np.repeat(sb, 16, axis=1) * S)
    assert np.array_equal(Z.astype(np.float32).astype(np.float64), Z)
    codes, scales, S_out = oracle.fp4_quantize(Z.astype(np.float32))
    # S = amax / (6*448) = (6*448*S)/(6*448)
    assert S_out == S
    assert np.array_equal(oracle.e4m3_value(scales), sb)
    lo, hi = codes & 15, codes >> 4
    dq = np.empty((rows, cols))
    dq[:, 0::2], dq[:, 1::2] = oracle.e2m1_value(lo), oracle.e2m1_value(hi)
    assert np.array_equal(dq, q)


def test_fp4_amax_maps_to_qmax():
    # Eq. 4: s = max|X| / q_max, so the largest element lands on q_max = 6
    Z = synth.normal_bf16((32, 128), sd=2.0, seed=4)
    Zf = oracle.bf16_value(Z)
    codes, scales, S = oracle.fp4_quantize(Zf)
    i = np.unravel_index(np.argmax(np.abs(Zf)), Zf.shape)
    code = (codes[i[0], i[1] // 2] >> (4 * (i[1] % 2))) & 15
    assert abs(oracle.e2m1_value([code])[0]) == 6.0
    assert oracle.e4m3_value([scales[i[0], i[1] // 16]])[0] == 448.0
    assert S == np.float32(np.abs(Zf).max()) / np.float32(2688.0)


def test_fp4_monotone_and_bounded_error():
    rng = np.random.default_rng(9)
    base = rng.standard_normal((1, 16)).astype(np.float32)
    sweep = np.linspace(-3, 3, 4001).astype(np.float32)
    Z = np.repeat(base, sweep.size, axis=0)
    Z[:, 5] = sweep
    codes, scales, S = oracle.fp4_quantize(Z, S=2.0 ** -6)
    c5 = (codes[:, 2] >> 4) & 15
    dq = oracle.e2m1_value(c5) * oracle.e4m3_value(scales[:, 0]) * S
    # blocks whose scale did not change must be monotone in the swept element
    for s in np.unique(scales[:, 0]):
        sel = scales[:, 0] == s
        assert np.all(np.diff(dq[sel]) >= 0)
    # element error at most half the coarsest step (2 * s_b * S) of its block
    err = np.abs(dq - sweep)
    assert np.all(err <= oracle.e4m3_value(scales[:, 0]) * S * 1.0 + 1e-12)


def test_worked_example_eq1_eq4():
    """Hand-derived example: one 1x2x2 cube of 16 channels.

    Tokens in (t,h,w) order carry d = (3, -1, 1, -3);  x[n][c] = m_c + d_n g_c with
      c = 0..7:   m_c = c/2, g_c = 1/16
      c = 8..14:  m_c = 1,   g_c = 7/64
      c = 15:     m_c = 14,  g_c = 0
    Every x is exact in BF16 and every partial sum exact in fp32, so:
      kernel token = m; max|m| = 14 -> s8 = 14/448 = 2^-5; q8 = E4M3(32 m) exactly
        (0,16,32,48,64,80,96,112 | 32 | 448);
      deltas d g; global amax = 3 * 7/64 = 21/64 -> S = (21/64)/2688 = 2^-13;
      tokens 0, 3 (|d| = 3): block amax 21/64, (21/64)/(6 * 2^-13) = 448 -> s_b = 448,
        eff = 448 * 2^-13 = 7/128; c < 8: (3/16)/(7/128) = 24/7 = 3.43 -> 3;
        c = 8..14: exactly 6; c = 15: +0;
      tokens 1, 2 (|d| = 1): block amax 7/64, (7/64)/(6 * 2^-13) = 448/3 = 149.3
        -> E4M3 144 (160 is farther), eff = 144 * 2^-13 = 9/512;
        c < 8: (1/16)/(9/512) = 3.56 -> 4 (past the 3.5 midpoint);
        c = 8..14: 7/64 / (9/512) = 6.22 -> 6 (saturated); c = 15: +0.
    """
    Ci = 16
    m = np.array([c / 2 for c in range(8)] + [1.0] * 7 + [14.0])
    g = np.array([1 / 16] * 8 + [7 / 64] * 7 + [0.0])
    d = np.array([3.0, -1.0, 1.0, -3.0])
    Xf = m[None, :] + d[:, None] * g[None, :]
    X = oracle.bf16_round_fast(Xf)
    assert np.array_equal(oracle.bf16_value(X).astype(np.float64), Xf)
    act = oracle.quantize_activations(X, 1, 2, 2, (1, 2, 2))
    assert np.array_equal(act["means"][0].astype(np.float64), m)
    assert act["s8"][0] == np.float32(2.0 ** -5)
    assert np.array_equal(oracle.e4m3_value(act["q8"][0]), 32 * m)
    assert act["amax_delta"] == np.float32(21 / 64)
    assert act["S_delta"] == np.float32(2.0 ** -13)
    assert list(oracle.e4m3_value(act["dscales"][:, 0])) == [448.0, 144.0, 144.0, 448.0]
    codes = act["dcodes"]
    got = np.empty((4, Ci), dtype=np.int64)
    got[:, 0::2], got[:, 1::2] = codes & 15, codes >> 4
    want = np.zeros((4, Ci), dtype=np.int64)
    for n, (lo, mid) in enumerate([(5, 7), (8 | 6, 8 | 7), (6, 7), (8 | 5, 8 | 7)]):
        want[n, :8], want[n, 8:15], want[n, 15] = lo, mid, 0
    assert np.array_equal(got, want)


# ------------------------------------------------------------------ Eq. 2 / Eq. 3 assembly

def _dequant_rows(codes, scales, S):
    rows, half = codes.shape
    v = np.empty((rows, half * 2))
    v[:, 0::2] = oracle.e2m1_value(codes & 15)
    v[:, 1::2] = oracle.e2m1_value(codes >> 4)
    return v * np.repeat(oracle.e4m3_value(scales), 16, axis=1) * S


@pytest.fixture(scope="module")
def tiny_case():
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    Wb = synth.weight(wl)
    L1, L2, sig = oracle.lowrank_factors(Wb, wl.rank)
    act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube)
    wq = oracle.quantize_weight(Wb, L1, L2)
    return wl, X, Wb, L1, L2, sig, act, wq


def test_split_product_matches_brute_force(tiny_case):
    wl, X, Wb, L1, L2, sig, act, wq = tiny_case
    # A' = dq(delta) in natural order + broadcast of the dequantised kernel token
    dqd = _dequant_rows(act["dcodes"], act["dscales"], act["S_delta"])[act["row_of_n"]]
    dqk = oracle.e4m3_value(act["q8"]) * act["s8"][:, None].astype(np.float64)
    A = dqd + dqk[act["cube_of_n"]]
    dqW = _dequant_rows(wq["wcodes"], wq["wscales"], wq["S_w"])
    l1, l2 = oracle.bf16_value(L1).astype(np.float64), oracle.bf16_value(L2).astype(np.float64)
    Y_bf = A @ dqW.T + (_x_f64(X) @ l1) @ l2
    Y = oracle.output_rows(act, wq, X, L1, L2, np.arange(wl.N))
    np.testing.assert_allclose(Y, Y_bf, rtol=1e-12, atol=1e-12 * np.abs(Y_bf).max())


def test_unit_cube_has_zero_deltas_and_reduces_to_w4a8(tiny_case):
    wl, X, Wb, L1, L2, sig, _, wq = tiny_case
    act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, (1, 1, 1))
    assert act["amax_delta"] == 0.0 and act["S_delta"] == 1.0
    assert not act["dcodes"].any() and not act["dscales"].any()
    assert np.array_equal(act["row_of_n"], np.arange(wl.N))
    # per-token W4A8: q8 s8 dq(R)^T, plus the low-rank term
    x = _x_f64(X)
    s8 = np.abs(oracle.bf16_value(X)).max(axis=1) / np.float32(448.0)
    assert np.array_equal(act["s8"], s8.astype(np.float32))
    dqW = _dequant_rows(wq["wcodes"], wq["wscales"], wq["S_w"])
    q = oracle.e4m3_value(act["q8"]) * act["s8"][:, None].astype(np.float64)
    l1, l2 = oracle.bf16_value(L1).astype(np.float64), oracle.bf16_value(L2).astype(np.float64)
    Y_ref = q @ dqW.T + (x @ l1) @ l2
    Y = oracle.output_rows(act, wq, X, L1, L2, np.arange(wl.N))
    np.testing.assert_allclose(Y, Y_ref, rtol=1e-12, atol=1e-12 * np.abs(Y_ref).max())


def test_bias_special_cases(tiny_case):
    """y = x W^T + b: an all-zero X leaves exactly b in every row (every other
    term vanishes: zero kernel tokens, zero deltas, zero low-rank input), and
    the bias moves no row's three terms (an all-zero b changes nothing)."""
    wl, X, Wb, L1, L2, sig, act, wq = tiny_case
    b = synth.normal_bf16((wl.Co,), sd=3.0, seed=11)
    X0 = np.zeros_like(X)
    act0 = oracle.quantize_activations(X0, wl.T, wl.H, wl.W, wl.cube)
    Y0 = oracle.output_rows(act0, wq, X0, L1, L2, np.arange(wl.N), bias=b)
    assert np.array_equal(Y0, np.broadcast_to(oracle.bf16_value(b).astype(np.float64), Y0.shape))
    rows = np.arange(0, wl.N, 7)
    Yb = oracle.output_rows(act, wq, X, L1, L2, rows, bias=np.zeros(wl.Co, np.uint16))
    assert np.array_equal(Yb, oracle.output_rows(act, wq, X, L1, L2, rows))


def test_residual_against_library_matmul(tiny_case):
    wl, X, Wb, L1, L2, *_ = tiny_case
    R = oracle.residual(Wb, L1, L2)
    l1, l2 = oracle.bf16_value(L1).astype(np.float64), oracle.bf16_value(L2).astype(np.float64)
    ref = oracle.bf16_value(Wb).astype(np.float64) - (l1 @ l2).T
    # different fp64 summation order: at most one fp32 rounding step apart
    assert np.all(np.abs(R - ref) <= np.spacing(np.abs(ref).astype(np.float32)))


def test_lowrank_eckart_young(tiny_case):
    wl, X, Wb, L1, L2, sig, *_ = tiny_case
    w = oracle.bf16_value(Wb).astype(np.float64)
    l1, l2 = oracle.bf16_value(L1).astype(np.float64), oracle.bf16_value(L2).astype(np.float64)
    err2 = np.linalg.norm(w - (l1 @ l2).T) ** 2
    tail = np.sum(sig[wl.rank:] ** 2)
    # BF16 rounding of the factors adds at most about 2^-8 relative on L1 L2
    rnd = (2.0 ** -8 * np.linalg.norm(l1 @ l2)) ** 2
    assert err2 <= (1 + 1e-3) * tail + 4 * rnd


def test_full_rank_factors_reconstruct_w():
    Wb = synth.normal_bf16((64, 48), sd=0.1, seed=21)
    L1, L2, sig = oracle.lowrank_factors(Wb, 48)
    w = oracle.bf16_value(Wb).astype(np.float64)
    rec = (oracle.bf16_value(L1).astype(np.float64) @ oracle.bf16_value(L2).astype(np.float64)).T
    assert np.linalg.norm(w - rec) <= 2.0 ** -7 * np.linalg.norm(w)


# ------------------------------------------------------------------ the method's claim

@pytest.mark.parametrize("name,shape", [("tiny", None), ("mid", (4, 16, 16, 512, 384))])
def test_delta_split_beats_plain_fp4(name, shape):
    """Design 1/3 and the cube-size ablation: on spatially and temporally
    correlated activations, quantising deltas against a local FP8 kernel token
    gives a lower Frobenius error than per-token-group FP4 of X itself."""
    wl = synth.WORKLOADS["tiny"]
    if shape:
        T, H, W, Ci, Co = shape
        wl = synth.Workload("mid", T, H, W, Ci, Co, 16, (1, 2, 2), (T, math.ceil(H / 4), math.ceil(W / 4)),
                            (0.01, 50.0), (0.01, 20.0))
    X = synth.activations(wl, seed=77)
    Wb = synth.weight(wl, seed=78)
    L1, L2, _ = oracle.lowrank_factors(Wb, wl.rank)
    wq = oracle.quantize_weight(Wb, L1, L2)
    rows = np.arange(0, wl.N, max(1, wl.N // 256))
    ref = _x_f64(X)[rows] @ oracle.bf16_value(Wb).astype(np.float64).T
    act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube)
    y_dq = oracle.output_rows(act, wq, X, L1, L2, rows)
    plain = oracle.quantize_plain(X)
    plain.update(row_of_n=None, cube_of_n=None, q8=None, s8=None)
    y_pl = oracle.output_rows(plain, wq, X, L1, L2, rows, kernel=False, cube_major=False)
    e_dq = np.linalg.norm(y_dq - ref) / np.linalg.norm(ref)
    e_pl = np.linalg.norm(y_pl - ref) / np.linalg.norm(ref)
    assert e_dq < e_pl, (e_dq, e_pl)
    assert e_dq < 0.2


def test_delta_magnitudes_smaller_than_x():
    """Design 1: residuals against the cube mean are smaller and have fewer outliers."""
    wl = synth.WORKLOADS["tiny"]
    X = synth.activations(wl)
    _, delta = oracle.cube_split_f64(X, wl.T, wl.H, wl.W, wl.cube)
    x = _x_f64(X)
    assert np.abs(delta).max() < 0.5 * np.abs(x).max()
    assert np.sqrt((delta ** 2).mean()) < 0.2 * np.sqrt((x ** 2).mean())


def test_worked_example_fixture():
    """The hand-derived worked example stored under tests/golden (closed-form
    values written by make_worked_example.py, no oracle involved)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "worked_cube_1x2x2.json")
    g = json.load(open(path))
    X = np.array(g["X_bf16"], dtype=np.uint16)
    act = oracle.quantize_activations(X, g["T"], g["H"], g["W"], tuple(g["cube"]))
    assert np.array_equal(act["means"][0], np.array(g["means"], np.float32))
    assert act["s8"][0] == np.float32(g["s8"])
    assert np.array_equal(act["q8"][0], np.array(g["q8"], np.uint8))
    assert act["amax_delta"] == np.float32(g["amax_delta"])
    assert act["S_delta"] == np.float32(g["S_delta"])
    assert np.array_equal(act["dscales"][:, 0], np.array(g["dscales"], np.uint8))
    assert np.array_equal(act["dcodes"], np.array(g["dcodes"], np.uint8))


# ------------------------------------------------------------------ kernel-token precision variants

def test_kernel_values_route_matches_fp8_kernel_term(tiny_case):
    """The replaceable kernel term (library fp64 product of dequantised kernel
    tokens) reproduces the oracle's own C kernel term for the FP8 tokens."""
    wl, X, Wb, L1, L2, sig, act, wq = tiny_case
    rows = np.arange(wl.N)
    y_c = oracle.output_rows(act, wq, X, L1, L2, rows)
    y_v = oracle.output_rows(act, wq, X, L1, L2, rows, kernel_values=oracle.kernel_tokens_dequantized(act, "fp8"))
    np.testing.assert_allclose(y_v, y_c, rtol=1e-12, atol=1e-12 * np.abs(y_c).max())


def test_kernel_variants_exact_on_representable_means():
    """Means already on a format's grid come back unchanged: BF16 values under
    the BF16 variant; E2M1 grid values times a power of two per group under the
    NVFP4 variant (up to the fp32 rounding of the per-tensor scale)."""
    rng = np.random.default_rng(5)
    bf = synth.normal_bf16((6, 64), sd=3.0, seed=9)
    m = oracle.bf16_value(bf)
    assert np.array_equal(oracle.kernel_tokens_dequantized({"means": m}, "bf16"), m.astype(np.float64))
    grid = oracle.e2m1_value(np.arange(8))
    v = grid[rng.integers(0, 8, size=(6, 64))] * np.where(rng.random((6, 64)) < 0.5, -1.0, 1.0)
    v[:, ::16] = 6.0                                   # every group reaches the top code
    v *= np.repeat(2.0 ** rng.integers(-6, 3, size=(6, 4)), 16, axis=1)
    got = oracle.kernel_tokens_dequantized({"means": v.astype(np.float32)}, "nvfp4")
    np.testing.assert_allclose(got, v, rtol=2.0 ** -22, atol=0)


@pytest.mark.parametrize("shape", [(4, 16, 16, 512, 384), (8, 16, 24, 512, 256)])
def test_kernel_precision_ablation(shape):
    """The note's kernel-token precision ablation (16 / 8 / 4 bit) on correlated
    synthetic activations: an FP8 kernel token costs almost nothing over BF16,
    an NVFP4 one loses accuracy (relative Frobenius error of Y against the
    unquantised X W^T)."""
    T, H, W, Ci, Co = shape
    wl = synth.Workload("mid", T, H, W, Ci, Co, 16, (1, 2, 2), (T, math.ceil(H / 4), math.ceil(W / 4)),
                        (0.01, 50.0), (0.01, 20.0))
    X = synth.activations(wl, seed=77)
    Wb = synth.weight(wl, seed=78)
    L1, L2, _ = oracle.lowrank_factors(Wb, wl.rank)
    wq = oracle.quantize_weight(Wb, L1, L2)
    rows = np.arange(0, wl.N, max(1, wl.N // 256))
    ref = _x_f64(X)[rows] @ oracle.bf16_value(Wb).astype(np.float64).T
    act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube)
    err = {}
    for f in oracle.KERNEL_FORMATS:
        y = oracle.output_rows(act, wq, X, L1, L2, rows, kernel_values=oracle.kernel_tokens_dequantized(act, f))
        err[f] = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert err["bf16"] <= err["fp8"] < 1.01 * err["bf16"], err
    assert err["nvfp4"] > 1.02 * err["fp8"], err


# ------------------------------------------------------------------ group-64 kernel scales

def test_group_kernel_scales_closed_form():
    """Per-group FP8 kernel tokens on a hand-built token whose group amaxes
    are 448 times powers of two: every quotient m / s8 is exact, so the codes
    are the E4M3 encodings of known values (E4M3: bias 7, three mantissa bits;
    448 = 0x7E, 1 = 0x38, -2 = 0xC0, 0.5 = 0x30, -3.5 = 0xC6, 2^-9 = 0x01), an
    all-zero group has scale 0 and zero codes, and one scale for the whole
    token (group = Ci) shrinks the small group onto coarser codes."""
    m = np.zeros((1, 192), np.float32)
    m[0, :4] = [56.0, 0.125, -0.25, 0.0625]                 # amax 56 -> s8 = 1/8
    m[0, 64:67] = [7.0, -7.0 / 128, 2.0 ** -15]             # amax 7  -> s8 = 1/64
    q8, s8 = oracle.fp8_kernel_tokens(m, 64)
    assert s8.tolist() == [[0.125, 1.0 / 64, 0.0]]
    assert q8[0, :4].tolist() == [0x7E, 0x38, 0xC0, 0x30] and not q8[0, 4:64].any()
    assert q8[0, 64:67].tolist() == [0x7E, 0xC6, 0x01] and not q8[0, 67:].any()
    q1, s1 = oracle.fp8_kernel_tokens(m, 192)
    assert s1.tolist() == [[0.125]]
    assert q1[0, 64] == 0x66                                 # 7 / (1/8) = 56 = 1.75 * 2^5


def test_group_equal_to_token_width_is_the_per_token_path(tiny_case):
    wl, X, Wb, L1, L2, sig, act, wq = tiny_case
    q8, s8 = oracle.fp8_kernel_tokens(act["means"], wl.Ci)
    assert np.array_equal(q8, act["q8"]) and np.array_equal(s8[:, 0], act["s8"])


@pytest.mark.parametrize("cube", [(1, 2, 2), (2, 4, 4)])
def test_group64_kernel_tokens_are_finer(cube):
    """With outlier channels, one scale per 64 channels quantises the kernel
    tokens more finely than one per token (the note's per-group-64 choice):
    lower error of the dequantised kernel tokens, no worse Y."""
    T, H, W, Ci, Co = 4, 16, 16, 512, 384
    wl = synth.Workload("mid", T, H, W, Ci, Co, 16, cube, (T, 4, 4), (0.01, 50.0), (0.01, 20.0))
    X = synth.activations(wl, seed=77)
    Wb = synth.weight(wl, seed=78)
    L1, L2, _ = oracle.lowrank_factors(Wb, wl.rank)
    wq = oracle.quantize_weight(Wb, L1, L2)
    rows = np.arange(0, wl.N, 4)
    ref = _x_f64(X)[rows] @ oracle.bf16_value(Wb).astype(np.float64).T
    ek, ey = {}, {}
    for kg in (0, 64):
        act = oracle.quantize_activations(X, T, H, W, cube, kernel_group=kg)
        assert act["s8"].shape == ((act["q8"].shape[0],) if kg == 0 else (act["q8"].shape[0], Ci // 64))
        kd = oracle.kernel_tokens_dequantized(act, "fp8")
        ek[kg] = np.linalg.norm(kd - act["means"]) / np.linalg.norm(act["means"])
        y = oracle.output_rows(act, wq, X, L1, L2, rows)
        ey[kg] = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert ek[64] < 0.8 * ek[0], ek
    assert ey[64] <= ey[0], ey


# ------------------------------------------------------------------ power-of-two scales (single-read option)

def _is_pow2(v):
    m, _ = math.frexp(float(v))
    return v > 0 and m == 0.5


def test_pow2_delta_scale_closed_form(tiny_case):
    """Power-of-two delta scale: S_delta is the smallest power of two >= amax / 2688; the
    kernel tokens are untouched (their scale keeps max|m| / 448, which maps each token's
    largest element exactly onto 448)."""
    wl, X, *_ = tiny_case
    act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube, pow2_scales=True)
    ref = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube)
    S, amax = act["S_delta"], act["amax_delta"]
    assert _is_pow2(S) and amax / 2688 <= S < amax / 1344
    assert oracle.pow2_scale(amax) == S and oracle.pow2_scale(0.0) == 1.0
    assert np.array_equal(act["q8"], ref["q8"]) and np.array_equal(act["s8"], ref["s8"])
    assert np.array_equal(act["means"], ref["means"])


def test_scale_byte_fixup_invariance():
    """The property a single-read encoder's fix-up pass relies on: encoded under S and
    under 2^j S (powers of two), a block keeps its E2M1 codes and its E4M3 scale code moves
    down by j binades (8 j in the code) whenever the shifted scale stays in E4M3's normal
    range, i.e. the scale's exponent field under S is at least j + 1.  Blocks below that
    are rounded on the subnormal grid instead: the set that needs re-encoding."""
    rng = np.random.default_rng(3)
    Z = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-12, 6, size=(64, 1)))).astype(np.float32)
    amax = float(np.abs(Z).max())
    S = float(oracle._L().or_pow2_ceil(amax / 2688.0))
    c1, s1, _ = oracle.fp4_quantize(Z, S)
    normal_blocks = subnormal = 0
    for j in (1, 2, 5):
        cj, sj, _ = oracle.fp4_quantize(Z, S * 2.0 ** j)
        ok = ((s1 >> 3) & 0xF) >= j + 1                           # the shifted scale stays normal
        assert np.array_equal(sj[ok].astype(int), s1[ok].astype(int) - 8 * j)
        blocks_ok = np.repeat(ok, 8, axis=1)                      # 8 code bytes per 16-channel block
        assert np.array_equal(cj[blocks_ok], c1[blocks_ok])
        normal_blocks += int(ok.sum())
        subnormal += int((~ok).sum())
    assert normal_blocks > 0 and subnormal > 0                    # both cases exercised


def test_pow2_scales_cost_little_accuracy():
    """The deviation's cost on correlated activations: the reconstruction error of the
    deltas with a power-of-two per-tensor scale stays within 2 % of the two-level
    reading's (the group-16 scales absorb the difference)."""
    wl = synth.Workload("mid", 4, 16, 16, 512, 384, 16, (1, 2, 2), (4, 4, 4), (0.01, 50.0), (0.01, 20.0))
    X = synth.activations(wl, seed=77)
    x = _x_f64(X)
    err = {}
    for p2 in (False, True):
        act = oracle.quantize_activations(X, wl.T, wl.H, wl.W, wl.cube, pow2_scales=p2)
        dqd = _dequant_rows(act["dcodes"], act["dscales"], act["S_delta"])[act["row_of_n"]]
        d = x - act["means"].astype(np.float64)[act["cube_of_n"]]
        err[p2] = np.linalg.norm(dqd - d) / np.linalg.norm(d)
    assert err[True] < 1.02 * err[False], err


# ------------------------------------------------------------------ C2: restricted weight scales (option)

def _c2_members():
    """{0} and every m 2^e (m in {1, 1.25, 1.5}) that E4M3 holds, up to 384: written out from
    the E4M3 value table (exponent field, mantissa field), independently of the oracle's search."""
    vals = {0.0}
    for code in range(1, 127):
        e, m = (code >> 3) & 15, code & 7
        v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        if v > 384:
            continue
        mant = v / 2.0 ** math.floor(math.log2(v))
        if mant in (1.0, 1.25, 1.5):
            vals.add(v)
    return sorted(vals)


def test_c2_scale_nearest_closed_form():
    """The restricted scale is the member of {0} U {1, 1.25, 1.5} x 2^e (E4M3 values up to 384)
    nearest to its argument, ties to the larger; the members' products with every E2M1 value
    need at most three fraction bits."""
    L = oracle._L()
    members = _c2_members()
    assert 384.0 in members and 5 * 2.0 ** -9 in members and 7 * 2.0 ** -9 not in members
    assert 2.5 * 2.0 ** -9 not in members and 1.75 not in members
    rng = np.random.default_rng(7)
    vals = np.concatenate([np.exp(rng.uniform(np.log(2.0 ** -12), np.log(500.0), 4000)),
                           members[1:], [(a + b) / 2 for a, b in zip(members, members[1:])]]).astype(np.float32)
    mv = np.array(members)
    for v in vals:
        r = L.or_c2_scale_nearest(float(v))
        d = np.abs(mv - float(v))
        best = mv[d == d.min()].max()
        assert r == best, (float(v), r, best)
    e2m1 = [0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in members[1:]:
        for q in e2m1:
            p = c * q
            frac = p / 2.0 ** math.floor(math.log2(p))
            assert (frac * 8) == int(frac * 8), (c, q)


@pytest.mark.parametrize("shape", [(256, 256, 16), (512, 1024, 32)])
def test_c2_weights_have_an_exact_fp8_form(shape):
    """Under the restricted scales every q s_b of a 32-channel block is an E4M3 value times
    one power of two: the FP8 operand with its UE8M0 exponents reproduces it exactly."""
    Co, Ci, r = shape
    wl = synth.Workload("c2", 1, 1, 1, Ci, Co, r, (1, 1, 1), (1, 1, 1), (0.0, 1.0), (0.01, 20.0))
    Wb = synth.weight(wl, seed=Co + Ci)
    L1, L2, _ = oracle.lowrank_factors(Wb, r)
    q = oracle.quantize_weight(Wb, L1, L2, c2=True)
    fp8, ue, inexact = oracle.c2_fp8_operand(q["wcodes"], q["wscales"])
    assert inexact == 0
    w = _dequant_rows(q["wcodes"], q["wscales"], 1.0)
    back = oracle.e4m3_value(fp8) * np.repeat(np.exp2(ue.astype(np.float64) - 127), 32, axis=1)
    assert np.array_equal(back, w)
    # every scale is {1, 1.25, 1.5} x 2^e: E4M3 mantissa field 0, 2 or 4 (or a subnormal k 2^-9, k <= 6)
    s = q["wscales"].astype(int)
    normal = (s >> 3) > 0
    assert np.all(np.isin(s[normal] & 7, (0, 2, 4))) and np.all(np.isin(s[~normal], (0, 1, 2, 3, 4, 5, 6)))
    # per 32 channels the largest |q s_b| / 2^u lies in [128, 256)
    big = np.abs(w).reshape(w.shape[0], -1, 32).max(axis=2)
    scaled = big / np.exp2(ue.astype(np.float64) - 127)
    assert np.all((scaled[big > 0] >= 128) & (scaled[big > 0] < 256))


def test_c2_accuracy_cost():
    """The price of the FP8-rate form: three scale mantissas instead of E4M3's eight, so the
    weight error grows a little (the default keeps Eq. 4's scales)."""
    wl = synth.Workload("c2", 1, 1, 1, 1024, 512, 32, (1, 1, 1), (1, 1, 1), (0.0, 1.0), (0.01, 20.0))
    Wb = synth.weight(wl, seed=5)
    L1, L2, _ = oracle.lowrank_factors(Wb, 32)
    R = oracle.residual(Wb, L1, L2).astype(np.float64)
    err = {}
    for c2 in (False, True):
        q = oracle.quantize_weight(Wb, L1, L2, c2=c2)
        err[c2] = np.linalg.norm(_dequant_rows(q["wcodes"], q["wscales"], q["S_w"]) - R) / np.linalg.norm(R)
    assert err[False] < err[True] < 1.15 * err[False], err


def test_single_read_encode_with_fixup_equals_direct_encode():
    """The single-read algorithm the power-of-two delta scale allows: each work item (rows x a
    range of channels) encodes under its own power-of-two scale S0 from its local max, then,
    once the global S is known, every block's scale code drops by 8 log2(S / S0) and its
    codes stay, except blocks without the exponent headroom, which are encoded again under S.
    The result equals encoding every item directly under S."""
    L = oracle._L()
    rng = np.random.default_rng(11)
    # rows of very different magnitude, so that items' local scales differ by several binades
    Z = (rng.standard_normal((96, 512)) * np.exp(rng.uniform(-9, 3, size=(96, 1)))).astype(np.float32)
    S = float(L.or_pow2_ceil(float(np.abs(Z).max()) / 2688.0))
    reencoded = 0
    for r0 in range(0, 96, 32):
        for c0 in range(0, 512, 128):
            item = np.ascontiguousarray(Z[r0:r0 + 32, c0:c0 + 128])
            S0 = float(L.or_pow2_ceil(float(np.abs(item).max()) / 2688.0))
            j = int(round(math.log2(S / S0)))
            codes0, scales0, _ = oracle.fp4_quantize(item, S0)
            codesS, scalesS, _ = oracle.fp4_quantize(item, S)
            ok = ((scales0.astype(int) >> 3) & 15) >= j + 1
            fixed_scales = np.where(ok, scales0.astype(int) - 8 * j, scalesS.astype(int))
            fixed_codes = np.where(np.repeat(ok, 8, axis=1), codes0, codesS)
            reencoded += int((~ok).sum())
            assert np.array_equal(fixed_scales, scalesS.astype(int))
            assert np.array_equal(fixed_codes, codesS)
    assert reencoded > 0      # the re-encode branch is exercised too


# ------------------------------------------------------------------ sampled cubes (the CPU baseline's sample)

@pytest.mark.parametrize("shape,cube", [((5, 9, 21), (2, 2, 2)), ((3, 10, 37), (1, 2, 2)), ((4, 6, 10), (4, 6, 10))])
def test_sampled_cubes_match_the_whole_tensor(shape, cube):
    """The CPU baseline quantises a seeded sample of cubes under the whole tensor's
    delta scale: the whole-tensor statistics pass must give the same amax as the
    full quantiser, the sampled cubes' codes, scales and kernel tokens the full
    quantiser's rows bit for bit (ragged edge cubes included), and their Y rows
    the full path's exactly."""
    T, H, W = shape
    wl = synth.Workload("sample", T, H, W, 256, 256, 16, cube, (T, 2, 2), (0.02, 40.0), (0.01, 20.0))
    X = synth.activations(wl, seed=31)
    act = oracle.quantize_activations(X, T, H, W, cube)
    amax = oracle.delta_amax(X, T, H, W, cube)
    assert np.float32(amax) == np.float32(act["amax_delta"])
    assert np.float32(oracle.tensor_scale(amax)) == np.float32(act["S_delta"])
    K = act["count"].size
    ks = np.unique(np.r_[np.random.default_rng(3).choice(K, size=min(5, K), replace=False), K - 1])[::-1].copy()
    sub = oracle.quantize_cubes(X, T, H, W, cube, ks, oracle.tensor_scale(amax))
    rows_cm = np.concatenate([np.arange(act["first"][k], act["first"][k] + act["count"][k]) for k in ks])
    assert np.array_equal(sub["dcodes"], act["dcodes"][rows_cm])
    assert np.array_equal(sub["dscales"], act["dscales"][rows_cm])
    assert np.array_equal(sub["q8"], act["q8"][ks]) and np.array_equal(sub["s8"], act["s8"][ks])
    assert np.array_equal(sub["rows"], act["n_of_row"][rows_cm])
    Wb = synth.weight(wl, seed=32)
    L1, L2, _ = oracle.lowrank_factors(Wb, 16)
    wq = oracle.quantize_weight(Wb, L1, L2)
    y_sub = oracle.output_rows(sub, wq, X, L1, L2, sub["rows"])
    y_full = oracle.output_rows(act, wq, X, L1, L2, sub["rows"])
    assert np.array_equal(y_sub, y_full)
