"""Pins for the oracle's number formats.

The oracle's FP4 (E2M1) and FP8 (E4M3) encoders follow the DeltaQuant page's
quantiser, Eq. 4 (round to the nearest level, FP4 q_max = 6), with the
readings round-to-nearest-even and saturation.  Each check below compares the
oracle with something other than itself: the bit-field definition of the
formats, torch's float8_e4m3fn cast (a library routine), brute-force nearest
search, and the page's own q_max.
"""
import numpy as np
import torch

import oracle


def _e2m1_from_fields(code):
    # E2M1: sign bit, two exponent bits with bias 1, one mantissa bit;
    # exponent field 0 is subnormal with value m * 2^(1-1) * 0.5.
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    v = (m * 0.5) if e == 0 else (1 + m * 0.5) * 2.0 ** (e - 1)
    return -v if s else v


def test_e2m1_table_matches_bit_fields():
    got = oracle.e2m1_value(np.arange(16))
    want = np.array([_e2m1_from_fields(c) for c in range(16)])
    assert np.array_equal(np.abs(got), np.abs(want))
    assert np.array_equal(np.signbit(got[8:]), np.ones(8, bool))


def test_e2m1_qmax_is_six():
    # Eq. 4: "q_max = 6 for 4-bit floating point"
    assert oracle.e2m1_value([7])[0] == 6.0
    assert oracle.e2m1_value(np.arange(8)).max() == 6.0


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_value(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                      # 0x7F and 0xFF only
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0


def test_e4m3_encode_matches_torch_dense_sweep():
    rng = np.random.default_rng(7)
    # every representable value, every midpoint, and its two fp32 neighbours,
    # plus a log-uniform sweep; |v| < 464 where torch's cast is finite
    vals = oracle.e4m3_value(np.arange(127))
    mids = (vals[:-1] + vals[1:]) / 2
    pts = np.concatenate([vals, mids, [448.0, 456.0, 463.9]]).astype(np.float32)
    nb = np.concatenate([pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    sweep = (np.exp(rng.uniform(np.log(1e-4), np.log(463.0), 200000))).astype(np.float32)
    v = np.concatenate([nb, sweep, [0.0]]).astype(np.float32)
    v = np.concatenate([v, -v])
    v = v[np.abs(v) < 464]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(v)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, (v[bad[:5]], ref[bad[:5]], got[bad[:5]])


def test_e4m3_saturates():
    v = np.array([464.0, 480.0, 1e6, 3e38, -500.0], np.float32)
    got = oracle.e4m3_encode(v)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_e2m1_encode_brute_force_nearest_even():
    mags = oracle.e2m1_value(np.arange(8))
    rng = np.random.default_rng(3)
    mids = (mags[:-1] + mags[1:]) / 2
    pts = np.concatenate([mags, mids, rng.uniform(0, 8, 100000)]).astype(np.float32)
    pts = np.concatenate([pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    got = oracle.e2m1_encode(pts)
    for v, c in zip(pts[:2000], got[:2000]):
        d = np.abs(mags - float(v))
        best = np.flatnonzero(d == d.min())
        want = 7 if v >= 6 else (best[0] if best.size == 1 else best[best % 2 == 0][0])
        assert c == want, (v, c, want)
    # vectorised check of the remainder: nearest, ties to even, saturation
    d = np.abs(mags[None, :] - pts[:, None].astype(np.float64))
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & (np.arange(8)[None, :] % 2 == 0)
    want = np.where(cand.sum(1) == 1, cand.argmax(1), even.argmax(1))
    want = np.where(pts >= 6, 7, want)
    assert np.array_equal(got, want.astype(np.uint8))


def test_e2m1_ties_listed():
    # round-half-even at every midpoint of the E2M1 magnitude ladder
    v = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0], np.float32)
    assert list(oracle.e2m1_value(oracle.e2m1_encode(v))) == [0, 1, 1, 2, 2, 4, 4, 6, 6]


def test_signed_zero_kept():
    v = np.array([-1e-9, -0.0, 1e-9, 0.0], np.float32)
    assert list(oracle.e2m1_encode(v)) == [8, 8, 0, 0]
    assert list(oracle.e4m3_encode(v)) == [0x80, 0x80, 0, 0]


def test_encode_decode_roundtrip_and_monotone():
    for enc, val, n in ((oracle.e2m1_encode, oracle.e2m1_value, 8), (oracle.e4m3_encode, oracle.e4m3_value, 127)):
        v = val(np.arange(n)).astype(np.float32)
        assert np.array_equal(enc(v), np.arange(n))
        s = np.sort(np.random.default_rng(1).uniform(0, float(v[-1]) * 1.2, 50000)).astype(np.float32)
        q = val(enc(s))
        assert np.all(np.diff(q) >= 0)


def test_bf16_round_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(oracle.bf16_round(v[:3000].astype(np.float64)), ref[:3000])
    assert np.array_equal(oracle.bf16_round_fast(v.astype(np.float64)), ref)
