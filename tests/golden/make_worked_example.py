"""Writes worked_cube_1x2x2.json: a hand-derived example of Eq. 1 and Eq. 4.

Source: papernotes.org, "DeltaQuant: 4-bit Video Diffusion Models with
Spatiotemporal Delta Smoothing", key design 3 (Eq. 1: kernel token = cube
mean, delta = token - mean) and key design 4 (Eq. 4: Q(X) = round(X/s) s,
s = max|X| / q_max, q_max = 6 for FP4), with the readings FP8 = E4M3 per-token
scale amax/448 and FP4 = E2M1 with E4M3 group-16 scales under a per-tensor
scale amax/(6*448).

The page prints no numbers for a worked example, so the expected values here
are derived by hand in closed form (see DERIVATION); this script only writes
them down.  It imports neither the oracle nor the library.
"""
import json
import os

DERIVATION = """
One 1x2x2 cube (T=1, H=2, W=2) of 16 channels; tokens in (t,h,w) order carry
d = (3, -1, 1, -3) and x[n][c] = m_c + d_n g_c with
  c = 0..7: m_c = c/2, g_c = 1/16;  c = 8..14: m_c = 1, g_c = 7/64;  c = 15: m_c = 14, g_c = 0.
All x are exact in BF16 and all partial sums exact in fp32, so the kernel token is m.
max|m| = 14 -> s8 = 14/448 = 2^-5, q8 = E4M3(32 m), exact.
Deltas d g: global amax 21/64 -> S = (21/64)/2688 = 2^-13, denom = 6 S.
|d| = 3 tokens: block amax 21/64 -> 448 exactly -> s_b = 448, eff = 7/128:
  c<8: (3/16)/(7/128) = 24/7 -> E2M1 3;  c=8..14: 6;  c=15: +0.
|d| = 1 tokens: block amax 7/64 -> 448/3 = 149.3 -> E4M3 144, eff = 9/512:
  c<8: (1/16)/(9/512) = 3.56 -> 4;  c=8..14: 6.22 -> 6 (saturates);  c=15: +0.
"""


def bf16_bits(v):
    import struct
    u = struct.unpack("<I", struct.pack("<f", v))[0]
    assert u & 0xFFFF == 0, v          # every value here is exact in BF16
    return u >> 16


def e4m3_code(v):
    """E4M3 code of a value that is exactly representable and normal:
    v = 2^(e-7) (1 + m/8), code = e << 3 | m (zero -> 0)."""
    import math
    if v == 0.0:
        return 0
    fr, ex = math.frexp(v)            # v = fr * 2^ex, fr in [0.5, 1)
    e = ex - 1 + 7
    m = (fr * 2 - 1) * 8
    assert m == int(m) and 1 <= e <= 15, v
    return (e << 3) | int(m)


def main():
    m = [c / 2 for c in range(8)] + [1.0] * 7 + [14.0]
    g = [1 / 16] * 8 + [7 / 64] * 7 + [0.0]
    d = [3.0, -1.0, 1.0, -3.0]
    X = [[bf16_bits(m[c] + d[n] * g[c]) for c in range(16)] for n in range(4)]
    q8 = [e4m3_code(32 * v) for v in m]
    # E2M1 codes: 3 -> 5, 4 -> 6, 6 -> 7, sign bit 8
    rows = []
    for dn in d:
        sign = 8 if dn < 0 else 0
        lo = (5 if abs(dn) == 3 else 6) | sign
        mid = 7 | sign
        rows.append([lo] * 8 + [mid] * 7 + [0])
    dcodes = [[r[2 * i] | (r[2 * i + 1] << 4) for i in range(8)] for r in rows]
    out = {
        "source": "papernotes.org DeltaQuant note, key design 3 (Eq. 1) and key design 4 (Eq. 4)",
        "derivation": DERIVATION.strip(),
        "T": 1, "H": 2, "W": 2, "cube": [1, 2, 2], "Ci": 16,
        "X_bf16": X,
        "means": m,
        "s8": 2.0 ** -5,
        "q8": q8,
        "amax_delta": 21 / 64,
        "S_delta": 2.0 ** -13,
        "dscales": [e4m3_code(448.0), e4m3_code(144.0), e4m3_code(144.0), e4m3_code(448.0)],
        "dcodes": dcodes,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "worked_cube_1x2x2.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
