"""CPU oracle for the DeltaQuant W4A4 linear layer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline may import this package; the library under video_diffusion_w4a4_b200
never does, and this package never imports it.

The arithmetic lives in dq_oracle.c (plain C, OpenMP over independent rows
and cubes).  This module compiles it, marshals numpy arrays, and adds the one
step that uses a library primitive: the truncated SVD of W from which the
low-rank factors L1, L2 are taken (DeltaQuant page, key design 4, Eq. 3,
following SVDQuant).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so in place.  -ffp-contract=off keeps every fp32
    operation a single IEEE rounding, as the oracle's readings require."""
    src = os.path.join(_HERE, "dq_oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", _SO, src, "-lm"])
    return _SO


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        P, I, F, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
        lib.or_bf16_value.argtypes = [ctypes.c_uint16]
        lib.or_bf16_value.restype = F
        lib.or_bf16_round.argtypes = [ctypes.c_double]
        lib.or_bf16_round.restype = ctypes.c_uint16
        lib.or_e2m1_value.argtypes = [I]
        lib.or_e2m1_value.restype = ctypes.c_double
        lib.or_e4m3_value.argtypes = [I]
        lib.or_e4m3_value.restype = ctypes.c_double
        lib.or_e2m1_encode.argtypes = [F]
        lib.or_e4m3_encode.argtypes = [F]
        lib.or_e2m1_encode_array.argtypes = [P, LL, P]
        lib.or_e4m3_encode_array.argtypes = [P, LL, P]
        lib.or_num_cubes.argtypes = [I] * 6
        lib.or_num_cubes.restype = LL
        lib.or_cube_order.argtypes = [I] * 6 + [P] * 5
        lib.or_cube_means.argtypes = [P] + [I] * 7 + [P]
        lib.or_cube_split_f64.argtypes = [P] + [I] * 7 + [P, P]
        lib.or_tensor_scale.argtypes = [F]
        lib.or_tensor_scale.restype = F
        lib.or_fp4_quantize.argtypes = [P, LL, I, F, P, P, P]
        lib.or_quantize_activations.argtypes = [P] + [I] * 7 + [P] * 7
        lib.or_quantize_activations_opt.argtypes = [P] + [I] * 7 + [P] * 7 + [I]
        lib.or_pow2_ceil.argtypes = [F]
        lib.or_c2_scale_nearest.argtypes = [F]
        lib.or_c2_scale_nearest.restype = F
        lib.or_fp4_quantize_c2.argtypes = [P, LL, I, P, P, P]
        lib.or_fp4_quantize_c2.restype = LL
        lib.or_c2_fp8_operand.argtypes = [P, P, LL, I, P, P]
        lib.or_c2_fp8_operand.restype = LL
        lib.or_pow2_ceil.restype = F
        lib.or_residual.argtypes = [P, P, P, I, I, I, P]
        lib.or_output_rows.argtypes = [P, P, F, P, P, P, I, P, P, P, F, I, I, P, P, P, I, P, LL, P]
        lib.or_fp8_kernel_tokens.argtypes = [P, LL, I, I, P, P]
        lib.or_num_threads.restype = I
        lib.or_gelu_erf.argtypes = [P, LL, P]
        lib.or_delta_amax.argtypes = [P] + [I] * 7 + [P]
        lib.or_quantize_cubes.argtypes = [P] + [I] * 7 + [P, LL, F, P, P, P, P, P]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


# --------------------------------------------------------------------------- formats

def e2m1_value(codes) -> np.ndarray:
    tab = np.array([_L().or_e2m1_value(c) for c in range(16)])
    return tab[np.asarray(codes, dtype=np.int64) & 15]


def e4m3_value(codes) -> np.ndarray:
    tab = np.array([_L().or_e4m3_value(c) for c in range(256)])
    return tab[np.asarray(codes, dtype=np.int64) & 255]


def e2m1_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _L().or_e2m1_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _L().or_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def bf16_value(b) -> np.ndarray:
    """BF16 bits -> float32 values, through the oracle's own decoder."""
    b = np.asarray(b, dtype=np.uint16)
    tab = np.array([_L().or_bf16_value(i) for i in range(65536)], dtype=np.float32)
    return tab[b]


def bf16_round(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    f = np.vectorize(lambda x: _L().or_bf16_round(float(x)), otypes=[np.uint16])
    return f(v) if v.size else v.astype(np.uint16)


def tensor_scale(amax: float) -> float:
    return float(_L().or_tensor_scale(amax))


def pow2_scale(amax: float) -> float:
    """The power-of-two per-tensor delta scale: the smallest power of two >= amax / 2688
    (1 if amax = 0), as quantize_activations(pow2_scales=True) takes it."""
    if amax == 0.0:
        return 1.0
    return float(_L().or_pow2_ceil(float(np.float32(np.float32(amax) / np.float32(2688.0)))))


# --------------------------------------------------------------------------- cubes

def num_cubes(T, H, W, t, h, w) -> int:
    return int(_L().or_num_cubes(T, H, W, t, h, w))


def cube_order(T, H, W, t, h, w) -> dict:
    N = T * H * W
    K = num_cubes(T, H, W, t, h, w)
    out = {k: np.empty(s, dtype=np.int32) for k, s in
           (("row_of_n", N), ("cube_of_n", N), ("n_of_row", N), ("count", K), ("first", K))}
    _L().or_cube_order(T, H, W, t, h, w, _p(out["row_of_n"]), _p(out["cube_of_n"]), _p(out["n_of_row"]),
                       _p(out["count"]), _p(out["first"]))
    return out


def cube_means(X, T, H, W, cube) -> np.ndarray:
    X = np.ascontiguousarray(X, dtype=np.uint16)
    Ci = X.shape[1]
    K = num_cubes(T, H, W, *cube)
    m = np.empty((K, Ci), dtype=np.float32)
    if _L().or_cube_means(_p(X), T, H, W, Ci, *cube, _p(m)):
        raise RuntimeError("or_cube_means failed")
    return m


def cube_split_f64(X, T, H, W, cube):
    """Eq. 1 in fp64 without quantisation: (mean K x Ci, delta N x Ci natural order)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    Ci = X.shape[1]
    K = num_cubes(T, H, W, *cube)
    mean = np.empty((K, Ci), dtype=np.float64)
    delta = np.empty((X.shape[0], Ci), dtype=np.float64)
    if _L().or_cube_split_f64(_p(X), T, H, W, Ci, *cube, _p(mean), _p(delta)):
        raise RuntimeError("or_cube_split_f64 failed")
    return mean, delta


# --------------------------------------------------------------------------- quantisers

def fp4_quantize(Z, S: float | None = None):
    """FP4 rows with E4M3 group-16 scales; returns (codes, scales, S)."""
    Z = np.ascontiguousarray(Z, dtype=np.float32)
    rows, cols = Z.shape
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    scales = np.empty((rows, cols // 16), dtype=np.uint8)
    S_out = ctypes.c_float(0)
    if _L().or_fp4_quantize(_p(Z), rows, cols, -1.0 if S is None else float(S), _p(codes), _p(scales),
                            ctypes.byref(S_out)):
        raise RuntimeError("or_fp4_quantize failed")
    return codes, scales, float(S_out.value)


def fp8_kernel_tokens(means, group: int):
    """FP8 E4M3 kernel tokens with one fp32 scale per `group` channels:
    returns (q8 K x Ci, s8 K x Ci/group)."""
    m = np.ascontiguousarray(means, dtype=np.float32)
    K, Ci = m.shape
    q8 = np.empty((K, Ci), np.uint8)
    s8 = np.empty((K, Ci // group), np.float32)
    if _L().or_fp8_kernel_tokens(_p(m), K, Ci, group, _p(q8), _p(s8)):
        raise RuntimeError("or_fp8_kernel_tokens failed")
    return q8, s8


def quantize_activations(X, T, H, W, cube, kernel_group: int = 0, pow2_scales: bool = False) -> dict:
    """Activation side of Eq. 2/3 over the whole X (natural (t,h,w) row order).

    kernel_group 0: one FP8 scale per kernel token (s8: K); 64: one per 64
    channels of a kernel token, the note's per-group kernel quantisation
    (s8: K x Ci/64).

    pow2_scales: a power-of-two per-tensor delta scale (the smallest power of two
    >= amax / 2688), a deviation that lets an encoder fix a block's scale byte up
    after the fact (see or_quantize_activations_opt)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    N, Ci = X.shape
    assert N == T * H * W
    K = num_cubes(T, H, W, *cube)
    out = dict(dcodes=np.empty((N, Ci // 2), np.uint8), dscales=np.empty((N, Ci // 16), np.uint8),
               q8=np.empty((K, Ci), np.uint8), s8=np.empty(K, np.float32),
               means=np.empty((K, Ci), np.float32))
    S = ctypes.c_float(0)
    amax = ctypes.c_float(0)
    rc = _L().or_quantize_activations_opt(_p(X), T, H, W, Ci, *cube, _p(out["dcodes"]), _p(out["dscales"]),
                                          ctypes.byref(S), _p(out["q8"]), _p(out["s8"]), _p(out["means"]),
                                          ctypes.byref(amax), int(pow2_scales))
    if rc:
        raise RuntimeError("or_quantize_activations failed")
    out["S_delta"] = float(S.value)
    out["amax_delta"] = float(amax.value)
    out["kernel_group"] = kernel_group
    out["pow2_scales"] = bool(pow2_scales)
    if kernel_group:
        out["q8"], out["s8"] = fp8_kernel_tokens(out["means"], kernel_group)
    out.update(cube_order(T, H, W, *cube))
    return out


def num_threads() -> int:
    """Threads the oracle's parallel loops use."""
    return int(_L().or_num_threads())


def delta_amax(X, T, H, W, cube) -> float:
    """The whole tensor's max |delta| (cube means and deltas of Eq. 1 in fp32)."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    a = ctypes.c_float(0)
    if _L().or_delta_amax(_p(X), T, H, W, X.shape[1], *cube, ctypes.byref(a)):
        raise RuntimeError("or_delta_amax failed")
    return float(a.value)


def quantize_cubes(X, T, H, W, cube, cubes, S: float) -> dict:
    """The activation side for the listed cubes only, under the per-tensor delta
    scale S of the whole tensor (per-token kernel scales).  Returns a dict that
    output_rows takes for the natural token rows of those cubes: compact delta rows
    (list order, (t,h,w) inside a cube), compact kernel tokens, and N-long maps
    row_of_n / cube_of_n into them (-1 outside the sample); `rows` lists the
    sample's natural token indices in compact row order."""
    X = np.ascontiguousarray(X, dtype=np.uint16)
    N, Ci = X.shape
    cubes = np.ascontiguousarray(cubes, dtype=np.int64)
    o = cube_order(T, H, W, *cube)
    counts = o["count"][cubes].astype(np.int64)
    R = int(counts.sum())
    out = dict(dcodes=np.empty((R, Ci // 2), np.uint8), dscales=np.empty((R, Ci // 16), np.uint8),
               q8=np.empty((cubes.size, Ci), np.uint8), s8=np.empty(cubes.size, np.float32))
    first = np.empty(cubes.size, np.int64)
    if _L().or_quantize_cubes(_p(X), T, H, W, Ci, *cube, _p(cubes), cubes.size, float(S), _p(out["dcodes"]),
                              _p(out["dscales"]), _p(out["q8"]), _p(out["s8"]), _p(first)):
        raise RuntimeError("or_quantize_cubes failed")
    rows = np.concatenate([o["n_of_row"][o["first"][k]:o["first"][k] + o["count"][k]] for k in cubes])
    row_of_n = np.full(N, -1, np.int32)
    row_of_n[rows] = np.arange(R, dtype=np.int32)
    cube_of_n = np.full(N, -1, np.int32)
    cube_of_n[rows] = np.repeat(np.arange(cubes.size, dtype=np.int32), counts)
    out.update(S_delta=float(np.float32(S)), kernel_group=0, row_of_n=row_of_n, cube_of_n=cube_of_n,
               rows=rows.astype(np.int64), first_row=first, cubes=cubes)
    return out


def quantize_plain(X) -> dict:
    """Plain per-token FP4 of X itself (no kernel/delta split), natural row order."""
    xf = bf16_value(X)
    codes, scales, S = fp4_quantize(xf)
    return dict(dcodes=codes, dscales=scales, S_delta=S)


def fp4_dequantize(codes, scales, S: float) -> np.ndarray:
    """fp64 values q * s_g * S of FP4 rows (codes: rows x cols/2, channel 2i in
    the low nibble of byte i; scales: rows x cols/16 E4M3)."""
    codes = np.asarray(codes, np.uint8)
    rows, half = codes.shape
    v = np.empty((rows, half * 2), np.float64)
    v[:, 0::2] = e2m1_value(codes & 15)
    v[:, 1::2] = e2m1_value(codes >> 4)
    return v * np.repeat(e4m3_value(scales), 16, axis=1) * float(S)


KERNEL_FORMATS = ("bf16", "fp8", "nvfp4")


def kernel_tokens_dequantized(act: dict, fmt: str = "fp8") -> np.ndarray:
    """The dequantised kernel tokens (K x Ci, fp64) at one of three precisions,
    the kernel-token precision ablation of the DeltaQuant note (16 / 8 / 4 bit):
      bf16   the fp32 cube means rounded to BF16 (nearest even);
      fp8    E4M3 codes under the per-token fp32 scale, the layer's own format;
      nvfp4  the means as two-level NVFP4: E2M1 codes, E4M3 group-16 scales and
             a per-tensor fp32 scale amax / (6 * 448), the delta tokens' format.
    The deltas stay those of the fp32 means in every variant; only the kernel
    term's operand changes."""
    m = np.asarray(act["means"], np.float32)
    if fmt == "bf16":
        return bf16_value(bf16_round(m)).astype(np.float64)
    if fmt == "fp8":
        s8 = np.asarray(act["s8"], np.float64).reshape(len(act["q8"]), -1)
        return e4m3_value(act["q8"]) * np.repeat(s8, act["q8"].shape[1] // s8.shape[1], axis=1)
    if fmt == "nvfp4":
        return fp4_dequantize(*fp4_quantize(m))
    raise ValueError(fmt)


# --------------------------------------------------------------------------- weight side

def lowrank_factors(Wbits, r: int, seed: int = 0):
    """Truncated SVD W^T ~ V_r S_r U_r^T split evenly: L1 = V_r S_r^1/2 (Ci x r),
    L2 = S_r^1/2 U_r^T (r x Co), each rounded to BF16.  Also returns all
    computed singular values (descending)."""
    Wf = bf16_value(Wbits).astype(np.float64)
    Co, Ci = Wf.shape
    if min(Co, Ci) <= 2048:
        U, s, Vt = np.linalg.svd(Wf, full_matrices=False)
        Ur, sr, Vr = U[:, :r], s[:r], Vt[:r].T
        sig = s
    else:
        from scipy.sparse.linalg import svds
        v0 = np.random.default_rng(seed).standard_normal(min(Co, Ci))
        U, s, Vt = svds(Wf, k=r, tol=0, v0=v0, which="LM")
        order = np.argsort(s)[::-1]
        Ur, sr, Vr = U[:, order], s[order], Vt[order].T
        sig = sr
    L1 = Vr * np.sqrt(sr)[None, :]
    L2 = (Ur * np.sqrt(sr)[None, :]).T
    return bf16_round_fast(L1), bf16_round_fast(L2), sig


def bf16_round_fast(v) -> np.ndarray:
    """Vectorised BF16 rounding, checked against the oracle's search-based
    bf16_round in the tests."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    f = v.astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lo = (u >> 16).astype(np.uint16)
    cand = np.stack([lo - 1, lo, lo + 1]).astype(np.uint16)
    vals = (cand.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    dist = np.abs(vals - v[None])
    dist[np.isnan(dist)] = np.inf
    best = dist.min(axis=0)
    tie_even = (dist == best[None]) & ((cand & 1) == 0)
    pick = np.where(tie_even.any(axis=0), np.argmax(tie_even, axis=0), np.argmin(dist, axis=0))
    return np.take_along_axis(cand, pick[None], axis=0)[0]


def residual(Wbits, L1, L2) -> np.ndarray:
    Wbits = np.ascontiguousarray(Wbits, dtype=np.uint16)
    L1 = np.ascontiguousarray(L1, dtype=np.uint16)
    L2 = np.ascontiguousarray(L2, dtype=np.uint16)
    Co, Ci = Wbits.shape
    r = L1.shape[1]
    R = np.empty((Co, Ci), dtype=np.float32)
    _L().or_residual(_p(Wbits), _p(L1), _p(L2), Co, Ci, r, _p(R))
    return R


def quantize_weight(Wbits, L1, L2, c2: bool = False) -> dict:
    """The residual R = W - L1 L2 in NVFP4 (Eq. 4 per group of 16).  c2: the restricted
    scale rule of or_fp4_quantize_c2 (an option for an exact FP8-rate kernel-token product)."""
    R = residual(Wbits, L1, L2)
    if not c2:
        codes, scales, S = fp4_quantize(R)
        return dict(R=R, wcodes=codes, wscales=scales, S_w=S)
    codes, scales, S, raised = fp4_quantize_c2(R)
    return dict(R=R, wcodes=codes, wscales=scales, S_w=S, raised=raised)


def fp4_quantize_c2(Z):
    """C2 FP4: restricted group scales {1, 1.25, 1.5} x 2^e (nearest); returns (codes, scales, S, raised)."""
    Z = np.ascontiguousarray(Z, dtype=np.float32)
    rows, cols = Z.shape
    codes = np.empty((rows, cols // 2), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    S = ctypes.c_float(0)
    raised = _L().or_fp4_quantize_c2(_p(Z), rows, cols, _p(codes), _p(scales), ctypes.byref(S))
    if raised < 0:
        raise ValueError("or_fp4_quantize_c2 needs a multiple of 32 columns")
    return codes, scales, float(S.value), int(raised)


def c2_fp8_operand(codes, scales):
    """E4M3 codes of q s_b / 2^u and the UE8M0 exponents u + 127 per 32 channels; with
    the count of elements not reproduced exactly."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    rows, half = codes.shape
    cols = half * 2
    fp8 = np.empty((rows, cols), np.uint8)
    ue = np.empty((rows, cols // 32), np.uint8)
    inexact = _L().or_c2_fp8_operand(_p(codes), _p(scales), rows, cols, _p(fp8), _p(ue))
    return fp8, ue, int(inexact)


# --------------------------------------------------------------------------- output

def output_rows(act: dict, wq: dict, X, L1, L2, rows, kernel: bool = True, lowrank: bool = True,
                cube_major: bool = True, bias=None, kernel_values=None) -> np.ndarray:
    """fp64 Y rows (Eq. 3) for natural token indices `rows`.

    bias (Co BF16 bits, optional): the linear layer's bias b, y = x W^T + b.  The
    method's equations carry no bias; with one, the plain reading is that b is
    added to every output row, after the three terms.

    kernel_values (K x Ci fp64, optional): dequantised kernel tokens that replace
    the FP8 ones in the kernel term (see kernel_tokens_dequantized); that term is
    then the fp64 library product kernel_values[k(n)] dq(R)^T."""
    if kernel_values is not None:
        Y = output_rows(act, wq, X, L1, L2, rows, kernel=False, lowrank=lowrank, cube_major=cube_major, bias=bias)
        dqR = fp4_dequantize(wq["wcodes"], wq["wscales"], wq["S_w"])
        kv = np.asarray(kernel_values, np.float64)[np.asarray(act["cube_of_n"])[np.asarray(rows)]]
        return Y + kv @ dqR.T
    X = np.ascontiguousarray(X, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    Co, Ci = wq["wcodes"].shape[0], wq["wcodes"].shape[1] * 2
    r = L1.shape[1] if (lowrank and L1 is not None) else 0
    Y = np.empty((rows.size, Co), dtype=np.float64)
    arow = np.ascontiguousarray(act["row_of_n"], np.int32) if cube_major else None
    cube = np.ascontiguousarray(act["cube_of_n"], np.int32) if kernel else None
    rc = _L().or_output_rows(_p(act["dcodes"]), _p(act["dscales"]), act["S_delta"], _p(arow),
                             _p(act["q8"]) if kernel else None, _p(act["s8"]) if kernel else None,
                             (act.get("kernel_group") or Ci) if kernel else Ci, _p(cube),
                             _p(wq["wcodes"]), _p(wq["wscales"]), wq["S_w"], Co, Ci, _p(X),
                             _p(np.ascontiguousarray(L1, np.uint16)) if r else None,
                             _p(np.ascontiguousarray(L2, np.uint16)) if r else None, r,
                             _p(rows), rows.size, _p(Y))
    if rc:
        raise RuntimeError("or_output_rows failed")
    if bias is not None:
        Y += bf16_value(np.asarray(bias, np.uint16).reshape(1, Co))
    return Y


# --------------------------------------------------------------------------- feed-forward block

def gelu_erf(y) -> np.ndarray:
    """GELU(y) = y Phi(y) = y erfc(-y / sqrt 2) / 2, element by element in fp64 (or_gelu_erf)."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty_like(y)
    _L().or_gelu_erf(_p(y), y.size, _p(out))
    return out


def ffn_hidden_rows(act: dict, wq: dict, X, L1, L2, rows, bias=None) -> np.ndarray:
    """fp64 hidden rows of a feed-forward block: GELU of the up-projection's Y rows
    (output_rows, natural token indices `rows`), before the hidden tensor's one
    rounding to BF16.  The down-projection then quantises that BF16 tensor as any
    layer input (quantize_activations)."""
    return gelu_erf(output_rows(act, wq, X, L1, L2, rows, bias=bias))
