"""Shared helpers for the GPU parity tests: run one layer through the C ABI on
the GPU, run the oracle on the same seeded inputs, and compare.

Tolerance (bit-exact for every quantised tensor; Y per element within
max(1 BF16 ulp of the reference, 1e-3 * RMS of the reference rows)) follows
the parity bar stated for this layer: fp32 tensor-core accumulation and a
BF16 output against an fp64 product of the same dequantised operands.
"""
from __future__ import annotations

import numpy as np

import oracle
import synth


def sf_unpermute(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """Scale-factor layout (include/deltaquant.h) -> plain rows x cols/16."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(cols // 16, dtype=np.int64)[None, :]
    off = ((r // 128) * (cols // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    return buf[off]


def sfa_unpermute(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """A-operand scale layout (include/deltaquant.h, dq_sfa_offset) -> plain rows x cols/16."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(cols // 16, dtype=np.int64)[None, :]
    kb, rr = b // 4, r % 128
    block = ((r // 128) * (cols // 256) + kb // 4) * 2 + (kb // 2) % 2
    off = block * 4096 + (rr // 8) * 256 + (kb % 2) * 128 + (rr % 8) * 16 + (rr // 32) * 4 + b % 4
    return buf[off]


def sfb_unpermute(buf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """B-operand scale layout (include/deltaquant.h, dq_sfb_offset) -> plain rows x cols/16.
    Each scale is stored four times, once per 32-lane quadrant (1024 bytes apart);
    the four copies must agree."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(cols // 16, dtype=np.int64)[None, :]
    n = r % 256
    word = 4 * (n // 128) + (n % 128) // 32
    bb = 4 * word + b % 4
    off = ((r // 256) * (cols // 64) + b // 4) * 4096 + ((n % 32) // 8) * 256 + (bb // 16) * 128 + (n % 8) * 16 \
        + bb % 16
    copies = [buf[off + 1024 * q] for q in range(4)]
    for q in range(1, 4):
        assert np.array_equal(copies[q], copies[0]), f"weight scale copy of quadrant {q} differs"
    return copies[0]


def packed_weight_parts(packed: np.ndarray) -> dict:
    """Codes, group scales (plain Co x Ci/16) and S_W of a packed weight blob, read
    through the offsets in its header (include/deltaquant.h)."""
    Co, Ci = (int(v) for v in packed[8:16].view(np.int32))
    off_codes, off_scales = (int(v) for v in packed[32:48].view(np.uint64))
    codes = packed[off_codes:off_codes + Co * Ci // 2].reshape(Co, Ci // 2)
    scales = sfb_unpermute(packed[off_scales:], Co, Ci)
    return dict(wcodes=codes, wscales=scales, S_w=packed[24:28].view(np.float32)[0], Co=Co, Ci=Ci)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def y_tolerance(y_ref: np.ndarray) -> np.ndarray:
    rms = np.sqrt(np.mean(y_ref ** 2))
    a = np.abs(y_ref)
    ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7), 0.0)
    return np.maximum(ulp, 1e-3 * rms)


def assert_y_close(y_bits: np.ndarray, y_ref: np.ndarray, what: str = "Y") -> dict:
    y = bf16_bits_to_f64(y_bits)
    tol = y_tolerance(y_ref)
    err = np.abs(y - y_ref)
    bad = err > tol
    info = dict(max_err_over_tol=float((err / tol).max()), n_bad=int(bad.sum()), n=int(err.size))
    assert not bad.any(), f"{what}: {info}, first bad at {np.argwhere(bad)[:5].tolist()}"
    return info


class Case:
    """One layer instance: workload, inputs, oracle factors."""

    def __init__(self, wl: synth.Workload, cube=None, seed=None, tau: int = 0, X=None, Wb=None, kernel_group: int = 0,
                 fp8_product: bool = False, pow2: bool = False):
        self.wl = wl
        self.kernel_group = kernel_group
        # the single-read quantiser: power-of-two per-tensor delta scale
        self.pow2 = pow2
        # the FP8 kernel-token product: weights packed with restricted (C2) scales
        self.fp8_product = fp8_product
        self.cube = tuple(cube or wl.cube)
        self.X = synth.activations(wl, seed=seed, tau=tau) if X is None else X
        self.Wb = synth.weight(wl, seed=seed) if Wb is None else Wb
        self.L1, self.L2, _ = oracle.lowrank_factors(self.Wb, wl.rank)

    # ---------------------------------------------------------------- GPU
    def run_gpu(self, dq, torch, stage_mask=7, packed_override=None, bias=None):
        wl, (t, h, w) = self.wl, self.cube
        packed, L1m, L2s, S_W = dq.dq_pack_weight_factors(self.Wb, self.L1, self.L2,
                                                          pack_flags=dq.DQ_PACK_C2 if self.fp8_product else 0)
        if bias is not None:
            dq.dq_pack_bias(packed, bias)
        if packed_override is not None:
            packed = packed_override(packed)
        dev = torch.device("cuda")
        Xd = torch.from_numpy(self.X.view(np.int16)).to(dev)
        Pd = torch.from_numpy(packed).to(dev)
        L1d = torch.from_numpy(L1m.view(np.int16)).to(dev)
        L2d = torch.from_numpy(L2s.view(np.int16)).to(dev)
        Yd = torch.empty((wl.N, wl.Co), dtype=torch.int16, device=dev)
        kg = self.kernel_group
        kp = dq.DQ_KERNEL_PRODUCT_FP8 if self.fp8_product else dq.DQ_KERNEL_PRODUCT_BF16
        ds = dq.DQ_DELTA_SCALE_POW2 if self.pow2 else dq.DQ_DELTA_SCALE_AMAX
        lay = dq.dq_workspace_layout_opts(wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, kernel_group=kg,
                                          kernel_product=kp, delta_scale=ds)
        ws = torch.zeros(lay.total_bytes, dtype=torch.uint8, device=dev)
        self.last_ws, self.last_layout, self.last_inputs = ws, lay, (Xd, Pd, L1d, L2d, Yd)
        if self.fp8_product or self.pow2:
            dq.dq_linear_forward_opts(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws,
                                      lay.total_bytes, stage_mask, None, torch.cuda.current_stream(),
                                      kernel_group=kg, kernel_product=kp, delta_scale=ds)
        elif kg:
            dq.dq_linear_forward_grouped(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, kg, Pd, L1d, L2d, Yd,
                                         ws, lay.total_bytes, stage_mask, None, torch.cuda.current_stream())
        else:
            dq.dq_linear_forward_ex(Xd, wl.T, wl.H, wl.W, t, h, w, wl.Ci, wl.Co, wl.rank, Pd, L1d, L2d, Yd, ws,
                                    lay.total_bytes, stage_mask, None, torch.cuda.current_stream())
        torch.cuda.synchronize()
        status = dq.dq_read_device_status(ws, torch.cuda.current_stream(), clear=True)
        wsh = ws.cpu().numpy()
        N, K, Ci = lay.N, lay.K, wl.Ci
        ns8 = Ci // kg if kg else 1
        acols = 2 * Ci if kg else Ci
        out = dict(status=status, layout=lay, S_W=S_W, packed=packed,
                   Y=Yd.cpu().numpy().view(np.uint16),
                   amax_delta=wsh[lay.off_scalars:lay.off_scalars + 4].view(np.float32)[0],
                   S_delta=wsh[lay.off_scalars + 4:lay.off_scalars + 8].view(np.float32)[0],
                   s8=wsh[lay.off_s8:lay.off_s8 + 4 * K * ns8].view(np.float32).reshape((K, ns8) if kg else (K,)),
                   q8=wsh[lay.off_q8:lay.off_q8 + K * Ci].reshape(K, Ci),
                   q8_bf16=None if self.fp8_product else
                   wsh[lay.off_q8_bf16:lay.off_q8_bf16 + 2 * K * acols].view(np.uint16).reshape(K, acols),
                   dcodes=wsh[lay.off_dcodes:lay.off_dcodes + N * Ci // 2].reshape(N, Ci // 2),
                   dscales=sfa_unpermute(wsh[lay.off_dscales:], N, Ci),
                   p=wsh[lay.off_p:lay.off_p + 4 * K * wl.Co].view(np.float32).reshape(K, wl.Co))
        if self.pow2:
            out["prov"] = wsh[lay.off_prov:lay.off_prov + N * (Ci // 64)].view(np.int8).reshape(N, Ci // 64)
        return out

    # ---------------------------------------------------------------- oracle
    def run_oracle(self):
        wl = self.wl
        act = oracle.quantize_activations(self.X, wl.T, wl.H, wl.W, self.cube, kernel_group=self.kernel_group,
                                          pow2_scales=self.pow2)
        wq = oracle.quantize_weight(self.Wb, self.L1, self.L2, c2=self.fp8_product)
        return act, wq

    def oracle_rows(self, act, wq, rows, bias=None):
        return oracle.output_rows(act, wq, self.X, self.L1, self.L2, rows, bias=bias)


def compare_quantised(g: dict, act: dict, wq: dict) -> None:
    """Every quantised tensor bit-exact against the oracle: the delta codes and
    scales, S_delta, the kernel tokens and their scales, and the packed weight's
    residual codes, group scales (all four per-quadrant copies) and S_W."""
    assert g["status"] == 0, g["status"]
    pw = packed_weight_parts(g["packed"])
    bad = np.argwhere(pw["wcodes"] != wq["wcodes"])
    assert bad.size == 0, ("weight codes", bad[:5].tolist())
    bad = np.argwhere(pw["wscales"] != wq["wscales"])
    assert bad.size == 0, ("weight scales", bad[:5].tolist())
    assert np.float32(pw["S_w"]) == np.float32(wq["S_w"])
    assert np.float32(g["amax_delta"]) == np.float32(act["amax_delta"])
    assert np.float32(g["S_delta"]) == np.float32(act["S_delta"])
    assert np.float32(g["S_W"]) == np.float32(wq["S_w"])
    assert np.array_equal(g["s8"], act["s8"]), "s8"
    bad = np.argwhere(g["q8"] != act["q8"])
    assert bad.size == 0, ("q8", bad[:5].tolist(), g["q8"][tuple(bad[0])], act["q8"][tuple(bad[0])])
    if g["q8_bf16"] is None:
        pass   # the FP8 kernel-token product reads q8 itself: no BF16 operand
    elif act.get("kernel_group"):
        # the product's operand: q8 s8 as BF16 hi + lo, within 2^-16 of the exact product
        Ci = act["q8"].shape[1]
        want = oracle.kernel_tokens_dequantized(act, "fp8")
        hl = bf16_bits_to_f64(g["q8_bf16"][:, :Ci]) + bf16_bits_to_f64(g["q8_bf16"][:, Ci:])
        assert np.all(np.abs(hl - want) <= 2.0 ** -16 * np.abs(want)), "q8 s8 as BF16 hi + lo"
    else:
        assert np.array_equal(bf16_bits_to_f64(g["q8_bf16"]), oracle.e4m3_value(act["q8"])), "q8 as BF16"
    bad = np.argwhere(g["dscales"] != act["dscales"])
    assert bad.size == 0, ("delta scales", bad[:5].tolist())
    bad = np.argwhere(g["dcodes"] != act["dcodes"])
    assert bad.size == 0, ("delta codes", bad[:5].tolist(), g["dcodes"][tuple(bad[0])], act["dcodes"][tuple(bad[0])])


def kernel_term_reference(act: dict, wq: dict, cubes: np.ndarray, bias=None):
    """The per-cube kernel term P'[k][o] = S_W sum_c (q8 s8)[k][c] (q s_b)[o][c] (+ b[o])
    of the sampled cubes, in fp64 from the oracle's kernel tokens and weight codes
    (Eq. 2/3, the single-token term; the bias joins once per cube).  Also returns
    S_W sum_c |(q8 s8)[k][c] (q s_b)[o][c]|, the magnitude that bounds the rounding
    error of an fp32 accumulation of the same sum."""
    cubes = np.asarray(cubes, np.int64)
    Ci = act["q8"].shape[1]
    s8 = np.asarray(act["s8"], np.float64).reshape(len(act["q8"]), -1)
    kv = oracle.e4m3_value(act["q8"][cubes]) * np.repeat(s8[cubes], Ci // s8.shape[1], axis=1)
    dqw = oracle.fp4_dequantize(wq["wcodes"], wq["wscales"], 1.0)
    S_W = float(np.float32(wq["S_w"]))
    ref = S_W * (kv @ dqw.T)
    mag = S_W * (np.abs(kv) @ np.abs(dqw).T)
    if bias is not None:
        b = oracle.bf16_value(np.asarray(bias, np.uint16)).astype(np.float64)
        ref = ref + b[None, :]
        mag = mag + np.abs(b)[None, :]
    return ref, mag


def assert_kernel_term_close(p_gpu: np.ndarray, act: dict, wq: dict, cubes, bias=None, extra_rel: float = 0.0):
    """P' (K x Co fp32, read from the workspace) on the sampled cubes against the fp64
    kernel term.  Bound: the worst-case error of accumulating Ci products in fp32
    (Ci * 2^-23 of the sum of |products|, twice the unit roundoff to allow for an
    accumulator that truncates), one fp32 rounding of the scaled result, and, for
    group-64 kernel scales, the BF16 hi + lo split of q8 s8 (extra_rel of the sum of
    |products|)."""
    cubes = np.asarray(cubes, np.int64)
    ref, mag = kernel_term_reference(act, wq, cubes, bias)
    Ci = act["q8"].shape[1]
    tol = (Ci * 2.0 ** -23 + extra_rel) * mag + 2.0 ** -23 * np.abs(ref)
    got = p_gpu[cubes].astype(np.float64)
    err = np.abs(got - ref)
    bad = err > tol
    info = dict(max_err_over_tol=float((err / np.where(tol > 0, tol, 1.0)).max()), n_bad=int(bad.sum()),
                n=int(err.size), max_rel_err=float((err / np.maximum(np.abs(ref), 1e-30)).max()))
    assert not bad.any(), f"P': {info}, first bad at {np.argwhere(bad)[:5].tolist()}"
    return info
