"""The library's offline weight packer (host C++) against the oracle.

Given the same BF16 factors L1, L2 (taken from the oracle's own SVD), the
residual codes, the group scales (through the scale-factor layout) and the
per-tensor scale must be bit-exact; the BF16 dequantised weight must equal
code * scale exactly.  The library's own randomised SVD is pinned by the
Eckart-Young bound with singular values from the oracle."""
import numpy as np
import pytest

import oracle
import synth


@pytest.fixture(scope="module")
def dq():
    import __graft_entry__
    __graft_entry__.build()
    import video_diffusion_w4a4_b200 as m
    return m


def _unpack_scales(dq, blob, off, rows, cols):
    """Weight scales from the B-operand scale layout; the four per-quadrant copies must agree."""
    idx = np.array([[dq.dq_sfb_offset(r, b, cols) for b in range(cols // 16)] for r in range(rows)])
    copies = [blob[off + idx + 1024 * q] for q in range(4)]
    for c in copies[1:]:
        assert np.array_equal(c, copies[0])
    return copies[0]


@pytest.mark.parametrize("shape", [(256, 256, 16), (512, 1024, 32), (1024, 512, 48)])
def test_pack_bit_exact(dq, shape):
    Co, Ci, r = shape
    wl = synth.Workload("pack", 1, 1, 1, Ci, Co, r, (1, 1, 1), (1, 1, 1), (0.0, 1.0), (0.01, 20.0))
    Wb = synth.weight(wl, seed=Co * 7 + Ci)
    L1, L2, _ = oracle.lowrank_factors(Wb, r)
    wq = oracle.quantize_weight(Wb, L1, L2)
    packed, L1m, L2s, S_W = dq.dq_pack_weight_factors(Wb, L1, L2)
    lay = dq.dq_packed_weight_layout(Co, Ci, r)
    hdr = packed[:256].view(np.uint32)
    assert hdr[0] == 0x31575144 and hdr[1] == 3
    assert hdr[7] == 0 and not packed[lay.off_bias:lay.total_bytes].any()     # no bias
    assert list(packed[32:72].view(np.uint64)) == [lay.off_codes, lay.off_scales, lay.off_dqw, lay.total_bytes,
                                                  lay.off_bias]
    assert list(packed[8:24].view(np.int32)) == [Co, Ci, r, lay.slab]
    assert packed[24:28].view(np.float32)[0] == np.float32(wq["S_w"]) == np.float32(S_W)
    codes = packed[lay.off_codes:lay.off_codes + Co * Ci // 2].reshape(Co, Ci // 2)
    assert np.array_equal(codes, wq["wcodes"])
    assert np.array_equal(_unpack_scales(dq, packed, lay.off_scales, Co, Ci), wq["wscales"])
    dqw = packed[lay.off_dqw:lay.off_dqw + Co * Ci * 2].view(np.uint16).reshape(Co, Ci)
    q = np.empty((Co, Ci))
    q[:, 0::2] = oracle.e2m1_value(wq["wcodes"] & 15)
    q[:, 1::2] = oracle.e2m1_value(wq["wcodes"] >> 4)
    want = q * np.repeat(oracle.e4m3_value(wq["wscales"]), 16, axis=1)
    assert np.array_equal(oracle.bf16_value(dqw).astype(np.float64), want)
    assert np.array_equal(L1m, L1.T)
    assert np.array_equal(L2s[:, :r], L2.T) and np.array_equal(L2s[:, r:2 * r], L2.T)
    assert not L2s[:, 2 * r:].any()


@pytest.mark.parametrize("shape", [(256, 256, 16), (768, 1024, 32)])
def test_library_svd_eckart_young(dq, shape):
    Co, Ci, r = shape
    wl = synth.Workload("svd", 1, 1, 1, Ci, Co, r, (1, 1, 1), (1, 1, 1), (0.0, 1.0), (0.01, 20.0))
    Wb = synth.weight(wl, seed=99)
    L1, L2 = dq.dq_lowrank_factors(Wb, r)
    w = oracle.bf16_value(Wb).astype(np.float64)
    sig = np.linalg.svd(w, compute_uv=False)
    l1, l2 = oracle.bf16_value(L1).astype(np.float64), oracle.bf16_value(L2).astype(np.float64)
    err2 = np.linalg.norm(w - (l1 @ l2).T) ** 2
    tail = np.sum(sig[r:] ** 2)
    rnd = (2.0 ** -8 * np.linalg.norm(l1 @ l2)) ** 2
    assert err2 <= (1 + 1e-3) * tail + 4 * rnd, (err2, tail, rnd)


def test_pack_weight_end_to_end_matches_factor_path(dq):
    wl = synth.WORKLOADS["tiny"]
    Wb = synth.weight(wl)
    packed, L1m, L2s = dq.dq_pack_weight(Wb, wl.rank)
    L1, L2 = dq.dq_lowrank_factors(Wb, wl.rank, seed=0)
    p2, L1m2, L2s2, _ = dq.dq_pack_weight_factors(Wb, L1, L2)
    assert np.array_equal(packed, p2) and np.array_equal(L1m, L1m2) and np.array_equal(L2s, L2s2)


def test_pack_bias_section(dq):
    """dq_pack_bias widens the BF16 bias exactly to fp32 in the bias section and
    sets header flag bit 0; clearing restores the blob bit for bit; a bias of
    the wrong length or a blob that is not a packed weight is refused."""
    Co, Ci, r = 512, 256, 16
    wl = synth.Workload("pack", 1, 1, 1, Ci, Co, r, (1, 1, 1), (1, 1, 1), (0.0, 1.0), (0.01, 20.0))
    Wb = synth.weight(wl, seed=3)
    L1, L2, _ = oracle.lowrank_factors(Wb, r)
    packed, *_ = dq.dq_pack_weight_factors(Wb, L1, L2)
    orig = packed.copy()
    lay = dq.dq_packed_weight_layout(Co, Ci, r)
    b = synth.normal_bf16((Co,), sd=2.0, seed=4)
    dq.dq_pack_bias(packed, b)
    assert packed[28:32].view(np.uint32)[0] == 1
    got = packed[lay.off_bias:lay.off_bias + 4 * Co].view(np.float32)
    assert np.array_equal(got, oracle.bf16_value(b))
    assert np.array_equal(packed[:lay.off_bias][256:], orig[:lay.off_bias][256:])
    dq.dq_pack_bias(packed, None)
    assert np.array_equal(packed, orig)
    with pytest.raises(ValueError):
        dq.dq_pack_bias(packed, b[:-1])
    bad = packed.copy()
    bad[0] ^= 1
    with pytest.raises(dq.DQError):
        dq.dq_pack_bias(bad, b)


@pytest.mark.parametrize("shape", [(256, 256), (512, 1024)])
def test_vectorised_weight_scale_map_matches_library(dq, shape):
    """The parity tests read the packed weight's scales at full size through a
    vectorised form of the B-operand scale layout; it must address the same bytes
    as the library's dq_sfb_offset (a scrambled blob makes every scale distinct
    enough to catch a wrong index)."""
    from dq_case import sfb_unpermute
    Co, Ci = shape
    nbytes = dq.dq_sfb_bytes(Co, Ci)
    blob = np.zeros(nbytes, np.uint8)
    plain = np.random.default_rng(Co + Ci).integers(0, 256, size=(Co, Ci // 16), dtype=np.uint8)
    for r in range(Co):
        for b in range(Ci // 16):
            off = dq.dq_sfb_offset(r, b, Ci)
            for q in range(4):
                blob[off + 1024 * q] = plain[r, b]
    assert np.array_equal(sfb_unpermute(blob, Co, Ci), plain)


@pytest.mark.parametrize("shape", [(256, 256, 16), (512, 1024, 32), (768, 512, 48)])
def test_pack_c2_bit_exact(dq, shape):
    """Restricted-scale (C2) packing against the oracle's C2 quantiser and FP8 form:
    residual codes, group scales (all quadrant copies), S_W, the E4M3 codes of
    q s_b / 2^u and the UE8M0 exponents (through the 1X scale layout, all four
    copies), bit for bit; header flag bit 1 set; the FP8 form times 2^u equals
    q s_b exactly."""
    from dq_case import packed_weight_parts, sfb_unpermute
    Co, Ci, r = shape
    wl = synth.Workload("pack", 1, 1, 1, Ci, Co, r, (1, 1, 1), (1, 1, 1), (0.0, 1.0), (0.01, 20.0))
    Wb = synth.weight(wl, seed=Co * 3 + Ci)
    L1, L2, _ = oracle.lowrank_factors(Wb, r)
    wq = oracle.quantize_weight(Wb, L1, L2, c2=True)
    fp8_o, ue_o, inexact = oracle.c2_fp8_operand(wq["wcodes"], wq["wscales"])
    assert inexact == 0
    packed, L1m, L2s, S_W = dq.dq_pack_weight_factors(Wb, L1, L2, pack_flags=dq.DQ_PACK_C2)
    lay = dq.dq_packed_weight_layout(Co, Ci, r)
    assert packed[28:32].view(np.uint32)[0] == 2          # the C2 flag, no bias
    pw = packed_weight_parts(packed)
    assert np.array_equal(pw["wcodes"], wq["wcodes"]) and np.array_equal(pw["wscales"], wq["wscales"])
    assert np.float32(S_W) == np.float32(wq["S_w"]) == np.float32(pw["S_w"])
    fp8 = packed[lay.off_dqw:lay.off_dqw + Co * Ci].reshape(Co, Ci)
    assert np.array_equal(fp8, fp8_o)
    # exponents: the B-operand layout of a Co x Ci/2 matrix, one "16-column block" per 32 channels
    ue = sfb_unpermute(packed[lay.off_dqw + Co * Ci:], Co, Ci // 2)
    assert np.array_equal(ue, ue_o)
    back = oracle.e4m3_value(fp8) * np.repeat(np.exp2(ue.astype(np.float64) - 127), 32, axis=1)
    q = np.empty((Co, Ci))
    q[:, 0::2] = oracle.e2m1_value(wq["wcodes"] & 15)
    q[:, 1::2] = oracle.e2m1_value(wq["wcodes"] >> 4)
    assert np.array_equal(back, q * np.repeat(oracle.e4m3_value(wq["wscales"]), 16, axis=1))
    # the default packing is unchanged by the option's existence
    p0, *_ = dq.dq_pack_weight_factors(Wb, L1, L2)
    assert p0[28:32].view(np.uint32)[0] == 0


def test_forward_options_are_checked(dq):
    """The FP8 kernel-token product takes per-token kernel scales only; unknown
    options are refused before anything runs."""
    args = (4, 8, 8, 1, 2, 2, 256, 256, 16)
    lay = dq.dq_workspace_layout_opts(*args, kernel_product=dq.DQ_KERNEL_PRODUCT_FP8)
    full = dq.dq_workspace_layout_opts(*args)
    assert lay.total_bytes < full.total_bytes and lay.off_dcodes == lay.off_q8_bf16   # no BF16 operand
    for kw in (dict(kernel_product=2), dict(kernel_group=64, kernel_product=dq.DQ_KERNEL_PRODUCT_FP8),
               dict(kernel_group=32)):
        with pytest.raises(dq.DQError):
            dq.dq_workspace_layout_opts(*args, **kw)
    with pytest.raises(dq.DQError):
        dq.dq_pack_weight_factors(np.zeros((256, 256), np.uint16), np.zeros((256, 16), np.uint16),
                                  np.zeros((16, 256), np.uint16), pack_flags=4)
