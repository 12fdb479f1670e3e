"""The C-ABI library: it loads without a GPU, exports every entry point that
include/deltaquant.h declares, and its host-side logic (index maps, layout
maps, argument checks) is right.  No test here launches device work."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dq():
    import __graft_entry__
    __graft_entry__.build()
    import video_diffusion_w4a4_b200 as m
    return m


def test_exports_every_declared_symbol(dq):
    hdr = open(os.path.join(ROOT, "include", "deltaquant.h")).read()
    names = re.findall(r"^\s*(?:int|const char\*)\s+(dq_\w+)\s*\(", hdr, flags=re.M)
    assert len(names) == len(set(names)) >= 19
    lib = ctypes.CDLL(dq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert dq.dq_abi_version() == 4


def test_status_strings(dq):
    assert dq.dq_status_string(0) == "ok"
    assert "timed out" in dq.dq_status_string(dq.DQ_ERR_DEVICE_TIMEOUT)
    assert dq.dq_status_string(999) == "unknown status"


@pytest.mark.parametrize("shape,cube", [((4, 8, 8), (1, 2, 2)), ((21, 45, 80), (2, 2, 2)), ((5, 7, 9), (2, 2, 2)),
                                        ((21, 30, 52), (1, 2, 2)), ((7, 5, 6), (2, 4, 4)), ((3, 5, 6), (1, 1, 1))])
def test_cube_major_row_matches_oracle(dq, shape, cube):
    T, H, W = shape
    o = oracle.cube_order(T, H, W, *cube)
    assert dq.dq_cube_count(T, H, W, *cube) == o["count"].size
    N = T * H * W
    for n in range(0, N, max(1, N // 1500)):
        row, k = dq.dq_cube_major_row(T, H, W, *cube, n)
        assert row == o["row_of_n"][n] and k == o["cube_of_n"][n]


def test_sf_offset_is_a_bijection(dq):
    for rows, cols in ((128, 64), (256, 512), (384, 1024)):
        total = dq.dq_sf_bytes(rows, cols)
        assert total == rows * cols // 16
        seen = np.zeros(total, bool)
        for r in range(rows):
            for b in range(cols // 16):
                off = dq.dq_sf_offset(r, b, cols)
                assert not seen[off]
                seen[off] = True
        assert seen.all()
    # ragged row counts are padded up to a whole group of 128 rows
    assert dq.dq_sf_bytes(129, 64) == 2 * 512


def test_sfa_offset_places_each_scale_in_its_quadrant_column(dq):
    """A-operand scale layout: injective; row r's scales of 64-column block kb land in the 16-byte
    line (row r, column half kb % 2) of their 4 KB block, at 32-bit word r // 32 of that line, so that
    after a 128x256-bit copy lane r holds them in tensor-memory column 4 (kb % 2) + r // 32."""
    for rows, cols in ((128, 256), (256, 512), (300, 1024)):
        total = dq.dq_sfa_bytes(rows, cols)
        assert total == -(-rows // 128) * (cols // 256) * 8192
        seen = np.zeros(total, bool)
        for r in range(rows):
            for b in range(cols // 16):
                off = dq.dq_sfa_offset(r, b, cols)
                assert not seen[off]
                seen[off] = True
                kb, rr = b // 4, r % 128
                block, inner = divmod(off, 4096)
                assert block == ((r // 128) * (cols // 256) + kb // 4) * 2 + (kb // 2) % 2
                line, byte = divmod(inner, 16)
                # core matrices of 8 rows x 16 bytes: row-group stride 256, column-half stride 128
                assert line == (rr // 8) * 16 + (kb % 2) * 8 + rr % 8
                assert byte == (rr // 32) * 4 + b % 4
        assert seen.sum() == rows * cols // 16
    with pytest.raises(dq.DQError):
        dq.dq_sfa_offset(0, 0, 192)


def test_sfb_offset_replicates_each_column_scale_into_every_quadrant(dq):
    """B-operand scale layout: the four per-quadrant copies of all scales cover every byte exactly once;
    the copy in lane r of the 4 KB block holds (row, block) with r % 32 == row % 32, in 32-bit word
    4 (n / 128) + (n % 128) / 32 (n = row % 256), byte block % 4 of that word."""
    for rows, cols in ((256, 64), (512, 256)):
        total = dq.dq_sfb_bytes(rows, cols)
        assert total == (rows // 256) * (cols // 64) * 4096
        seen = np.zeros(total, bool)
        for r in range(rows):
            for b in range(cols // 16):
                off0 = dq.dq_sfb_offset(r, b, cols)
                for q in range(4):
                    off = off0 + 1024 * q
                    assert not seen[off]
                    seen[off] = True
                    block, inner = divmod(off, 4096)
                    assert block == (r // 256) * (cols // 64) + b // 4
                    lane = (inner // 256) * 8 + (inner % 128) // 16
                    byte = ((inner % 256) // 128) * 16 + inner % 16
                    n = r % 256
                    assert lane == 32 * q + r % 32
                    assert byte // 4 == 4 * (n // 128) + (n % 128) // 32 and byte % 4 == b % 4
        assert seen.all()


def test_layouts_are_aligned_and_ordered(dq):
    L = dq.dq_workspace_layout_get(21, 30, 52, 1, 2, 2, 5120, 5120, 32)
    offs = [L.off_status, L.off_scalars, L.off_kamax, L.off_s8, L.off_q8, L.off_q8_bf16, L.off_dcodes,
            L.off_dscales, L.off_u_part, L.off_u_hilo, L.off_p, L.total_bytes]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert L.N == 32760 and L.K == 8190 and L.slab == 64
    P = dq.dq_packed_weight_layout(5120, 5120, 32)
    assert P.off_codes == 256 and P.off_codes % 256 == 0 and P.off_scales % 256 == 0 and P.off_dqw % 256 == 0
    assert P.off_bias >= P.off_dqw + 5120 * 5120 * 2 and P.off_bias % 256 == 0
    assert P.total_bytes >= P.off_bias + 5120 * 4
    assert dq.dq_lowrank_slab_width(16) == 64 and dq.dq_lowrank_slab_width(48) == 128


def test_argument_checks_before_any_launch(dq):
    ws = 256 * 1024
    good = dict(X=0x10000, packed_W=0x20000, L1_mma=0x30000, L2_slab=0x40000, Y=0x50000, workspace=0x60000)

    def call(T=4, H=8, W=8, t=1, h=2, w=2, Ci=256, Co=256, r=16, ws_bytes=1 << 40, **ptrs):
        a = dict(good)
        a.update(ptrs)
        return dq._lib.dq_linear_forward_ex(a["X"], T, H, W, t, h, w, Ci, Co, r, a["packed_W"], a["L1_mma"],
                                            a["L2_slab"], a["Y"], a["workspace"], ws_bytes, 7, None, None)

    assert call(Ci=100) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(Co=384) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(r=24) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(r=256, Ci=512, Co=512) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(t=5) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(t=4, h=9, w=8) == dq.DQ_ERR_UNSUPPORTED_SHAPE       # cube taller than the lattice
    assert call(T=0) == dq.DQ_ERR_INVALID_ARG
    assert call(X=0) == dq.DQ_ERR_INVALID_ARG
    assert call(Y=0x50008) == dq.DQ_ERR_ALIGNMENT
    assert call(ws_bytes=ws) == dq.DQ_ERR_WORKSPACE_TOO_SMALL
    assert dq._lib.dq_linear_forward_ex(0x10000, 4, 8, 8, 1, 2, 2, 256, 256, 16, 0x20000, 0x30000, 0x40000, 0x50000,
                                        0x60000, 1 << 40, 32, None, None) == dq.DQ_ERR_INVALID_ARG   # unknown stage bit
