"""Host logic of the feed-forward block (no GPU): which pairs of cube partitions
let the up-projection's epilogue form the down-projection's statistics.

dq_ffn_fused_statistics (the library's O(N) check on its own cube-major row map)
against a statement built on the oracle's cube enumeration: every down cube's
tokens, in its (t,h,w) order, sit on consecutive rows of the up-projection's
cube-major order inside one aligned group of 32 rows, and hold at most 32 tokens."""
import numpy as np
import pytest

import oracle


def _fusable(T, H, W, cu, cd):
    if int(np.prod(cd)) > 32:
        return False
    ou, od = oracle.cube_order(T, H, W, *cu), oracle.cube_order(T, H, W, *cd)
    for k in range(od["count"].size):
        f, c = od["first"][k], od["count"][k]
        ru = ou["row_of_n"][od["n_of_row"][f:f + c]]
        if not np.array_equal(ru, ru[0] + np.arange(c)) or ru[0] // 32 != ru[-1] // 32:
            return False
    return True


CASES = [(21, 45, 80, (2, 2, 2), (1, 2, 2)), (3, 5, 12, (2, 2, 2), (1, 2, 2)), (4, 8, 8, (1, 2, 2), (1, 2, 2)),
         (5, 6, 16, (2, 2, 4), (1, 1, 4)), (3, 7, 9, (1, 1, 1), (1, 1, 1)), (4, 8, 8, (1, 2, 2), (2, 1, 1)),
         (5, 7, 9, (2, 2, 2), (2, 2, 2)), (5, 7, 9, (1, 2, 2), (1, 1, 2)), (8, 6, 16, (4, 2, 8), (4, 2, 8)),
         (4, 4, 16, (2, 2, 8), (2, 2, 8)), (6, 16, 24, (2, 2, 2), (1, 2, 2)), (21, 30, 52, (1, 2, 2), (1, 2, 2)),
         (7, 9, 11, (1, 1, 1), (1, 1, 1)), (6, 8, 8, (2, 4, 4), (1, 4, 4)), (6, 8, 8, (2, 4, 4), (2, 2, 2)),
         (2, 3, 5, (2, 3, 5), (1, 1, 1))]


@pytest.mark.parametrize("T,H,W,cu,cd", CASES)
def test_fused_statistics_predicate(T, H, W, cu, cd):
    import video_diffusion_w4a4_b200 as dq
    assert dq.dq_ffn_fused_statistics(T, H, W, cu, cd) == _fusable(T, H, W, cu, cd)


def test_fused_statistics_rejects_bad_arguments():
    import video_diffusion_w4a4_b200 as dq
    with pytest.raises(dq.DQError):
        dq.dq_ffn_fused_statistics(4, 8, 8, (0, 2, 2), (1, 2, 2))
    with pytest.raises(dq.DQError):
        dq.dq_ffn_fused_statistics(4, 8, 8, (1, 2, 2), (5, 2, 2))


def test_ffn_forward_argument_errors():
    """dq_ffn_forward's argument checks, which run before any device call: flags, cubes,
    each layer's shape, the pointers, and both workspaces' sizes."""
    import ctypes

    import video_diffusion_w4a4_b200 as dq
    T, H, W, cu, cd = 4, 8, 8, (2, 2, 2), (1, 2, 2)
    Ci, Cf, Co, r = 256, 512, 256, 32
    fake = 1 << 20   # a 256-byte-aligned stand-in address; nothing is dereferenced on these paths
    ld = dq.dq_workspace_layout_opts(T, H, W, *cd, Cf, Co, r)

    def call(flags=0, cube_up=cu, Ci_=Ci, rank_down=r, ws_down_bytes=ld.total_bytes, ws_up_bytes=1 << 30, hid=fake):
        a3 = lambda c: (ctypes.c_int * 3)(*c)
        return dq._lib.dq_ffn_forward(fake, T, H, W, a3(cube_up), a3(cd), Ci_, Cf, Co, r, rank_down, fake, fake,
                                      fake, fake, fake, fake, hid or None, fake, fake, ws_up_bytes, fake,
                                      ws_down_bytes, flags, None, None)

    assert call(flags=2) == dq.DQ_ERR_INVALID_ARG
    assert call(cube_up=(0, 2, 2)) == dq.DQ_ERR_INVALID_ARG
    assert call(Ci_=300) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(rank_down=8) == dq.DQ_ERR_UNSUPPORTED_SHAPE
    assert call(ws_down_bytes=ld.total_bytes - 1) == dq.DQ_ERR_WORKSPACE_TOO_SMALL
    assert call(ws_up_bytes=16) == dq.DQ_ERR_WORKSPACE_TOO_SMALL
    assert call(hid=0) == dq.DQ_ERR_INVALID_ARG
    assert call(hid=fake + 16) == dq.DQ_ERR_ALIGNMENT


def test_epilogue_option_is_checked():
    import video_diffusion_w4a4_b200 as dq
    dq.dq_workspace_layout_opts(4, 8, 8, 1, 2, 2, 256, 256, 16, epilogue=dq.DQ_EPILOGUE_GELU)
    with pytest.raises(dq.DQError):
        dq.dq_workspace_layout_opts(4, 8, 8, 1, 2, 2, 256, 256, 16, epilogue=2)
