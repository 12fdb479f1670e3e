"""Python binding of libdeltaquant (the C ABI in include/deltaquant.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels (or, for the offline packer, its C++ host code).  Device
buffers are passed as torch tensors (their data_ptr) or raw integer
addresses; streams as torch.cuda.Stream or raw cudaStream_t integers.  The
functions keep the C names.  If the shared library is missing this module
raises ImportError: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdeltaquant.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python video_diffusion_w4a4_b200/build.py` "
                      "(or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

DQ_OK = 0
DQ_ERR_INVALID_ARG = 1
DQ_ERR_UNSUPPORTED_SHAPE = 2
DQ_ERR_ALIGNMENT = 3
DQ_ERR_WORKSPACE_TOO_SMALL = 4
DQ_ERR_CUDA = 5
DQ_ERR_DEVICE_TIMEOUT = 6
DQ_ERR_BAD_PACKED_WEIGHT = 7
DQ_ERR_NO_DEVICE = 8
DQ_ERR_ALLOC = 9
DQ_STAGE_QUANTIZE, DQ_STAGE_KERNEL_GEMM, DQ_STAGE_MAIN_GEMM, DQ_STAGE_ALL = 1, 2, 4, 7
DQ_STAGE_STATS, DQ_STAGE_ENCODE = 8, 16
DQ_KERNEL_SCALE_PER_TOKEN, DQ_KERNEL_SCALE_GROUP64 = 0, 64
DQ_NOALLOC_WORKSPACE = 1   # dq_read_device_status: the fixed array of dq_linear_forward_noalloc
DQ_PACK_C2 = 1
DQ_KERNEL_PRODUCT_BF16, DQ_KERNEL_PRODUCT_FP8 = 0, 1
DQ_DELTA_SCALE_AMAX, DQ_DELTA_SCALE_POW2 = 0, 1
DQ_HOST_OVERLAP_PREVIOUS = 1
DQ_EPILOGUE_NONE, DQ_EPILOGUE_GELU = 0, 1
DQ_FFN_SEPARATE_STATISTICS = 1


class dq_packed_layout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t), ("off_codes", ctypes.c_size_t), ("off_scales", ctypes.c_size_t),
                ("off_dqw", ctypes.c_size_t), ("off_bias", ctypes.c_size_t), ("Co", ctypes.c_int), ("Ci", ctypes.c_int), ("rank", ctypes.c_int),
                ("slab", ctypes.c_int)]


class dq_workspace_layout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t)] + [
        (n, ctypes.c_size_t) for n in ("off_status", "off_scalars", "off_kamax", "off_s8", "off_q8", "off_q8_bf16",
                                       "off_dcodes", "off_dscales", "off_u_part", "off_u_hilo", "off_p", "off_means")] + [
        ("N", ctypes.c_longlong), ("K", ctypes.c_longlong), ("N_pad", ctypes.c_longlong), ("K_pad", ctypes.c_longlong),
        ("splits", ctypes.c_int), ("slab", ctypes.c_int), ("kernel_group", ctypes.c_int), ("off_prov", ctypes.c_size_t)]


class dq_forward_options(ctypes.Structure):
    _fields_ = [("kernel_group", ctypes.c_int), ("kernel_product", ctypes.c_int), ("delta_scale", ctypes.c_int),
                ("epilogue", ctypes.c_int)]


_P, _I, _SZ, _LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
_SIGS = {
    "dq_status_string": ([_I], ctypes.c_char_p),
    "dq_last_cuda_error": ([], ctypes.c_char_p),
    "dq_abi_version": ([], _I),
    "dq_cube_count": ([_I] * 6 + [ctypes.POINTER(_LL)], _I),
    "dq_cube_major_row": ([_I] * 6 + [_LL, ctypes.POINTER(_LL), ctypes.POINTER(_LL)], _I),
    "dq_sf_offset": ([_LL, _I, _I, ctypes.POINTER(_SZ)], _I),
    "dq_sf_bytes": ([_LL, _I, ctypes.POINTER(_SZ)], _I),
    "dq_sfa_offset": ([_LL, _I, _I, ctypes.POINTER(_SZ)], _I),
    "dq_sfb_offset": ([_LL, _I, _I, ctypes.POINTER(_SZ)], _I),
    "dq_sfb_bytes": ([_LL, _I, ctypes.POINTER(_SZ)], _I),
    "dq_sfa_bytes": ([_LL, _I, ctypes.POINTER(_SZ)], _I),
    "dq_packed_weight_layout": ([_I, _I, _I, ctypes.POINTER(dq_packed_layout)], _I),
    "dq_packed_weight_bytes": ([_I, _I, _I, ctypes.POINTER(_SZ)], _I),
    "dq_lowrank_slab_width": ([_I], _I),
    "dq_lowrank_factors": ([_P, _I, _I, _I, ctypes.c_uint64, _P, _P], _I),
    "dq_pack_weight_factors": ([_P, _P, _P, _I, _I, _I, _P, _SZ, _P, _P, ctypes.POINTER(ctypes.c_float)], _I),
    "dq_pack_weight": ([_P, _I, _I, _I, _P, _SZ, _P, _P], _I),
    "dq_pack_weight_factors_ex": ([_P, _P, _P, _I, _I, _I, _I, _P, _SZ, _P, _P, ctypes.POINTER(ctypes.c_float)], _I),
    "dq_workspace_layout_opts": ([_I] * 9 + [ctypes.POINTER(dq_forward_options), ctypes.POINTER(dq_workspace_layout)],
                                 _I),
    "dq_linear_forward_opts": ([_P] + [_I] * 9 + [ctypes.POINTER(dq_forward_options), _P, _P, _P, _P, _P, _SZ, _I, _P,
                                                   _P], _I),
    "dq_pack_bias": ([_P, _I, _P, _SZ], _I),
    "dq_workspace_layout_get": ([_I] * 9 + [ctypes.POINTER(dq_workspace_layout)], _I),
    "dq_workspace_bytes": ([_I] * 9 + [ctypes.POINTER(_SZ)], _I),
    "dq_linear_forward": ([_P] + [_I] * 9 + [_P, _P, _P, _P, _P], _I),
    "dq_linear_forward_ex": ([_P] + [_I] * 9 + [_P, _P, _P, _P, _P, _SZ, _I, _P, _P], _I),
    "dq_linear_forward_grouped": ([_P] + [_I] * 10 + [_P, _P, _P, _P, _P, _SZ, _I, _P, _P], _I),
    "dq_workspace_layout_grouped": ([_I] * 10 + [ctypes.POINTER(dq_workspace_layout)], _I),
    "dq_workspace_bytes_grouped": ([_I] * 10 + [ctypes.POINTER(_SZ)], _I),
    "dq_linear_forward_host": ([_P] + [_I] * 9 + [_P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "dq_linear_forward_host_ex": ([_P] + [_I] * 9 + [_P, _P, _P, _P, _P, _P, _P, _SZ, _I, _P], _I),
    "dq_linear_forward_noalloc": ([_P] + [_I] * 9 + [_P, _P, _P, _P, _P], _I),
    "dq_read_device_status": ([_P, _P, ctypes.POINTER(_I), _I], _I),
    "dq_ffn_forward": ([_P, _I, _I, _I, _P, _P] + [_I] * 5 + [_P] * 8 + [_P, _SZ, _P, _SZ, _I, _P, _P], _I),
    "dq_ffn_fused_statistics": ([_I, _I, _I, _P, _P, ctypes.POINTER(_I)], _I),
    "dq_ffn_forward_opts": ([_P, _I, _I, _I, _P, _P] + [_I] * 5 +
                            [ctypes.POINTER(dq_forward_options), ctypes.POINTER(dq_forward_options)] + [_P] * 8 +
                            [_P, _SZ, _P, _SZ, _I, _P, _P], _I),
    "dq_selftest_bounded_wait": ([_I, _P, ctypes.POINTER(_I)], _I),
    "dq_selftest_convert": ([_P, _LL, _P, _P, _P, _P], _I),
    "dq_selftest_gelu": ([_P, _LL, _P, _P], _I),
    "dq_selftest_divide": ([_LL, ctypes.c_uint64, ctypes.POINTER(ctypes.c_ulonglong), _P, _P], _I),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class DQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        detail = f" [{_lib.dq_last_cuda_error().decode()}]" if status == DQ_ERR_CUDA else ""
        super().__init__(f"{fn}: {dq_status_string(status)} ({status}){detail}")
        self.status = status


def _check(fn: str, rc: int) -> None:
    if rc != DQ_OK:
        raise DQError(fn, rc)


def _ptr(x) -> int | None:
    """Device/host address of a torch tensor, numpy array or raw int."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ------------------------------------------------------------------ layout maps

def dq_status_string(status: int) -> str:
    return _lib.dq_status_string(status).decode()


def dq_abi_version() -> int:
    return _lib.dq_abi_version()


def dq_cube_count(T, H, W, t, h, w) -> int:
    K = ctypes.c_longlong()
    _check("dq_cube_count", _lib.dq_cube_count(T, H, W, t, h, w, ctypes.byref(K)))
    return K.value


def dq_cube_major_row(T, H, W, t, h, w, n) -> tuple[int, int]:
    row, cube = ctypes.c_longlong(), ctypes.c_longlong()
    _check("dq_cube_major_row", _lib.dq_cube_major_row(T, H, W, t, h, w, n, ctypes.byref(row), ctypes.byref(cube)))
    return row.value, cube.value


def dq_sf_offset(row: int, block: int, cols: int) -> int:
    off = ctypes.c_size_t()
    _check("dq_sf_offset", _lib.dq_sf_offset(row, block, cols, ctypes.byref(off)))
    return off.value


def dq_sfa_offset(row: int, block: int, cols: int) -> int:
    off = _SZ()
    _check("dq_sfa_offset", _lib.dq_sfa_offset(row, block, cols, ctypes.byref(off)))
    return off.value


def dq_sfb_offset(row: int, block: int, cols: int) -> int:
    off = _SZ()
    _check("dq_sfb_offset", _lib.dq_sfb_offset(row, block, cols, ctypes.byref(off)))
    return off.value


def dq_sfb_bytes(rows: int, cols: int) -> int:
    b = _SZ()
    _check("dq_sfb_bytes", _lib.dq_sfb_bytes(rows, cols, ctypes.byref(b)))
    return b.value


def dq_sfa_bytes(rows: int, cols: int) -> int:
    b = _SZ()
    _check("dq_sfa_bytes", _lib.dq_sfa_bytes(rows, cols, ctypes.byref(b)))
    return b.value


def dq_sf_bytes(rows: int, cols: int) -> int:
    b = ctypes.c_size_t()
    _check("dq_sf_bytes", _lib.dq_sf_bytes(rows, cols, ctypes.byref(b)))
    return b.value


def dq_lowrank_slab_width(rank: int) -> int:
    return _lib.dq_lowrank_slab_width(rank)


def dq_packed_weight_layout(Co, Ci, rank) -> dq_packed_layout:
    L = dq_packed_layout()
    _check("dq_packed_weight_layout", _lib.dq_packed_weight_layout(Co, Ci, rank, ctypes.byref(L)))
    return L


def dq_packed_weight_bytes(Co, Ci, rank) -> int:
    b = ctypes.c_size_t()
    _check("dq_packed_weight_bytes", _lib.dq_packed_weight_bytes(Co, Ci, rank, ctypes.byref(b)))
    return b.value


# ------------------------------------------------------------------ offline packing (host arrays)

def dq_lowrank_factors(W: np.ndarray, rank: int, seed: int = 0):
    """W: uint16 BF16 bits (Co, Ci).  Returns (L1 (Ci, r), L2 (r, Co)) as BF16 bits."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    Co, Ci = W.shape
    L1 = np.empty((Ci, rank), np.uint16)
    L2 = np.empty((rank, Co), np.uint16)
    _check("dq_lowrank_factors", _lib.dq_lowrank_factors(W.ctypes.data, Co, Ci, rank, seed, L1.ctypes.data,
                                                         L2.ctypes.data))
    return L1, L2


def dq_pack_weight_factors(W: np.ndarray, L1: np.ndarray, L2: np.ndarray, pack_flags: int = 0):
    """Returns (packed blob uint8, L1_mma (r, Ci) BF16 bits, L2_slab (Co, slab) BF16 bits, S_W).
    pack_flags: 0 or DQ_PACK_C2 (dq_pack_weight_factors_ex)."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    L1 = np.ascontiguousarray(L1, dtype=np.uint16)
    L2 = np.ascontiguousarray(L2, dtype=np.uint16)
    Co, Ci = W.shape
    r = L1.shape[1]
    lay = dq_packed_weight_layout(Co, Ci, r)
    packed = np.empty(lay.total_bytes, np.uint8)
    L1m = np.empty((r, Ci), np.uint16)
    L2s = np.empty((Co, lay.slab), np.uint16)
    S = ctypes.c_float()
    _check("dq_pack_weight_factors_ex",
           _lib.dq_pack_weight_factors_ex(W.ctypes.data, L1.ctypes.data, L2.ctypes.data, Co, Ci, r, pack_flags,
                                          packed.ctypes.data, packed.size, L1m.ctypes.data, L2s.ctypes.data,
                                          ctypes.byref(S)))
    return packed, L1m, L2s, S.value


def dq_pack_bias(packed: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    """Set (bias: uint16 BF16 bits, (Co,)) or clear (None) the bias of a host packed blob, in place."""
    assert packed.dtype == np.uint8 and packed.flags["C_CONTIGUOUS"]
    Co = int(packed[8:12].view(np.int32)[0])
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    if b is not None and b.size != Co:
        raise ValueError(f"bias has {b.size} values, the packed weight has Co = {Co}")
    _check("dq_pack_bias", _lib.dq_pack_bias(None if b is None else b.ctypes.data, Co, packed.ctypes.data,
                                             packed.size))
    return packed


def dq_pack_weight(W: np.ndarray, rank: int):
    """SVD factors (seed 0) + packing.  Returns (packed, L1_mma, L2_slab)."""
    W = np.ascontiguousarray(W, dtype=np.uint16)
    Co, Ci = W.shape
    lay = dq_packed_weight_layout(Co, Ci, rank)
    packed = np.empty(lay.total_bytes, np.uint8)
    L1m = np.empty((rank, Ci), np.uint16)
    L2s = np.empty((Co, lay.slab), np.uint16)
    _check("dq_pack_weight", _lib.dq_pack_weight(W.ctypes.data, Co, Ci, rank, packed.ctypes.data, packed.size,
                                                 L1m.ctypes.data, L2s.ctypes.data))
    return packed, L1m, L2s


# ------------------------------------------------------------------ online (device)

def dq_workspace_layout_get(T, H, W, t, h, w, Ci, Co, rank) -> dq_workspace_layout:
    L = dq_workspace_layout()
    _check("dq_workspace_layout_get", _lib.dq_workspace_layout_get(T, H, W, t, h, w, Ci, Co, rank, ctypes.byref(L)))
    return L


def dq_workspace_layout_grouped(T, H, W, t, h, w, Ci, Co, rank, kernel_group) -> dq_workspace_layout:
    """Workspace carve-up for a kernel-token scale granularity (DQ_KERNEL_SCALE_*)."""
    L = dq_workspace_layout()
    _check("dq_workspace_layout_grouped", _lib.dq_workspace_layout_grouped(T, H, W, t, h, w, Ci, Co, rank,
                                                                           kernel_group, ctypes.byref(L)))
    return L


def _options(kernel_group=DQ_KERNEL_SCALE_PER_TOKEN, kernel_product=DQ_KERNEL_PRODUCT_BF16,
             delta_scale=DQ_DELTA_SCALE_AMAX, epilogue=DQ_EPILOGUE_NONE):
    o = dq_forward_options()
    o.kernel_group, o.kernel_product, o.delta_scale, o.epilogue = kernel_group, kernel_product, delta_scale, epilogue
    return o


def dq_workspace_layout_opts(T, H, W, t, h, w, Ci, Co, rank, kernel_group=DQ_KERNEL_SCALE_PER_TOKEN,
                             kernel_product=DQ_KERNEL_PRODUCT_BF16, delta_scale=DQ_DELTA_SCALE_AMAX,
                             epilogue=DQ_EPILOGUE_NONE) -> dq_workspace_layout:
    """Workspace carve-up for the forward options (dq_forward_options fields as keywords)."""
    L = dq_workspace_layout()
    o = _options(kernel_group, kernel_product, delta_scale, epilogue)
    _check("dq_workspace_layout_opts", _lib.dq_workspace_layout_opts(T, H, W, t, h, w, Ci, Co, rank, ctypes.byref(o),
                                                                     ctypes.byref(L)))
    return L


def dq_linear_forward_opts(X, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y, workspace,
                           workspace_bytes, stage_mask=DQ_STAGE_ALL, stage_events=None, stream=None,
                           kernel_group=DQ_KERNEL_SCALE_PER_TOKEN, kernel_product=DQ_KERNEL_PRODUCT_BF16,
                           delta_scale=DQ_DELTA_SCALE_AMAX, epilogue=DQ_EPILOGUE_NONE) -> None:
    """dq_linear_forward_ex with forward options (dq_forward_options fields as keywords)."""
    o = _options(kernel_group, kernel_product, delta_scale, epilogue)
    _check("dq_linear_forward_opts",
           _lib.dq_linear_forward_opts(_ptr(X), T, H, W, t, h, w, Ci, Co, rank, ctypes.byref(o), _ptr(packed_W),
                                       _ptr(L1_mma), _ptr(L2_slab), _ptr(Y), _ptr(workspace), workspace_bytes,
                                       stage_mask, _events(stage_events), _stream(stream)))


def dq_ffn_fused_statistics(T, H, W, cube_up, cube_down) -> bool:
    """Whether dq_ffn_forward forms the down-projection's statistics in the up-projection's epilogue."""
    cu, cd = (ctypes.c_int * 3)(*cube_up), (ctypes.c_int * 3)(*cube_down)
    f = ctypes.c_int()
    _check("dq_ffn_fused_statistics", _lib.dq_ffn_fused_statistics(T, H, W, cu, cd, ctypes.byref(f)))
    return bool(f.value)


def dq_ffn_forward(X, T, H, W, cube_up, cube_down, Ci, Cf, Co, rank_up, rank_down, packed_up, L1_up, L2_up,
                   packed_down, L1_down, L2_down, Hid, Y, ws_up, ws_up_bytes, ws_down, ws_down_bytes, ffn_flags=0,
                   stage_events=None, stream=None) -> None:
    """A feed-forward block: Hid = BF16(GELU(up(X))), Y = down(Hid) (include/deltaquant.h)."""
    cu, cd = (ctypes.c_int * 3)(*cube_up), (ctypes.c_int * 3)(*cube_down)
    _check("dq_ffn_forward",
           _lib.dq_ffn_forward(_ptr(X), T, H, W, cu, cd, Ci, Cf, Co, rank_up, rank_down, _ptr(packed_up), _ptr(L1_up),
                               _ptr(L2_up), _ptr(packed_down), _ptr(L1_down), _ptr(L2_down), _ptr(Hid), _ptr(Y),
                               _ptr(ws_up), ws_up_bytes, _ptr(ws_down), ws_down_bytes, ffn_flags,
                               _events(stage_events, 8), _stream(stream)))


def dq_ffn_forward_opts(X, T, H, W, cube_up, cube_down, Ci, Cf, Co, rank_up, rank_down, packed_up, L1_up, L2_up,
                        packed_down, L1_down, L2_down, Hid, Y, ws_up, ws_up_bytes, ws_down, ws_down_bytes, ffn_flags=0,
                        stage_events=None, stream=None, opts_up=None, opts_down=None) -> None:
    """dq_ffn_forward with per-layer forward options: opts_up / opts_down are dicts of
    dq_forward_options fields (kernel_group, kernel_product, delta_scale), None for the defaults."""
    cu, cd = (ctypes.c_int * 3)(*cube_up), (ctypes.c_int * 3)(*cube_down)
    ou = _options(**(opts_up or {}))
    od = _options(**(opts_down or {}))
    _check("dq_ffn_forward_opts",
           _lib.dq_ffn_forward_opts(_ptr(X), T, H, W, cu, cd, Ci, Cf, Co, rank_up, rank_down, ctypes.byref(ou),
                                    ctypes.byref(od), _ptr(packed_up), _ptr(L1_up), _ptr(L2_up), _ptr(packed_down),
                                    _ptr(L1_down), _ptr(L2_down), _ptr(Hid), _ptr(Y), _ptr(ws_up), ws_up_bytes,
                                    _ptr(ws_down), ws_down_bytes, ffn_flags, _events(stage_events, 8),
                                    _stream(stream)))


def dq_workspace_bytes_grouped(T, H, W, t, h, w, Ci, Co, rank, kernel_group) -> int:
    """Workspace bytes for a kernel-token scale granularity (DQ_KERNEL_SCALE_*)."""
    b = ctypes.c_size_t()
    _check("dq_workspace_bytes_grouped", _lib.dq_workspace_bytes_grouped(T, H, W, t, h, w, Ci, Co, rank, kernel_group,
                                                                         ctypes.byref(b)))
    return b.value


def dq_workspace_bytes(T, H, W, t, h, w, Ci, Co, rank) -> int:
    b = ctypes.c_size_t()
    _check("dq_workspace_bytes", _lib.dq_workspace_bytes(T, H, W, t, h, w, Ci, Co, rank, ctypes.byref(b)))
    return b.value


def dq_linear_forward(X, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y, stream=None) -> None:
    _check("dq_linear_forward", _lib.dq_linear_forward(_ptr(X), T, H, W, t, h, w, Ci, Co, rank, _ptr(packed_W),
                                                       _ptr(L1_mma), _ptr(L2_slab), _ptr(Y), _stream(stream)))


def _events(stage_events, n: int = 4):
    if stage_events is None:
        return None
    handles = [e.cuda_event if hasattr(e, "cuda_event") else e for e in stage_events]
    if len(handles) != n or not all(handles):
        raise ValueError(f"stage_events needs {n} created CUDA events (record a torch.cuda.Event once first)")
    arr = (ctypes.c_void_p * n)(*handles)
    return ctypes.cast(arr, ctypes.c_void_p)


def dq_linear_forward_grouped(X, T, H, W, t, h, w, Ci, Co, rank, kernel_group, packed_W, L1_mma, L2_slab, Y,
                              workspace, workspace_bytes, stage_mask=DQ_STAGE_ALL, stage_events=None,
                              stream=None) -> None:
    """dq_linear_forward_ex with kernel_group: DQ_KERNEL_SCALE_PER_TOKEN or DQ_KERNEL_SCALE_GROUP64."""
    _check("dq_linear_forward_grouped",
           _lib.dq_linear_forward_grouped(_ptr(X), T, H, W, t, h, w, Ci, Co, rank, kernel_group, _ptr(packed_W),
                                          _ptr(L1_mma), _ptr(L2_slab), _ptr(Y), _ptr(workspace), workspace_bytes,
                                          stage_mask, _events(stage_events), _stream(stream)))


def dq_linear_forward_ex(X, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y, workspace,
                         workspace_bytes, stage_mask=DQ_STAGE_ALL, stage_events=None, stream=None) -> None:
    ev = _events(stage_events)
    _check("dq_linear_forward_ex",
           _lib.dq_linear_forward_ex(_ptr(X), T, H, W, t, h, w, Ci, Co, rank, _ptr(packed_W), _ptr(L1_mma),
                                     _ptr(L2_slab), _ptr(Y), _ptr(workspace), workspace_bytes, stage_mask, ev,
                                     _stream(stream)))


def dq_linear_forward_host(X_host, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y_host, X_dev, Y_dev,
                           workspace, workspace_bytes, stream=None) -> None:
    _check("dq_linear_forward_host",
           _lib.dq_linear_forward_host(_ptr(X_host), T, H, W, t, h, w, Ci, Co, rank, _ptr(packed_W), _ptr(L1_mma),
                                       _ptr(L2_slab), _ptr(Y_host), _ptr(X_dev), _ptr(Y_dev), _ptr(workspace),
                                       workspace_bytes, _stream(stream)))


def dq_linear_forward_host_ex(X_host, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y_host, X_dev,
                              Y_dev, workspace, workspace_bytes, host_flags=0, stream=None) -> None:
    """dq_linear_forward_host with host_flags (DQ_HOST_OVERLAP_PREVIOUS)."""
    _check("dq_linear_forward_host_ex",
           _lib.dq_linear_forward_host_ex(_ptr(X_host), T, H, W, t, h, w, Ci, Co, rank, _ptr(packed_W),
                                          _ptr(L1_mma), _ptr(L2_slab), _ptr(Y_host), _ptr(X_dev), _ptr(Y_dev),
                                          _ptr(workspace), workspace_bytes, host_flags, _stream(stream)))


def dq_linear_forward_noalloc(X, T, H, W, t, h, w, Ci, Co, rank, packed_W, L1_mma, L2_slab, Y, stream=None) -> None:
    _check("dq_linear_forward_noalloc",
           _lib.dq_linear_forward_noalloc(_ptr(X), T, H, W, t, h, w, Ci, Co, rank, _ptr(packed_W), _ptr(L1_mma),
                                          _ptr(L2_slab), _ptr(Y), _stream(stream)))


def dq_read_device_status(workspace=None, stream=None, clear: bool = False) -> int:
    s = ctypes.c_int()
    _check("dq_read_device_status",
           _lib.dq_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(s), int(clear)))
    return s.value


def dq_selftest_bounded_wait(budget_us: int, stream=None) -> int:
    s = ctypes.c_int()
    _check("dq_selftest_bounded_wait", _lib.dq_selftest_bounded_wait(budget_us, _stream(stream), ctypes.byref(s)))
    return s.value


def dq_selftest_convert(inp, n, e2m1, e4m3, e4m3_value, stream=None) -> None:
    _check("dq_selftest_convert", _lib.dq_selftest_convert(_ptr(inp), n, _ptr(e2m1), _ptr(e4m3), _ptr(e4m3_value),
                                                           _stream(stream)))


def dq_selftest_gelu(inp, n, out, stream=None) -> None:
    _check("dq_selftest_gelu", _lib.dq_selftest_gelu(_ptr(inp), n, _ptr(out), _stream(stream)))


def dq_selftest_divide(n: int, seed: int = 1, stream=None):
    """Returns (mismatch count, first mismatching (a, b) or None)."""
    cnt = ctypes.c_ulonglong()
    ab = np.zeros(2, np.float32)
    _check("dq_selftest_divide", _lib.dq_selftest_divide(n, seed, ctypes.byref(cnt), ab.ctypes.data, _stream(stream)))
    return cnt.value, (tuple(ab.tolist()) if cnt.value else None)


def loaded_library_path() -> str:
    return LIB_PATH
