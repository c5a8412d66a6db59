"""ctypes view of the C ABIs in include/jamba_ssm.h and include/jamba_ssm_proj.h
(argument marshalling only).

The structures below mirror the headers field by field.  Loading fails loudly
when a library has not been built: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libjamba_ssm.so")
PROJ_LIB_PATH = os.path.join(_PKG, "libjamba_ssm_proj.so")

(OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT,
 ERR_NO_DEVICE) = range(8)
STATUS_BYTES = 16  # JAMBA_SSM_STATUS_BYTES
BF16, F32 = 0, 1

# Every symbol the header declares.
EXPORTS = (
    "jamba_ssm_scan",
    "jamba_ssm_scan_workspace_size",
    "jamba_ssm_scan_ckpt_size",
    "jamba_ssm_scan_bwd",
    "jamba_ssm_scan_bwd_workspace_size",
    "jamba_ssm_scan_bwd_noalloc",
    "jamba_ssm_ssd_scan",
    "jamba_ssm_state_update",
    "jamba_ssm_scan_plan",
    "jamba_ssm_scan_variant_info",
    "jamba_ssm_get_status",
    "jamba_ssm_last_cuda_error",
    "jamba_ssm_status_string",
    "jamba_ssm_abi_version",
)
# Every symbol jamba_ssm_proj.h declares.
PROJ_EXPORTS = (
    "jamba_ssm_x_proj",
    "jamba_ssm_dt_proj",
    "jamba_ssm_proj_get_status",
    "jamba_ssm_proj_last_cuda_error",
    "jamba_ssm_proj_abi_version",
)

_vp = ctypes.c_void_p
_fp = ctypes.c_void_p  # float* passed as raw address


class ScanParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
        ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
        ("io_dtype", ctypes.c_int32), ("delta_softplus", ctypes.c_int32),
        ("x", _vp), ("delta", _vp), ("z", _vp),
        ("B", _vp), ("C", _vp),
        ("A", _fp), ("D", _fp), ("delta_bias", _fp), ("h0", _fp),
        ("out", _vp), ("h_final", _fp),
        ("kernel_variant", ctypes.c_int32), ("debug_flags", ctypes.c_uint32),
        ("timeout_cycles", ctypes.c_uint64),
        # ABI version 2
        ("cu_seqlens", _vp), ("total_tokens", ctypes.c_int64),
        ("state_indices", _vp), ("num_slots", ctypes.c_int64),
        # ABI version 3
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        # ABI version 4
        ("ckpt", _fp),
    ]


class StateUpdateParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("batch", ctypes.c_int64), ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
        ("io_dtype", ctypes.c_int32), ("delta_softplus", ctypes.c_int32),
        ("state", _fp),
        ("x", _vp), ("delta", _vp), ("z", _vp),
        ("B", _vp), ("C", _vp),
        ("A", _fp), ("D", _fp), ("delta_bias", _fp),
        ("out", _vp),
        # ABI version 2
        ("state_indices", _vp), ("num_slots", ctypes.c_int64),
        ("debug_flags", ctypes.c_uint32), ("timeout_cycles", ctypes.c_uint64),
        # ABI version 3
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
    ]


class ScanBwdParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
        ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
        ("io_dtype", ctypes.c_int32), ("delta_softplus", ctypes.c_int32),
        ("x", _vp), ("delta", _vp), ("z", _vp),
        ("B", _vp), ("C", _vp),
        ("A", _fp), ("D", _fp), ("delta_bias", _fp), ("h0", _fp),
        ("dout", _vp), ("dh_final", _fp),
        ("dx", _vp), ("ddelta", _vp), ("dz", _vp),
        ("dB", _vp), ("dC", _vp),
        ("dA", _fp), ("dD", _fp), ("ddelta_bias", _fp), ("dh0", _fp),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("debug_flags", ctypes.c_uint32), ("timeout_cycles", ctypes.c_uint64),
        # ABI version 4
        ("ckpt", _fp),
    ]


class SsdParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
        ("headdim", ctypes.c_int64), ("d_state", ctypes.c_int64),
        ("io_dtype", ctypes.c_int32), ("delta_softplus", ctypes.c_int32),
        ("x", _vp), ("delta", _vp), ("z", _vp),
        ("B", _vp), ("C", _vp),
        ("A", _fp), ("D", _fp), ("delta_bias", _fp), ("h0", _fp),
        ("out", _vp), ("h_final", _fp),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("debug_flags", ctypes.c_uint32), ("timeout_cycles", ctypes.c_uint64),
    ]


class DtProjParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("ntok", ctypes.c_int64), ("d_inner", ctypes.c_int64), ("dt_rank", ctypes.c_int64),
        ("dt_low_hi", _vp), ("dt_low_lo", _vp), ("W_dt", _vp), ("delta", _vp),
        ("timeout_cycles", ctypes.c_uint64),
        ("debug_flags", ctypes.c_uint32),  # version 2
    ]


class XProjParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_size_t),
        ("ntok", ctypes.c_int64), ("d_inner", ctypes.c_int64), ("dt_rank", ctypes.c_int64),
        ("d_state", ctypes.c_int64),
        ("u", _vp), ("W_x", _vp), ("w_dt", _fp), ("w_B", _fp), ("w_C", _fp),
        ("eps", ctypes.c_float), ("k_split", ctypes.c_int32),
        ("dt_low_hi", _vp), ("dt_low_lo", _vp), ("B", _vp), ("C", _vp),
        ("timeout_cycles", ctypes.c_uint64),
        ("debug_flags", ctypes.c_uint32),  # version 2
    ]


class JambaSSMError(RuntimeError):
    def __init__(self, status: int, what: str, cuda_error=None):
        self.status = status
        msg = status_string(status)
        if status == ERR_CUDA:
            code = lib().jamba_ssm_last_cuda_error() if cuda_error is None else cuda_error
            msg += f" (cudaError {code})"
        super().__init__(f"{what}: {msg}")


_lock = threading.Lock()
_lib = None
_proj_lib = None


def lib():
    """Load libjamba_ssm.so (raises if it is missing: build it first)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is not built; run selective_state_space_26_b200.build.build()"
                        " (nvcc, sm_100a). There is no CPU fallback.")
                L = ctypes.CDLL(LIB_PATH)
                L.jamba_ssm_scan.restype = ctypes.c_int
                L.jamba_ssm_scan.argtypes = [ctypes.POINTER(ScanParams), _vp]
                L.jamba_ssm_state_update.restype = ctypes.c_int
                L.jamba_ssm_state_update.argtypes = [ctypes.POINTER(StateUpdateParams), _vp]
                i32p, i64p = ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int64)
                L.jamba_ssm_scan_plan.restype = ctypes.c_int
                L.jamba_ssm_scan_plan.argtypes = [ctypes.POINTER(ScanParams), i32p, i32p, i32p,
                                                  i32p, i64p]
                L.jamba_ssm_scan_variant_info.restype = ctypes.c_int
                L.jamba_ssm_scan_variant_info.argtypes = [ctypes.c_int32] + [i32p] * 5
                L.jamba_ssm_get_status.restype = ctypes.c_int
                L.jamba_ssm_get_status.argtypes = [_vp, _vp]
                L.jamba_ssm_scan_workspace_size.restype = ctypes.c_size_t
                L.jamba_ssm_scan_workspace_size.argtypes = [ctypes.c_int64] * 4
                L.jamba_ssm_scan_ckpt_size.restype = ctypes.c_size_t
                L.jamba_ssm_scan_ckpt_size.argtypes = [ctypes.c_int64] * 4
                L.jamba_ssm_scan_bwd.restype = ctypes.c_int
                L.jamba_ssm_scan_bwd.argtypes = [ctypes.POINTER(ScanBwdParams), _vp]
                L.jamba_ssm_ssd_scan.restype = ctypes.c_int
                L.jamba_ssm_ssd_scan.argtypes = [ctypes.POINTER(SsdParams), _vp]
                L.jamba_ssm_scan_bwd_noalloc.restype = ctypes.c_int
                L.jamba_ssm_scan_bwd_noalloc.argtypes = [ctypes.POINTER(ScanBwdParams), _vp]
                L.jamba_ssm_scan_bwd_workspace_size.restype = ctypes.c_size_t
                L.jamba_ssm_scan_bwd_workspace_size.argtypes = [ctypes.c_int64] * 4
                L.jamba_ssm_last_cuda_error.restype = ctypes.c_int
                L.jamba_ssm_last_cuda_error.argtypes = []
                L.jamba_ssm_status_string.restype = ctypes.c_char_p
                L.jamba_ssm_status_string.argtypes = [ctypes.c_int]
                L.jamba_ssm_abi_version.restype = ctypes.c_int
                L.jamba_ssm_abi_version.argtypes = []
                _lib = L
    return _lib


def proj_lib():
    """Load libjamba_ssm_proj.so (raises if it is missing: build it first)."""
    global _proj_lib
    if _proj_lib is None:
        with _lock:
            if _proj_lib is None:
                if not os.path.exists(PROJ_LIB_PATH):
                    raise RuntimeError(
                        f"{PROJ_LIB_PATH} is not built; run selective_state_space_26_b200.build."
                        "build() (nvcc, sm_100a). There is no CPU fallback.")
                L = ctypes.CDLL(PROJ_LIB_PATH)
                L.jamba_ssm_x_proj.restype = ctypes.c_int
                L.jamba_ssm_x_proj.argtypes = [ctypes.POINTER(XProjParams), _vp]
                L.jamba_ssm_dt_proj.restype = ctypes.c_int
                L.jamba_ssm_dt_proj.argtypes = [ctypes.POINTER(DtProjParams), _vp]
                L.jamba_ssm_proj_get_status.restype = ctypes.c_int
                L.jamba_ssm_proj_get_status.argtypes = [_vp]
                L.jamba_ssm_proj_last_cuda_error.restype = ctypes.c_int
                L.jamba_ssm_proj_last_cuda_error.argtypes = []
                L.jamba_ssm_proj_abi_version.restype = ctypes.c_int
                L.jamba_ssm_proj_abi_version.argtypes = []
                _proj_lib = L
    return _proj_lib


def status_string(status: int) -> str:
    return lib().jamba_ssm_status_string(int(status)).decode()


# struct_size of the ABI version 1 and 2 structures (the fields before the
# next version's), for callers built against those versions
SCAN_PARAMS_V1_SIZE = ScanParams.cu_seqlens.offset
STATE_UPDATE_PARAMS_V1_SIZE = StateUpdateParams.state_indices.offset
SCAN_PARAMS_V2_SIZE = ScanParams.workspace.offset
STATE_UPDATE_PARAMS_V2_SIZE = StateUpdateParams.workspace.offset
SCAN_PARAMS_V3_SIZE = ScanParams.ckpt.offset
SCAN_BWD_PARAMS_V3_SIZE = ScanBwdParams.ckpt.offset


def new_scan_params(**kw) -> ScanParams:
    p = ScanParams()
    p.struct_size = ctypes.sizeof(ScanParams)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def new_state_update_params(**kw) -> StateUpdateParams:
    p = StateUpdateParams()
    p.struct_size = ctypes.sizeof(StateUpdateParams)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def call_scan(p: ScanParams, stream: int) -> int:
    return lib().jamba_ssm_scan(ctypes.byref(p), _vp(stream or None))


def call_state_update(p: StateUpdateParams, stream: int) -> int:
    return lib().jamba_ssm_state_update(ctypes.byref(p), _vp(stream or None))


def scan_plan(p: ScanParams):
    v, g, cc, grid = (ctypes.c_int32() for _ in range(4))
    tasks = ctypes.c_int64()
    st = lib().jamba_ssm_scan_plan(ctypes.byref(p), ctypes.byref(v), ctypes.byref(g),
                                   ctypes.byref(cc), ctypes.byref(grid), ctypes.byref(tasks))
    if st != OK:
        raise JambaSSMError(st, "jamba_ssm_scan_plan")
    return dict(variant=v.value, lanes_per_channel=g.value, channels_per_cta=cc.value,
                grid=grid.value, tasks=tasks.value)


def variant_info(k: int):
    vals = [ctypes.c_int32() for _ in range(5)]
    st = lib().jamba_ssm_scan_variant_info(int(k), *[ctypes.byref(v) for v in vals])
    if st != OK:
        return None
    keys = ("io_dtype", "d_state", "lanes_per_channel", "warps_per_cta", "time_tile")
    return dict(zip(keys, (v.value for v in vals)))


def get_status(stream: int, workspace: int = 0) -> int:
    return lib().jamba_ssm_get_status(_vp(workspace or None), _vp(stream or None))


def scan_workspace_size(batch: int, seqlen: int, d_inner: int, d_state: int) -> int:
    return lib().jamba_ssm_scan_workspace_size(batch, seqlen, d_inner, d_state)


def scan_ckpt_size(batch: int, seqlen: int, d_inner: int, d_state: int) -> int:
    return lib().jamba_ssm_scan_ckpt_size(batch, seqlen, d_inner, d_state)


def scan_bwd_workspace_size(batch: int, seqlen: int, d_inner: int, d_state: int) -> int:
    return lib().jamba_ssm_scan_bwd_workspace_size(batch, seqlen, d_inner, d_state)


def new_scan_bwd_params(**kw) -> ScanBwdParams:
    p = ScanBwdParams()
    p.struct_size = ctypes.sizeof(ScanBwdParams)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def new_ssd_params(**kw) -> SsdParams:
    p = SsdParams()
    p.struct_size = ctypes.sizeof(SsdParams)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def call_ssd(p: SsdParams, stream: int) -> int:
    return lib().jamba_ssm_ssd_scan(ctypes.byref(p), _vp(stream or None))


def call_scan_bwd(p: ScanBwdParams, stream: int) -> int:
    return lib().jamba_ssm_scan_bwd(ctypes.byref(p), _vp(stream or None))


def new_dt_proj_params(**kw) -> DtProjParams:
    p = DtProjParams()
    p.struct_size = ctypes.sizeof(DtProjParams)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def new_x_proj_params(**kw) -> XProjParams:
    p = XProjParams()
    p.struct_size = ctypes.sizeof(XProjParams)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def call_x_proj(p: XProjParams, stream: int) -> int:
    return proj_lib().jamba_ssm_x_proj(ctypes.byref(p), _vp(stream or None))


def call_dt_proj(p: DtProjParams, stream: int) -> int:
    return proj_lib().jamba_ssm_dt_proj(ctypes.byref(p), _vp(stream or None))


def proj_get_status(stream: int) -> int:
    return proj_lib().jamba_ssm_proj_get_status(_vp(stream or None))
