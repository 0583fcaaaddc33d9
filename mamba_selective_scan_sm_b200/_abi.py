"""ctypes view of the C ABI declared in include/ssm.h (no CUDA calls here)."""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libssm_b200.so")

SSM_F32, SSM_BF16 = 0, 1
STATUS = {
    0: "SSM_OK", 1: "SSM_ERR_NULL_ARG", 2: "SSM_ERR_BAD_SHAPE", 3: "SSM_ERR_BAD_DTYPE",
    4: "SSM_ERR_MISALIGNED", 5: "SSM_ERR_WORKSPACE", 6: "SSM_ERR_UNSUPPORTED", 7: "SSM_ERR_CUDA",
    8: "SSM_ERR_TIMEOUT", 9: "SSM_ERR_ALIAS",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

# Every symbol include/ssm.h declares.
EXPORTS = (
    "ssm_abi_version", "ssm_status_string", "ssm_last_error_detail", "ssm_causal_conv1d_fwd",
    "ssm_selective_scan_workspace_size", "ssm_selective_scan_fwd", "ssm_selective_state_update",
    "ssm_selective_state_update_ex", "ssm_device_error", "ssm_selective_scan_fwd_noalloc",
    "ssm_wait_selftest",
)
NOALLOC_SCRATCH_BYTES = 8 << 20
ABI_VERSION = 4            # SSM_ABI_VERSION of include/ssm.h this mirror follows

_P = ctypes.c_void_p
_FP = ctypes.POINTER(ctypes.c_float)
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64


class ScanArgs(ctypes.Structure):
    """Mirror of ssm_scan_args_t (field order and types as in include/ssm.h)."""
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("batch", _I64), ("dim", _I64), ("seqlen", _I64), ("dstate", _I64),
        ("u", _P), ("delta", _P), ("A", _P), ("B", _P), ("C", _P), ("D", _P), ("z", _P),
        ("delta_bias", _P), ("delta_softplus", _I32), ("reverse", _I32),
        ("conv_weight", _P), ("conv_bias", _P), ("conv_width", _I32),
        ("A_rev", _P), ("D_rev", _P), ("delta_bias_rev", _P),
        ("out", _P), ("final_state", _P), ("final_state_rev", _P),
        ("workspace", _P), ("workspace_bytes", ctypes.c_size_t),
        ("num_chunks", _I32),
        ("initial_state", _P), ("conv_history", _P), ("conv_state_out", _P),
        ("seq_starts", _P), ("num_seqs", _I32),
        ("channel_last", _I32), ("stride_u", _I64), ("stride_delta", _I64), ("stride_z", _I64),
        ("stride_out", _I64), ("stride_B", _I64), ("stride_C", _I64),
        ("a_heads", _I32), ("bc_shared", _I32),
    ]


class UpdateArgs(ctypes.Structure):
    """Mirror of ssm_update_args_t (field order and types as in include/ssm.h)."""
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("batch", _I64), ("dim", _I64), ("dstate", _I64),
        ("state", _P), ("conv_state", _P), ("x", _P), ("dt", _P), ("A", _P), ("B_t", _P),
        ("C_t", _P), ("D", _P), ("z", _P), ("dt_bias", _P), ("dt_softplus", _I32),
        ("conv_weight", _P), ("conv_bias", _P), ("conv_width", _I32), ("out", _P),
        ("a_heads", _I32),
    ]


class LibraryMissing(RuntimeError):
    pass


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Open libssm_b200.so and declare the ABI. Raises LibraryMissing if it is not built."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise LibraryMissing(
            f"{path} is not built; run `python -c 'import __graft_entry__ as g; g.build()'` "
            "or `python mamba_selective_scan_sm_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    lib.ssm_abi_version.restype = ctypes.c_int
    lib.ssm_abi_version.argtypes = []
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_status_string.argtypes = [ctypes.c_int]
    lib.ssm_last_error_detail.restype = ctypes.c_char_p
    lib.ssm_last_error_detail.argtypes = []
    lib.ssm_causal_conv1d_fwd.restype = ctypes.c_int
    lib.ssm_causal_conv1d_fwd.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I32, _I32,
                                          ctypes.c_int, _P]
    lib.ssm_selective_scan_workspace_size.restype = ctypes.c_int
    lib.ssm_selective_scan_workspace_size.argtypes = [ctypes.POINTER(ScanArgs),
                                                      ctypes.POINTER(ctypes.c_size_t)]
    lib.ssm_selective_scan_fwd.restype = ctypes.c_int
    lib.ssm_selective_scan_fwd.argtypes = [ctypes.POINTER(ScanArgs), _P]
    lib.ssm_selective_state_update.restype = ctypes.c_int
    lib.ssm_selective_state_update.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I32, _P,
                                               _P, _I32, _P, _I64, _I64, _I64, ctypes.c_int, _P]
    lib.ssm_selective_state_update_ex.restype = ctypes.c_int
    lib.ssm_selective_state_update_ex.argtypes = [ctypes.POINTER(UpdateArgs), _P]
    lib.ssm_selective_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssm_selective_scan_fwd_noalloc.argtypes = [ctypes.POINTER(ScanArgs), _P]
    lib.ssm_device_error.restype = ctypes.c_int
    lib.ssm_device_error.argtypes = [ctypes.POINTER(_I32), _P]
    lib.ssm_wait_selftest.restype = ctypes.c_int
    lib.ssm_wait_selftest.argtypes = [ctypes.c_uint64, _P]
    if lib.ssm_abi_version() != ABI_VERSION:
        raise LibraryMissing(f"{path} implements ABI {lib.ssm_abi_version()}, this binding "
                             f"expects {ABI_VERSION}: rebuild the library")
    if path == LIB_PATH:
        _lib = lib
    return lib


class SSMError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status
        self.name = STATUS.get(status, str(status))
        self.detail = detail


def check(lib, status: int) -> None:
    if status != 0:
        raise SSMError(status, (lib.ssm_last_error_detail() or b"").decode())
