"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/ssm.h declares, and rejects bad arguments with the documented
status codes before launching anything. Pointers here are fake addresses; every
case fails validation, so none is ever dereferenced."""
import ctypes
import os
import re
import subprocess

import pytest

from mamba_selective_scan_sm_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_abi.LIB_PATH):
        from mamba_selective_scan_sm_b200 import build
        build.build()
    return _abi.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(ssm_\w+)\s*\(", src, flags=re.M)))


def test_header_and_binding_agree():
    assert declared_functions() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ssm_\w+)", out))
    assert set(declared_functions()) <= exported
    for name in declared_functions():
        assert hasattr(lib, name)


def test_version_and_status_strings(lib):
    assert lib.ssm_abi_version() == _abi.ABI_VERSION == 4
    for code, name in _abi.STATUS.items():
        assert lib.ssm_status_string(code)
    assert lib.ssm_status_string(999) == b"unknown status"


FAKE = 0x7F0000000000   # 256-byte aligned fake device address, never dereferenced


def _args(**kw):
    a = _abi.ScanArgs()
    a.dtype, a.batch, a.dim, a.seqlen, a.dstate = 1, 2, 64, 128, 16
    base = FAKE
    for i, f in enumerate(["u", "delta", "A", "B", "C", "out"]):
        setattr(a, f, base + i * (1 << 24))
    a.delta_softplus = 1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def _scan(lib, a):
    return lib.ssm_selective_scan_fwd(ctypes.byref(a), None)


@pytest.mark.parametrize("field,value,status", [
    ("dtype", 7, "SSM_ERR_BAD_DTYPE"),
    ("dstate", 0, "SSM_ERR_BAD_SHAPE"),
    ("dstate", 129, "SSM_ERR_BAD_SHAPE"),
    ("a_heads", 5, "SSM_ERR_BAD_SHAPE"),          # does not divide dim 64
    ("a_heads", -1, "SSM_ERR_BAD_SHAPE"),
    ("bc_shared", 2, "SSM_ERR_BAD_SHAPE"),
    ("seqlen", -1, "SSM_ERR_BAD_SHAPE"),
    ("batch", 70000, "SSM_ERR_UNSUPPORTED"),
    ("num_chunks", -2, "SSM_ERR_BAD_SHAPE"),
    ("u", None, "SSM_ERR_NULL_ARG"),
    ("A", None, "SSM_ERR_NULL_ARG"),
    ("out", None, "SSM_ERR_NULL_ARG"),
    ("u", FAKE + 1, "SSM_ERR_MISALIGNED"),
    ("A", FAKE + 2, "SSM_ERR_MISALIGNED"),
    ("out", FAKE + (1 << 24) + 64, "SSM_ERR_ALIAS"),
    ("final_state_rev", FAKE + (1 << 30), "SSM_ERR_UNSUPPORTED"),
])
def test_scan_rejects_bad_arguments(lib, field, value, status):
    a = _args(**{field: value})
    assert _scan(lib, a) == _abi.STATUS_CODE[status]
    assert lib.ssm_last_error_detail()


def test_scan_conv_width_and_bidirectional_chunks(lib):
    assert _scan(lib, _args(conv_weight=FAKE + (1 << 30), conv_width=5)) == 2
    a = _args(A_rev=FAKE + (1 << 30), num_chunks=4)
    assert _scan(lib, a) == _abi.STATUS_CODE["SSM_ERR_UNSUPPORTED"]


CONV = dict(conv_weight=FAKE + (1 << 30), conv_width=4)


@pytest.mark.parametrize("kw,status", [
    (dict(initial_state=FAKE + (1 << 29), reverse=1), "SSM_ERR_UNSUPPORTED"),
    (dict(initial_state=FAKE + (1 << 29), A_rev=FAKE + (1 << 30)), "SSM_ERR_UNSUPPORTED"),
    (dict(conv_history=FAKE + (1 << 29), reverse=1, **CONV), "SSM_ERR_UNSUPPORTED"),
    (dict(conv_history=FAKE + (1 << 29)), "SSM_ERR_NULL_ARG"),
    (dict(conv_state_out=FAKE + (1 << 29)), "SSM_ERR_NULL_ARG"),
    (dict(initial_state=FAKE + (1 << 29) + 2), "SSM_ERR_MISALIGNED"),
    (dict(conv_history=FAKE + (1 << 29) + 1, **CONV), "SSM_ERR_MISALIGNED"),
    (dict(conv_state_out=FAKE + 64, **CONV), "SSM_ERR_ALIAS"),                 # inside u
    (dict(conv_state_out=FAKE + 5 * (1 << 24) + 64, **CONV), "SSM_ERR_ALIAS"),  # inside out
    (dict(conv_state_out=FAKE + (1 << 29), conv_history=FAKE + (1 << 29) + 96, **CONV),
     "SSM_ERR_ALIAS"),
    (dict(initial_state=FAKE + (1 << 29), final_state=FAKE + (1 << 29) + 64, num_chunks=4,
          seqlen=4096, workspace=FAKE + (1 << 31), workspace_bytes=1 << 20), "SSM_ERR_ALIAS"),
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=3), "SSM_ERR_UNSUPPORTED"),            # batch 2
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=3, batch=1, reverse=1), "SSM_ERR_UNSUPPORTED"),
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=3, batch=1, A_rev=FAKE + (1 << 30)),
     "SSM_ERR_UNSUPPORTED"),
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=3, batch=1, initial_state=FAKE + (1 << 28)),
     "SSM_ERR_UNSUPPORTED"),
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=0, batch=1), "SSM_ERR_BAD_SHAPE"),
    (dict(seq_starts=FAKE + (1 << 29) + 2, num_seqs=3, batch=1), "SSM_ERR_MISALIGNED"),
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=3, batch=1, a_heads=4), "SSM_ERR_UNSUPPORTED"),
    (dict(seq_starts=FAKE + (1 << 29), num_seqs=3, batch=1, bc_shared=1), "SSM_ERR_UNSUPPORTED"),
    # time-invariant B, C are fp32: 4-byte alignment even for bf16 activations
    (dict(bc_shared=1, B=FAKE + 3 * (1 << 24) + 2), "SSM_ERR_MISALIGNED"),
])
def test_scan_continuation_arguments(lib, kw, status):
    """initial_state / conv_history / conv_state_out: forward scans, a fused conv for the
    conv ones, aligned, and outputs that do not overlap what the scan reads; packed
    sequences: batch 1, forward, no initial state or history, at least one sequence."""
    assert _scan(lib, _args(**kw)) == _abi.STATUS_CODE[status]
    assert lib.ssm_last_error_detail()


@pytest.mark.parametrize("mirror,ctype", [(_abi.ScanArgs, "ssm_scan_args_t"),
                                           (_abi.UpdateArgs, "ssm_update_args_t")])
def test_args_layout_matches_header(tmp_path, mirror, ctype):
    """The ctypes mirrors have the C structs' sizes and field offsets (compiled with gcc)."""
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    names = [f[0] for f in mirror._fields_]
    body = "\n".join(f'printf("%zu\\n", offsetof({ctype}, {n}));' for n in names)
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"ssm.h\"\n"
                   "int main(void) {\n" + body +
                   f'\nprintf("%zu\\n", sizeof({ctype}));\nreturn 0;\n}}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", inc, str(src), "-o", str(exe)])
    got = [int(v) for v in subprocess.check_output([str(exe)]).split()]
    want = [getattr(mirror, n).offset for n in names] + [ctypes.sizeof(mirror)]
    assert got == want


def test_scan_args_null(lib):
    assert lib.ssm_selective_scan_fwd(None, None) == 1
    n = ctypes.c_size_t()
    assert lib.ssm_selective_scan_workspace_size(None, ctypes.byref(n)) == 1


def test_workspace_size_query(lib):
    n = ctypes.c_size_t()
    a = _args(num_chunks=1)
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 0                               # single pass, one direction
    # automatic: 2 x 64 channels in 8-channel CTAs fill few of the 148 SMs' slots, so the
    # sequence (2 tiles of 64 bf16 steps in these narrow splits) is split into as many
    # chunks as it has tiles: one summary chunk
    a = _args()
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 1 * 2 * 64 * 16 * 8
    a = _args(dtype=0)                                # fp32: 8 tiles of 16 steps
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 7 * 2 * 64 * 16 * 8
    a = _args(dim=9472 * 2)                           # enough channels: one pass
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 0
    a = _args(num_chunks=4, batch=1, dim=64, seqlen=4096)
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 3 * 1 * 64 * 16 * 8              # (chunks-1) x rows x states x (P, S)
    a = _args(A_rev=FAKE + (1 << 30))                 # bf16 bidirectional: fp32 partial
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 2 * 64 * 128 * 4
    a = _args(A_rev=FAKE + (1 << 30), dtype=0)        # fp32 bidirectional: out holds it
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 0
    # d_state 100 runs in the 128-state split: the carry holds 128 (P, S) pairs per row
    a = _args(num_chunks=4, batch=1, dim=64, seqlen=4096, dstate=100, a_heads=8)
    assert lib.ssm_selective_scan_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 3 * 1 * 64 * 128 * 8


def test_scan_workspace_too_small(lib):
    a = _args(num_chunks=4, seqlen=4096, workspace=FAKE + (1 << 31), workspace_bytes=16)
    assert _scan(lib, a) == _abi.STATUS_CODE["SSM_ERR_WORKSPACE"]
    a = _args(num_chunks=4, seqlen=4096)
    assert _scan(lib, a) == _abi.STATUS_CODE["SSM_ERR_WORKSPACE"]


def test_conv_rejects_bad_arguments(lib):
    f = lib.ssm_causal_conv1d_fwd
    X, W, O = FAKE, FAKE + (1 << 24), FAKE + (1 << 25)
    assert f(X, W, None, O, 2, 4, 16, 4, 1, 9, None) == 3
    assert f(X, W, None, O, 2, 4, 16, 5, 1, 1, None) == 2
    assert f(X, W, None, O, 2, 4, -1, 4, 1, 1, None) == 2
    assert f(None, W, None, O, 2, 4, 16, 4, 1, 1, None) == 1
    assert f(X + 1, W, None, O, 2, 4, 16, 4, 1, 1, None) == 4
    assert f(X, W, None, X + 8, 2, 4, 16, 4, 1, 1, None) == 9
    assert f(None, None, None, None, 0, 4, 16, 4, 1, 1, None) == 0   # empty: nothing to do


def test_state_update_rejects_bad_arguments(lib):
    f = lib.ssm_selective_state_update
    p = [FAKE + i * (1 << 24) for i in range(16)]
    good = [p[0], p[1], p[2], p[3], p[4], p[5], p[6], None, None, None, 1, None, None, 0, p[7],
            4, 8, 16, 1, None]
    bad = list(good); bad[17] = 17
    assert f(*bad) == 2
    bad = list(good); bad[0] = None
    assert f(*bad) == 1
    bad = list(good); bad[18] = 5
    assert f(*bad) == 3
    bad = list(good); bad[0] = p[0] + 2
    assert f(*bad) == 4
    bad = list(good); bad[11] = p[8]; bad[13] = 4; bad[1] = None   # conv without conv_state
    assert f(*bad) == 1
    bad = list(good); bad[14] = p[2]                                # out aliases x
    assert f(*bad) == 9
    z = list(good); z[15] = 0
    assert f(*z) == 0                                               # empty batch


def test_device_error_null(lib):
    assert lib.ssm_device_error(None, None) == 1


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(_abi.LibraryMissing):
        _abi.load(str(tmp_path / "missing.so"))


def test_wait_selftest_rejects_limits_out_of_range(lib):
    assert lib.ssm_wait_selftest(10, None) == _abi.STATUS_CODE["SSM_ERR_BAD_SHAPE"]
    assert lib.ssm_wait_selftest(10 ** 10, None) == _abi.STATUS_CODE["SSM_ERR_BAD_SHAPE"]



def test_binding_workspace_query_for_heads_and_time_invariant_bc(lib):
    """The binding's host-only workspace query with A given per head (d_state must then
    be passed) and with time-invariant B/C; CPU tensors are enough (shapes only)."""
    import torch
    import mamba_selective_scan_sm_b200 as ssm
    u = torch.empty(1, 64, 4096, dtype=torch.bfloat16)
    A_heads = torch.empty(8)
    with pytest.raises(ValueError):
        ssm.ssm_selective_scan_workspace_size(u, A_heads, num_chunks=4)
    n = ssm.ssm_selective_scan_workspace_size(u, A_heads, num_chunks=4, dstate=128)
    assert n == 3 * 64 * 128 * 8                      # (chunks-1) x rows x 128 x (P, S)
    A = torch.empty(64, 16)
    n = ssm.ssm_selective_scan_workspace_size(u, A, num_chunks=4, bc_shared=True)
    assert n == 3 * 64 * 16 * 8
    with pytest.raises(RuntimeError):                 # 64 channels are not 5 whole heads
        ssm.ssm_selective_scan_workspace_size(u, torch.empty(5), num_chunks=4, dstate=16)


def _update_args(**kw):
    a = _abi.UpdateArgs()
    a.dtype, a.batch, a.dim, a.dstate = 1, 2, 64, 128
    for i, f in enumerate(["state", "x", "dt", "A", "B_t", "C_t", "out"]):
        setattr(a, f, FAKE + i * (1 << 24))
    a.dt_softplus = 1
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(dstate=129), "SSM_ERR_BAD_SHAPE"),
    (dict(a_heads=5), "SSM_ERR_BAD_SHAPE"),                 # does not divide dim 64
    (dict(a_heads=-2), "SSM_ERR_BAD_SHAPE"),
    (dict(dtype=9), "SSM_ERR_BAD_DTYPE"),
    (dict(x=None), "SSM_ERR_NULL_ARG"),
    (dict(state=FAKE + 2), "SSM_ERR_MISALIGNED"),
    (dict(out=FAKE + 1 * (1 << 24) + 64), "SSM_ERR_ALIAS"),  # inside x
    (dict(conv_weight=FAKE + (1 << 30), conv_width=4, conv_state=FAKE + 4096),
     "SSM_ERR_ALIAS"),                                       # conv state inside the SSM state
    (dict(conv_weight=FAKE + (1 << 30), conv_width=4), "SSM_ERR_NULL_ARG"),
    (dict(dstate=16, a_heads=0, conv_weight=FAKE + (1 << 30), conv_width=7), "SSM_ERR_BAD_SHAPE"),
])
def test_state_update_ex_rejects_bad_arguments(lib, kw, status):
    """The decode entry for d_state up to 128 and A per head validates before launching
    (d_state <= 16 with per-state A goes through the first entry's checks)."""
    assert lib.ssm_selective_state_update_ex(ctypes.byref(_update_args(**kw)), None) == \
        _abi.STATUS_CODE[status]
    assert lib.ssm_last_error_detail()
    assert lib.ssm_selective_state_update_ex(None, None) == _abi.STATUS_CODE["SSM_ERR_NULL_ARG"]
