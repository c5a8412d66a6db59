"""Host-side checks of the C ABIs that need no GPU: each library loads, exports
every function its header (include/jamba_ssm.h, include/jamba_ssm_proj.h)
declares, its structures have the layout the binding assumes, and argument
validation rejects bad calls before any CUDA work is enqueued (fake,
never-dereferenced pointer values are enough)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from selective_state_space_26_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jamba_ssm.h")
PROJ_HEADER = os.path.join(ROOT, "include", "jamba_ssm_proj.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jamba_ssm_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTS), names
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in names:
        assert n in exported, f"{n} declared in the header but not exported"
        assert hasattr(L, n)


@pytest.fixture(scope="module")
def P():
    build.build()
    return _lib.proj_lib()


def test_every_declared_proj_symbol_is_exported(P):
    names = declared_functions(PROJ_HEADER)
    assert set(names) == set(_lib.PROJ_EXPORTS), names
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.PROJ_LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for n in names:
        assert n in exported, f"{n} declared in the header but not exported"
    # the projection library keeps its kernels and status word to itself
    assert not [e for e in exported if "jssm" in e], "internal symbols exported"
    assert P.jamba_ssm_proj_abi_version() == 2


def test_struct_layout_matches_header(tmp_path):
    fields = {
        "jamba_ssm_scan_params": _lib.ScanParams,
        "jamba_ssm_state_update_params": _lib.StateUpdateParams,
        "jamba_ssm_dt_proj_params": _lib.DtProjParams,
        "jamba_ssm_x_proj_params": _lib.XProjParams,
    }
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "jamba_ssm.h"',
             '#include "jamba_ssm_proj.h"', "int main(void) {"]
    for cname, cls in fields.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), "-o", str(exe), str(src)], check=True)
    got = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    for row in filter(None, got):
        cname, f, v = row.split()
        cls = fields[cname]
        if f == "size":
            assert ctypes.sizeof(cls) == int(v), cname
        else:
            assert getattr(cls, f).offset == int(v), (cname, f)


def test_status_strings_and_version(L):
    assert L.jamba_ssm_abi_version() == 4
    for s in range(8):
        assert _lib.status_string(s) != "unknown status"
    assert _lib.status_string(99) == "unknown status"


def test_status_codes_match_header(tmp_path):
    """The binding's status constants are the header's enum values (the
    contract's order: ERR_WORKSPACE = 4, ERR_CUDA = 5, ERR_TIMEOUT = 6)."""
    names = ["OK", "ERR_INVALID_ARG", "ERR_UNSUPPORTED", "ERR_MISALIGNED", "ERR_WORKSPACE",
             "ERR_CUDA", "ERR_TIMEOUT", "ERR_NO_DEVICE"]
    body = "".join(f'printf("{n} %d\\n", (int)JAMBA_SSM_{n});' for n in names)
    src = tmp_path / "enums.c"
    src.write_text('#include <stdio.h>\n#include "jamba_ssm.h"\nint main(void) {' + body +
                   'printf("STATUS_BYTES %d\\n", JAMBA_SSM_STATUS_BYTES); return 0; }')
    exe = tmp_path / "enums"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), "-o", str(exe), str(src)], check=True)
    got = dict(line.split() for line in subprocess.run(
        [str(exe)], capture_output=True, text=True, check=True).stdout.splitlines())
    for n in names:
        assert int(got[n]) == getattr(_lib, n), n
    assert (_lib.ERR_WORKSPACE, _lib.ERR_CUDA, _lib.ERR_TIMEOUT) == (4, 5, 6)
    assert int(got["STATUS_BYTES"]) == _lib.STATUS_BYTES


def test_scan_workspace_size(L):
    """The scan stores no carry between chunks of a sequence, so its workspace
    is the status block at every size."""
    for sizes in [(1, 4096, 8192, 16), (16, 16384, 8192, 16), (1, 1 << 18, 8192, 16),
                  (0, 0, 8, 1), (3, 77, 64, 4)]:
        assert _lib.scan_workspace_size(*sizes) == _lib.STATUS_BYTES


def test_variant_table(L):
    infos = []
    k = 1
    while (info := _lib.variant_info(k)) is not None:
        infos.append(info)
        k += 1
    assert len(infos) >= 9
    for i in infos:
        ns = i["d_state"] // i["lanes_per_channel"]
        assert ns * i["lanes_per_channel"] == i["d_state"]
        assert ns == 2 or ns % 4 == 0
        assert 32 % i["lanes_per_channel"] == 0
        assert i["time_tile"] % i["lanes_per_channel"] == 0
    assert _lib.variant_info(0) is None


def _valid_scan(**kw):
    base = dict(batch=2, seqlen=100, d_inner=256, d_state=16, io_dtype=_lib.BF16,
                delta_softplus=1, x=0x10000000, delta=0x20000000, z=0x30000000,
                B=0x40000000, C=0x50000000, A=0x60000000, D=0x70000000,
                delta_bias=0x80000000, h0=None, out=0x90000000, h_final=0xA0000000)
    base.update(kw)
    return _lib.new_scan_params(**base)


def _scan(p):
    return _lib.call_scan(p, 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(batch=-1), _lib.ERR_INVALID_ARG),
    (dict(seqlen=-5), _lib.ERR_INVALID_ARG),
    (dict(d_inner=0), _lib.ERR_INVALID_ARG),
    (dict(io_dtype=7), _lib.ERR_INVALID_ARG),
    (dict(d_state=5), _lib.ERR_UNSUPPORTED),
    (dict(d_state=3), _lib.ERR_UNSUPPORTED),
    (dict(d_state=32), _lib.ERR_UNSUPPORTED),
    (dict(d_state=4, batch=70000, seqlen=1), _lib.ERR_UNSUPPORTED),  # small-state grid
    (dict(d_inner=12), _lib.ERR_UNSUPPORTED),         # bf16 row not a multiple of 16 bytes
    (dict(kernel_variant=99), _lib.ERR_UNSUPPORTED),
    (dict(kernel_variant=8), _lib.ERR_UNSUPPORTED),   # an fp32 variant for bf16 data
    (dict(kernel_variant=5), _lib.ERR_UNSUPPORTED),   # a d_state=8 variant for d_state=16
    (dict(x=None), _lib.ERR_INVALID_ARG),
    (dict(A=None), _lib.ERR_INVALID_ARG),
    (dict(out=None), _lib.ERR_INVALID_ARG),
    (dict(x=0x10000002), _lib.ERR_MISALIGNED),
    (dict(B=0x40000008), _lib.ERR_MISALIGNED),
    (dict(h0=0xB0000004), _lib.ERR_MISALIGNED),
    (dict(D=0x70000002), _lib.ERR_MISALIGNED),
    (dict(out=0x10000000 + 64), _lib.ERR_INVALID_ARG),  # out overlaps x
    (dict(h_final=0x90000000 + 1024), _lib.ERR_INVALID_ARG),  # h_final inside out
    (dict(h0=0xA0000000 + 16), _lib.ERR_INVALID_ARG),  # h0 partially overlaps h_final
    (dict(batch=1 << 20, seqlen=1 << 20, d_inner=1 << 12), _lib.ERR_UNSUPPORTED),
    (dict(io_dtype=_lib.F32, d_state=6), _lib.ERR_UNSUPPORTED),
    (dict(io_dtype=_lib.F32, d_inner=10), _lib.ERR_UNSUPPORTED),
    (dict(workspace=0xC0000008, workspace_bytes=64), _lib.ERR_MISALIGNED),
    (dict(workspace=0xC0000000, workspace_bytes=8), _lib.ERR_WORKSPACE),
    (dict(workspace=0xC0000000, workspace_bytes=0), _lib.ERR_WORKSPACE),
])
def test_scan_argument_errors(L, kw, expect):
    assert _scan(_valid_scan(**kw)) == expect


def test_scan_struct_size_and_null(L):
    p = _valid_scan()
    p.struct_size = 8
    assert _scan(p) == _lib.ERR_INVALID_ARG
    assert L.jamba_ssm_scan(None, None) == _lib.ERR_INVALID_ARG
    assert L.jamba_ssm_state_update(None, None) == _lib.ERR_INVALID_ARG


def _valid_update(**kw):
    base = dict(batch=4, d_inner=64, d_state=16, io_dtype=_lib.BF16, delta_softplus=1,
                state=0x10000000, x=0x20000000, delta=0x30000000, z=0x40000000,
                B=0x50000000, C=0x60000000, A=0x70000000, D=None, delta_bias=None,
                out=0x80000000)
    base.update(kw)
    return _lib.new_state_update_params(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(batch=-1), _lib.ERR_INVALID_ARG),
    (dict(d_state=3), _lib.ERR_UNSUPPORTED),
    (dict(d_state=12), _lib.ERR_UNSUPPORTED),
    (dict(d_state=2, batch=70000), _lib.ERR_UNSUPPORTED),  # small-state grid
    (dict(d_state=2, state=0x10000002), _lib.ERR_MISALIGNED),
    (dict(workspace=0x90000004, workspace_bytes=16), _lib.ERR_MISALIGNED),
    (dict(workspace=0x90000000, workspace_bytes=4), _lib.ERR_WORKSPACE),
    (dict(state=None), _lib.ERR_INVALID_ARG),
    (dict(state=0x10000008), _lib.ERR_MISALIGNED),
    (dict(x=0x20000001), _lib.ERR_MISALIGNED),
    (dict(io_dtype=_lib.F32, x=0x20000002), _lib.ERR_MISALIGNED),
    (dict(out=0x20000000), _lib.ERR_INVALID_ARG),     # out aliases x
    (dict(out=0x10000000 + 256), _lib.ERR_INVALID_ARG),  # out inside the state
])
def test_state_update_argument_errors(L, kw, expect):
    assert _lib.call_state_update(_valid_update(**kw), 0) == expect


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_no_device(L):
    assert _scan(_valid_scan()) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    assert _lib.call_state_update(_valid_update(), 0) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    # every d_state of the contract passes validation (the small ones too)
    for n in (1, 2, 4, 8, 16):
        for io in (_lib.BF16, _lib.F32):
            assert _scan(_valid_scan(d_state=n, io_dtype=io)) in \
                (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA), (n, io)
            assert _lib.call_state_update(_valid_update(d_state=n, io_dtype=io), 0) in \
                (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA), (n, io)
    # a big enough, aligned workspace is accepted
    assert _scan(_valid_scan(workspace=0xC0000000, workspace_bytes=16)) in \
        (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    p = _valid_scan(batch=0)
    assert _scan(p) == _lib.OK or _scan(p) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)


@pytest.mark.parametrize("kw,expect", [
    (dict(cu_seqlens=0x1000, total_tokens=-1), _lib.ERR_INVALID_ARG),
    (dict(cu_seqlens=0x1002, total_tokens=64), _lib.ERR_MISALIGNED),
    (dict(state_indices=0x2000, num_slots=0), _lib.ERR_INVALID_ARG),
    (dict(state_indices=0x2001, num_slots=4), _lib.ERR_MISALIGNED),
    (dict(cu_seqlens=0x1000, total_tokens=1 << 32), _lib.ERR_UNSUPPORTED),
    # packed: out overlapping x is measured with total_tokens rows
    (dict(cu_seqlens=0x1000, total_tokens=64, out=0x10000000 + 256 * 2 * 10),
     _lib.ERR_INVALID_ARG),
    # a state cache of num_slots rows that overlaps out
    (dict(state_indices=0x2000, num_slots=1 << 20, h_final=0x90000000 - 1024),
     _lib.ERR_INVALID_ARG),
])
def test_serving_layout_argument_errors(L, kw, expect):
    assert _scan(_valid_scan(**kw)) == expect


def test_state_update_slot_argument_errors(L):
    assert _lib.call_state_update(_valid_update(state_indices=0x3000, num_slots=0), 0) == \
        _lib.ERR_INVALID_ARG
    assert _lib.call_state_update(_valid_update(state_indices=0x3002, num_slots=8), 0) == \
        _lib.ERR_MISALIGNED
    # a cache of num_slots rows is checked for overlap with out
    assert _lib.call_state_update(_valid_update(state_indices=0x3000, num_slots=1 << 16,
                                                out=0x10000000 + (1 << 20)), 0) == \
        _lib.ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_version_1_struct_size_is_accepted(L):
    """A caller built against ABI version 1 passes the shorter struct: the
    serving fields read as absent and validation goes on to the device."""
    p = _valid_scan()
    p.struct_size = _lib.SCAN_PARAMS_V1_SIZE
    p.cu_seqlens = 0x1002  # garbage past the version-1 size: must be ignored
    assert _scan(p) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    p.struct_size = _lib.SCAN_PARAMS_V1_SIZE - 8
    assert _scan(p) == _lib.ERR_INVALID_ARG
    u = _valid_update()
    u.struct_size = _lib.STATE_UPDATE_PARAMS_V1_SIZE
    u.state_indices = 0x3001
    assert _lib.call_state_update(u, 0) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    u.struct_size = _lib.STATE_UPDATE_PARAMS_V1_SIZE - 8
    assert _lib.call_state_update(u, 0) == _lib.ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_version_2_struct_size_is_accepted(L):
    """A version-2 caller's struct ends before the workspace fields: whatever
    lies past it is ignored (no workspace)."""
    p = _valid_scan(workspace=0xC0000004, workspace_bytes=1)  # invalid if it were read
    p.struct_size = _lib.SCAN_PARAMS_V2_SIZE
    assert _scan(p) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    u = _valid_update(workspace=0x90000004, workspace_bytes=1)
    u.struct_size = _lib.STATE_UPDATE_PARAMS_V2_SIZE
    assert _lib.call_state_update(u, 0) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)


_A16 = 0x7f0000000000  # fake, 16-byte aligned, never dereferenced


def _dt_proj_call(P, **kw):
    base = dict(ntok=300, d_inner=8192, dt_rank=256, dt_low_hi=_A16, dt_low_lo=_A16 + 0x1000000,
                W_dt=_A16 + 0x2000000, delta=_A16 + 0x10000000)
    base.update(kw)
    return _lib.call_dt_proj(_lib.new_dt_proj_params(**base), 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(ntok=-1), _lib.ERR_INVALID_ARG),
    (dict(d_inner=0), _lib.ERR_INVALID_ARG),
    (dict(dt_rank=0), _lib.ERR_INVALID_ARG),
    (dict(dt_low_hi=None), _lib.ERR_INVALID_ARG),
    (dict(W_dt=None), _lib.ERR_INVALID_ARG),
    (dict(delta=None), _lib.ERR_INVALID_ARG),
    (dict(d_inner=8190), _lib.ERR_UNSUPPORTED),
    (dict(dt_rank=250), _lib.ERR_UNSUPPORTED),
    (dict(dt_rank=1 << 17), _lib.ERR_UNSUPPORTED),
    (dict(ntok=1 << 31), _lib.ERR_UNSUPPORTED),
    (dict(dt_low_hi=_A16 + 8), _lib.ERR_MISALIGNED),
    (dict(dt_low_lo=_A16 + 0x1000000 + 2), _lib.ERR_MISALIGNED),
    (dict(delta=_A16 + 0x10000000 + 4), _lib.ERR_MISALIGNED),
    (dict(delta=_A16 + 0x2000000), _lib.ERR_INVALID_ARG),  # overlaps W_dt
])
def test_dt_proj_argument_errors(P, kw, expect):
    assert _dt_proj_call(P, **kw) == expect


def test_dt_proj_struct_size_and_no_device(P):
    p = _lib.new_dt_proj_params(ntok=1, d_inner=8, dt_rank=8, dt_low_hi=_A16,
                                W_dt=_A16 + 0x1000, delta=_A16 + 0x2000)
    assert P.jamba_ssm_dt_proj(None, None) == _lib.ERR_INVALID_ARG
    p.struct_size = 8
    assert _lib.call_dt_proj(p, 0) == _lib.ERR_INVALID_ARG
    p.struct_size = ctypes.sizeof(_lib.DtProjParams)
    if not torch.cuda.is_available():
        assert _lib.call_dt_proj(p, 0) == _lib.ERR_NO_DEVICE


def test_dt_proj_empty_batch_needs_no_pointers(P):
    # an empty torch tensor's data_ptr() is 0: zero tokens must not check pointers
    assert _lib.call_dt_proj(_lib.new_dt_proj_params(ntok=0, d_inner=256, dt_rank=256), 0) == \
        _lib.OK
    assert _lib.call_dt_proj(_lib.new_dt_proj_params(ntok=0, d_inner=250, dt_rank=256), 0) == \
        _lib.ERR_UNSUPPORTED


def _x_proj_call(P, **kw):
    base = dict(ntok=4096, d_inner=8192, dt_rank=256, d_state=16, u=_A16,
                W_x=_A16 + 0x10000000, w_dt=_A16 + 0x11000000, w_B=_A16 + 0x11001000,
                w_C=_A16 + 0x11002000, eps=1e-6, dt_low_hi=_A16 + 0x20000000,
                dt_low_lo=_A16 + 0x21000000, B=_A16 + 0x22000000, C=_A16 + 0x22100000)
    base.update(kw)
    return _lib.call_x_proj(_lib.new_x_proj_params(**base), 0)


@pytest.mark.parametrize("kw,expect", [
    (dict(ntok=-1), _lib.ERR_INVALID_ARG),
    (dict(eps=-1.0), _lib.ERR_INVALID_ARG),
    (dict(eps=float("nan")), _lib.ERR_INVALID_ARG),
    (dict(k_split=3), _lib.ERR_INVALID_ARG),
    (dict(k_split=16), _lib.ERR_INVALID_ARG),
    (dict(u=None), _lib.ERR_INVALID_ARG),
    (dict(C=None), _lib.ERR_INVALID_ARG),
    (dict(dt_rank=128), _lib.ERR_UNSUPPORTED),
    (dict(d_state=8), _lib.ERR_UNSUPPORTED),
    (dict(d_inner=8191), _lib.ERR_UNSUPPORTED),
    (dict(u=_A16 + 8), _lib.ERR_MISALIGNED),
    (dict(B=_A16 + 0x22000000 + 2), _lib.ERR_MISALIGNED),
    (dict(w_dt=_A16 + 0x11000000 + 2), _lib.ERR_MISALIGNED),
    (dict(dt_low_lo=_A16 + 0x20000000), _lib.ERR_INVALID_ARG),  # overlaps dt_low_hi
    (dict(B=_A16 + 0x100), _lib.ERR_INVALID_ARG),                # overlaps u
])
def test_x_proj_argument_errors(P, kw, expect):
    assert _x_proj_call(P, **kw) == expect


def test_x_proj_empty_and_no_device(P):
    assert _lib.call_x_proj(_lib.new_x_proj_params(ntok=0, d_inner=8192, dt_rank=256,
                                                   d_state=16), 0) == _lib.OK
    if not torch.cuda.is_available():
        assert _x_proj_call(P, w_dt=None, w_B=None, w_C=None) == _lib.ERR_NO_DEVICE


def test_proj_abi_from_plain_c(P, tmp_path):
    """The projection library's boundary is C: a gcc-built program with no
    Python in it includes the header, links the library and gets the
    documented statuses back (host-side paths only; no GPU needed)."""
    exe = tmp_path / "proj_abi_check"
    libdir = os.path.dirname(_lib.PROJ_LIB_PATH)
    subprocess.run(["gcc", "-O1", "-Wall", "-Werror", "-o", str(exe),
                    os.path.join(ROOT, "tests", "c", "proj_abi_check.c"), "-I",
                    os.path.join(ROOT, "include"), "-L", libdir, "-ljamba_ssm_proj",
                    f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "passed" in r.stdout


# ---------------------------------------------------------------- ABI version 4
_CK = 0xB0000000  # fake, 16-byte aligned, clear of every buffer of _valid_scan


@pytest.mark.parametrize("kw,expect", [
    (dict(ckpt=_CK + 8), _lib.ERR_MISALIGNED),
    (dict(ckpt=_CK, cu_seqlens=0x3000, total_tokens=100), _lib.ERR_UNSUPPORTED),
    (dict(ckpt=_CK, state_indices=0x3000, num_slots=4), _lib.ERR_UNSUPPORTED),
    (dict(ckpt=_CK, d_state=4), _lib.ERR_UNSUPPORTED),      # bf16 d_state 4: no backward
    (dict(ckpt=_CK, kernel_variant=3), _lib.ERR_UNSUPPORTED),  # a variant without that kernel
    (dict(ckpt=0x90000000), _lib.ERR_INVALID_ARG),          # on top of out
    (dict(ckpt=0x10000000 - 0x100), _lib.ERR_INVALID_ARG),  # runs into x
])
def test_scan_checkpoint_argument_errors(L, kw, expect):
    assert _scan(_valid_scan(**kw)) == expect


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_scan_with_checkpoints_reaches_the_device_query(L):
    assert _scan(_valid_scan(ckpt=_CK)) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    # fp32 I/O also takes d_state 4
    assert _scan(_valid_scan(ckpt=_CK, io_dtype=_lib.F32, d_state=4)) in (
        _lib.ERR_NO_DEVICE, _lib.ERR_CUDA)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_version_3_struct_size_is_accepted(L):
    """A version-3 caller's struct ends before ckpt: whatever lies past it is
    ignored, for the scan and for the backward (and its no-allocation form)."""
    p = _valid_scan(ckpt=_CK + 8)  # misaligned if it were read
    p.struct_size = _lib.SCAN_PARAMS_V3_SIZE
    assert _scan(p) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    b = _valid_bwd(ckpt=_CK + 8)
    b.struct_size = _lib.SCAN_BWD_PARAMS_V3_SIZE
    assert _lib.call_scan_bwd(b, 0) in (_lib.ERR_NO_DEVICE, _lib.ERR_CUDA)
    b.struct_size = _lib.SCAN_BWD_PARAMS_V3_SIZE - 8
    assert _lib.call_scan_bwd(b, 0) == _lib.ERR_INVALID_ARG
    n = _valid_bwd(ckpt=_CK + 8, workspace=None, workspace_bytes=0)
    n.struct_size = _lib.SCAN_BWD_PARAMS_V3_SIZE
    assert L.jamba_ssm_scan_bwd_noalloc(ctypes.byref(n), None) in (_lib.ERR_NO_DEVICE,
                                                                     _lib.ERR_CUDA)


def _valid_bwd(**kw):
    base = dict(batch=1, seqlen=100, d_inner=256, d_state=16, io_dtype=_lib.BF16,
                delta_softplus=1, x=0x10000000, delta=0x11000000, z=0x12000000,
                B=0x13000000, C=0x14000000, A=0x15000000, dout=0x16000000, dx=0x17000000,
                ddelta=0x18000000, dz=0x19000000, dB=0x1A000000, dC=0x1B000000,
                workspace=0x40000000, workspace_bytes=1 << 26)
    base.update(kw)
    return _lib.new_scan_bwd_params(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(ckpt=_CK + 8), _lib.ERR_MISALIGNED),
    (dict(ckpt=0x17000000), _lib.ERR_INVALID_ARG),  # an output (dx) on top of it
])
def test_backward_checkpoint_argument_errors(L, kw, expect):
    assert _lib.call_scan_bwd(_valid_bwd(**kw), 0) == expect


def test_checkpoint_size(L):
    # ceil(100 / 16) = 7 checkpoints per sequence
    assert _lib.scan_ckpt_size(2, 100, 256, 16) == 2 * 7 * 256 * 16 * 4
    assert _lib.scan_ckpt_size(1, 0, 256, 16) == 0
    assert _lib.scan_ckpt_size(1, 16, 8, 8) == 8 * 8 * 4
    assert _lib.scan_ckpt_size(-1, 16, 8, 8) == 0



def _valid_ssd(**kw):
    base = dict(batch=2, seqlen=100, nheads=8, headdim=64, d_state=16, io_dtype=_lib.BF16,
                delta_softplus=1, x=0x10000000, delta=0x20000000, z=0x30000000,
                B=0x40000000, C=0x50000000, A=0x60000000, D=0x70000000,
                delta_bias=0x80000000, h0=None, out=0x90000000, h_final=0xA0000000)
    base.update(kw)
    return _lib.new_ssd_params(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(batch=-1), _lib.ERR_INVALID_ARG),
    (dict(seqlen=-5), _lib.ERR_INVALID_ARG),
    (dict(nheads=0), _lib.ERR_INVALID_ARG),
    (dict(headdim=0), _lib.ERR_INVALID_ARG),
    (dict(d_state=0), _lib.ERR_INVALID_ARG),
    (dict(io_dtype=7), _lib.ERR_INVALID_ARG),
    (dict(d_state=4), _lib.ERR_UNSUPPORTED),
    (dict(d_state=32), _lib.ERR_UNSUPPORTED),
    (dict(headdim=48), _lib.ERR_UNSUPPORTED),   # heads of whole 32-channel slices
    (dict(nheads=4), _lib.ERR_UNSUPPORTED),     # bf16 delta rows of 16-byte multiples
    (dict(batch=70000), _lib.ERR_UNSUPPORTED),  # grid y
    (dict(x=None), _lib.ERR_INVALID_ARG),
    (dict(delta=None), _lib.ERR_INVALID_ARG),
    (dict(A=None), _lib.ERR_INVALID_ARG),
    (dict(out=None), _lib.ERR_INVALID_ARG),
    (dict(x=0x10000002), _lib.ERR_MISALIGNED),
    (dict(B=0x40000008), _lib.ERR_MISALIGNED),
    (dict(h0=0xB0000004), _lib.ERR_MISALIGNED),
    (dict(A=0x60000002), _lib.ERR_MISALIGNED),
    (dict(out=0x10000000 + 64), _lib.ERR_INVALID_ARG),        # out overlaps x
    (dict(out=0x20000000), _lib.ERR_INVALID_ARG),             # out overlaps delta
    (dict(h_final=0x90000000 + 1024), _lib.ERR_INVALID_ARG),  # h_final inside out
    (dict(h0=0xA0000000 + 16), _lib.ERR_INVALID_ARG),         # h0 partially overlaps h_final
    (dict(workspace=0xC0000008, workspace_bytes=64), _lib.ERR_MISALIGNED),
    (dict(workspace=0xC0000000, workspace_bytes=8), _lib.ERR_WORKSPACE),
])
def test_ssd_argument_errors(L, kw, expect):
    """jamba_ssm_ssd_scan's checks, all taken before any device is touched."""
    assert _lib.call_ssd(_valid_ssd(**kw), 0) == expect


def test_ssd_struct_size_and_null(L):
    p = _valid_ssd()
    p.struct_size = 8
    assert _lib.call_ssd(p, 0) == _lib.ERR_INVALID_ARG
    assert L.jamba_ssm_ssd_scan(None, None) == _lib.ERR_INVALID_ARG
