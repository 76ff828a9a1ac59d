"""The C ABI without a GPU: the library loads, exports every entry point that
include/wkv.h declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

from wkv_recurrence_b200 import _abi
from wkv_recurrence_b200 import build as wbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wkv.h")


@pytest.fixture(scope="module")
def L():
    wbuild.build()
    return _abi.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"WKV_API\s+[\w\s\*]+?\b(wkv_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_binding_structs_match_the_header(tmp_path):
    """The ctypes structs of the binding have the header's fields, sizes and
    offsets (compiled against include/wkv.h with the host C compiler)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    structs = {"wkv_options": _abi.wkv_options, "wkv_cstate": _abi.wkv_cstate, "wkv_state": _abi.wkv_state,
               "wkv_ext": _abi.wkv_ext}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "wkv.h"', "int main(void) {"]
    for name, ct in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in ct._fields_:
            lines.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    want = []
    for name, ct in structs.items():
        want.append(f"{name} size {ctypes.sizeof(ct)}")
        for field, _ in ct._fields_:
            want.append(f"{name} {field} {getattr(ct, field).offset}")
    assert [g for g in got if g] == want
    # and the header has no field the binding lacks
    text = open(HEADER).read()
    body = re.search(r"typedef struct \{([^}]*)\} wkv_options;", text).group(1)
    header_fields = re.findall(r"\b(\w+);", body)
    assert header_fields == [f for f, _ in _abi.wkv_options._fields_]


def test_status_strings(L):
    for code in range(8):
        s = _abi.status_string(code)
        assert s and s != "unknown status"
    assert _abi.status_string(99) == "unknown status"
    assert L.wkv_version() >= 100
    assert L.wkv_last_cuda_error().decode().startswith("cuda")


def test_forward_host_sizes_and_argument_checks(L):
    F32, BF16 = _abi.WKV_F32, _abi.WKV_BF16
    # two segments of k, v and out, the carried state, the forward's workspace
    a = L.wkv_forward_host_buffer_size(1, 65536, 2048, F32, F32, 4096)
    assert a >= 2 * 3 * 4096 * 2048 * 4 + 3 * 2048 * 4 + L.wkv_forward_workspace_size(1, 4096, 2048, None)
    assert L.wkv_forward_host_buffer_size(1, 65536, 2048, F32, F32, 0) == a  # default: 64 MB of k and v
    assert L.wkv_forward_host_buffer_size(1, 65536, 2048, BF16, BF16, 4096) < a
    assert L.wkv_forward_host_buffer_size(1, 100, 64, 7, F32, 0) == 0
    assert L.wkv_forward_host_buffer_size(-1, 100, 64, F32, F32, 0) == 0
    # argument errors come back before anything is queued (no device needed)
    assert L.wkv_forward_host(1, 10, 64, None, None, F32, None, None, None, F32, None, None, None, 0, 0,
                              None) == _abi.WKV_ERR_INVALID_ARG
    assert L.wkv_forward_host(1, 10, 64, None, None, 9, None, None, None, F32, None, None, None, 0, 0,
                              None) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert L.wkv_forward_host(1, 10, 64, None, None, F32, None, None, None, BF16, None, None, None, 0, 0,
                              None) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert L.wkv_forward_host(1, 10, 64, None, None, F32, None, None, None, F32, None, None, None, 0, -5,
                              None) == _abi.WKV_ERR_INVALID_ARG


def test_workspace_size(L):
    # sequential kernel: the 256-byte header only
    assert L.wkv_forward_workspace_size(16, 4096, 4096, None) == 256
    # three-launch scan: header + chunk totals + incoming states; grows with T
    o3 = _abi.wkv_options(kernel=3)
    a = L.wkv_forward_workspace_size(8, 1024, 768, ctypes.byref(o3))
    b = L.wkv_forward_workspace_size(8, 2048, 768, ctypes.byref(o3))
    assert 256 < a < b
    # cluster scan: a flag and a prefix per segment after the first and channel
    # group, and room for the single-launch scan that misaligned inputs take
    o5, o3, o2 = (_abi.wkv_options(kernel=k) for k in (5, 3, 2))
    for T in (2048, 4096, 4097, 16384):
        auto = o3 if 8 * T * 768 <= 1 << 24 else o5  # the automatic choice
        assert L.wkv_forward_workspace_size(8, T, 768, None) == L.wkv_forward_workspace_size(8, T, 768, ctypes.byref(auto))
        for o in (o5, o3):
            assert L.wkv_forward_workspace_size(8, T, 768, ctypes.byref(o)) >= \
                L.wkv_forward_workspace_size(8, T, 768, ctypes.byref(o2))
    assert L.wkv_forward_workspace_size(-1, 4, 4, None) == 0
    o = _abi.wkv_options(kernel=2, chunk_len=48)
    assert L.wkv_forward_workspace_size(1, 64, 64, ctypes.byref(o)) == 0
    o = _abi.wkv_options(kernel=2, chunk_len=32, lookback_group=4)
    assert L.wkv_forward_workspace_size(1, 64, 64, ctypes.byref(o)) > 256


def test_forward_kernel_choice(L):
    F32, BF16 = _abi.WKV_F32, _abi.WKV_BF16
    # many channels or short sequences: the sequential kernel; otherwise the
    # three-launch scan
    assert L.wkv_forward_kernel(16, 4096, 4096, BF16, None) == 1
    assert L.wkv_forward_kernel(8, 64, 64, F32, None) == 1
    assert L.wkv_forward_kernel(8, 1024, 768, F32, None) == 3
    assert L.wkv_forward_kernel(8, 2049, 768, F32, None) == 3
    # few channels and k, v larger than L2 (more than 2^24 elements each): the
    # cluster scan
    assert L.wkv_forward_kernel(1, 8192, 2048, F32, None) == 3
    assert L.wkv_forward_kernel(1, 8193, 2048, F32, None) == 5
    assert L.wkv_forward_kernel(8, 2049, 1024, BF16, None) == 5
    assert L.wkv_forward_kernel(1, 65536, 2048, F32, None) == 5
    assert L.wkv_forward_kernel(1, 65536, 2049, F32, None) == 2  # rows TMA cannot address
    # an explicit choice stands, except that the TMA scans fall back to the
    # single-launch scan when a row pitch is not a multiple of 16 bytes
    for kernel in (1, 2, 3, 4, 5):
        o = _abi.wkv_options(kernel=kernel)
        assert L.wkv_forward_kernel(2, 500, 64, F32, ctypes.byref(o)) == kernel
        assert L.wkv_forward_kernel(2, 500, 65, F32, ctypes.byref(o)) == (2 if kernel in (3, 4, 5) else kernel)
    for bad in (dict(cta_warps=3), dict(cta_warps=16), dict(cta_warps=32), dict(span=8), dict(span=16)):
        o = _abi.wkv_options(kernel=5, **bad)
        assert L.wkv_forward_kernel(2, 100, 64, F32, ctypes.byref(o)) == 0
    assert L.wkv_forward_launches(8, 1024, 768, F32, ctypes.byref(_abi.wkv_options(kernel=5))) == 1
    assert L.wkv_forward_launches(1, 65536, 2048, F32, None) == 1
    assert L.wkv_forward_launches(1, 8192, 2048, F32, None) == 3
    assert L.wkv_forward_launches(2, 20, 64, F32, ctypes.byref(_abi.wkv_options(kernel=3))) == 2
    assert L.wkv_forward_launches(16, 4096, 4096, BF16, None) == 1
    assert L.wkv_forward_kernel(-1, 4, 4, F32, None) == 0
    assert L.wkv_forward_kernel(1, 4, 4, 9, None) == 0
    o = _abi.wkv_options(kernel=4, stages=1)
    assert L.wkv_forward_kernel(1, 4, 4, F32, ctypes.byref(o)) == 0


FAKE = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails its checks first


def fwd(L, B=1, T=4, C=8, k=FAKE, v=FAKE, kvd=0, w=FAKE, u=FAKE, out=FAKE, od=0, sin=None, sout=None,
        ws=ctypes.c_void_p(0x100000), wsb=1 << 20, opts=None):
    return L.wkv_forward(B, T, C, k, v, kvd, w, u, out, od, sin, sout, ws, wsb, None, opts)


def test_forward_rejects_bad_arguments(L):
    assert fwd(L, B=-1) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, T=-3) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, T=1 << 24) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, kvd=7) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert fwd(L, kvd=_abi.WKV_F32, od=_abi.WKV_BF16) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert fwd(L, k=None) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, out=None) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, w=None) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, ws=None) == _abi.WKV_ERR_INVALID_ARG
    assert fwd(L, ws=ctypes.c_void_p(0x100010)) == _abi.WKV_ERR_MISALIGNED
    assert fwd(L, T=4096, C=8, wsb=16) == _abi.WKV_ERR_WORKSPACE_TOO_SMALL
    bad_state = _abi.wkv_cstate(0x1000, None, 0x1000)
    assert fwd(L, sin=ctypes.byref(bad_state)) == _abi.WKV_ERR_INVALID_ARG
    bad_out = _abi.wkv_state(0x1000, 0x1000, None)
    assert fwd(L, sout=ctypes.byref(bad_out)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(kernel=6)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(kernel=5, cta_warps=16)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    # per-token decays with a look-back kernel, or without w_t and without w
    ext = _abi.wkv_ext(0x2000, None)
    for kernel in (2, 4):
        o = _abi.wkv_options(kernel=kernel)
        assert L.wkv_forward_ext(1, 4, 8, FAKE, FAKE, 0, FAKE, FAKE, FAKE, 0, None, None, ctypes.c_void_p(0x100000),
                                 1 << 20, None, ctypes.byref(o), ctypes.byref(ext)) == _abi.WKV_ERR_INVALID_ARG
    assert L.wkv_forward_ext(1, 4, 8, FAKE, FAKE, 0, None, FAKE, FAKE, 0, None, None, ctypes.c_void_p(0x100000),
                             1 << 20, None, None, None) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(kernel=4, chunk_len=128, span=8)  # 16 warps per role: too many
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    for bad_stages in (1, 9, -1):
        o = _abi.wkv_options(kernel=4, stages=bad_stages)
        assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(kernel=2, chunk_len=100)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(wait_timeout_ns=-5)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(inject_enable=2)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(kernel=2, span=12)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    o = _abi.wkv_options(kernel=1, seq_threads=48)
    assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG
    for bad in (dict(seq_vec=3), dict(seq_vec=-1), dict(kernel=3, replay_chunks=3), dict(kernel=3, replay_chunks=-1), dict(kernel=3, scan_segments=8), dict(kernel=3, scan_segments=32),
                dict(kernel=3, scan_segments=-1)):
        o = _abi.wkv_options(**{"kernel": 1, **bad})
        assert fwd(L, opts=ctypes.byref(o)) == _abi.WKV_ERR_INVALID_ARG


def test_step_rejects_bad_arguments(L):
    s = _abi.wkv_cstate(0x1000, 0x1000, 0x1000)
    so = _abi.wkv_state(0x1000, 0x1000, 0x1000)
    P = ctypes.byref
    assert L.wkv_step(-1, 4, FAKE, FAKE, 0, FAKE, FAKE, FAKE, 0, P(s), P(so), None) == _abi.WKV_ERR_INVALID_ARG
    assert L.wkv_step(2, 4, FAKE, FAKE, 0, FAKE, FAKE, FAKE, 0, None, P(so), None) == _abi.WKV_ERR_INVALID_ARG
    assert L.wkv_step(2, 4, FAKE, FAKE, 0, FAKE, FAKE, FAKE, 0, P(s), None, None) == _abi.WKV_ERR_INVALID_ARG
    assert L.wkv_step(2, 4, FAKE, FAKE, 3, FAKE, FAKE, FAKE, 0, P(s), P(so), None) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert L.wkv_step(2, 4, FAKE, FAKE, 0, FAKE, FAKE, FAKE, 1, P(s), P(so), None) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert L.wkv_step(2, 4, None, FAKE, 0, FAKE, FAKE, FAKE, 0, P(s), P(so), None) == _abi.WKV_ERR_INVALID_ARG
    # nothing to do: no device needed
    assert L.wkv_step(0, 4, None, None, 0, None, None, None, 0, P(s), P(so), None) == _abi.WKV_OK


def test_zero_sized_forward_needs_no_device(L):
    assert fwd(L, B=0, k=None, v=None, out=None) == _abi.WKV_OK
    assert fwd(L, C=0, k=None, v=None, out=None, w=None, u=None) == _abi.WKV_OK


def test_binding_fails_loudly_without_cuda_tensors():
    import torch
    import wkv_recurrence_b200 as W
    x = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        W.forward(x, x, torch.zeros(8), torch.zeros(8))


def test_noalloc_rejects_bad_arguments_before_any_device_work(L):
    """wkv_forward_noalloc runs every argument check of wkv_forward before it
    looks up its scratch array or queues anything (no device exists here, so
    reaching the device would return WKV_ERR_CUDA instead)."""
    def na(B=1, T=4, C=8, k=FAKE, v=FAKE, kvd=0, w=FAKE, u=FAKE, out=FAKE, od=0, sin=None, sout=None):
        return L.wkv_forward_noalloc(B, T, C, k, v, kvd, w, u, out, od, sin, sout, None)
    assert na(kvd=7) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert na(kvd=_abi.WKV_F32, od=_abi.WKV_BF16) == _abi.WKV_ERR_UNSUPPORTED_DTYPE
    assert na(k=None) == _abi.WKV_ERR_INVALID_ARG
    assert na(out=None) == _abi.WKV_ERR_INVALID_ARG
    assert na(u=None) == _abi.WKV_ERR_INVALID_ARG
    assert na(sin=ctypes.byref(_abi.wkv_cstate(0x1000, None, 0x1000))) == _abi.WKV_ERR_INVALID_ARG
    assert na(sout=ctypes.byref(_abi.wkv_state(0x1000, 0x1000, None))) == _abi.WKV_ERR_INVALID_ARG
    # sizes out of range are refused before any plan is made from them
    assert na(B=-1) == _abi.WKV_ERR_INVALID_ARG
    assert na(T=1 << 24) == _abi.WKV_ERR_INVALID_ARG
    assert na(B=1 << 40, C=1 << 40) == _abi.WKV_ERR_INVALID_ARG
    assert L.wkv_forward_workspace_size(1 << 40, 4, 1 << 40, None) == 0
    assert na(B=0, k=None, v=None, out=None) == _abi.WKV_OK
