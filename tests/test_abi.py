"""The C ABI without a GPU: the library loads, exports every symbol include/attn.h
declares, and rejects bad arguments on the host before anything is launched."""
import ctypes
import os
import re

import pytest

import io_aware_exact_qk_b200 as attn
from io_aware_exact_qk_b200 import build as attn_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    attn_build.build()
    return attn.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(attn_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"attn_fwd", "attn_bwd", "attn_fwd_workspace_size", "attn_bwd_workspace_size",
            "attn_get_device_error", "attn_status_string", "attn_last_error_message", "attn_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(lib):
    assert lib.attn_status_string(0) == b"ok"
    assert lib.attn_status_string(4) == b"device pipeline wait timed out"
    assert attn.attn_version() == 100


def _fwd(lib, **kw):
    a = dict(q=16, k=16, v=16, cu=None, batch=1, seqlen=8, max_seqlen=8, total=8, hq=2, hkv=2, d=64,
             scale=0.125, causal=0, dtype=0, o=16, lse=16, ws=None, wsb=0, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.attn_fwd(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["cu"]), a["batch"], a["seqlen"],
                        a["max_seqlen"], a["total"], a["hq"], a["hkv"], a["d"], a["scale"], a["causal"],
                        a["dtype"], vp(a["o"]), vp(a["lse"]), vp(a["ws"]), a["wsb"], vp(a["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(d=48), attn.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), attn.ATTN_ERR_UNSUPPORTED),
    (dict(hq=3, hkv=2), attn.ATTN_ERR_UNSUPPORTED),
    (dict(hq=0), attn.ATTN_ERR_INVALID_ARG),
    (dict(dtype=7), attn.ATTN_ERR_UNSUPPORTED),
    (dict(total=9), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), attn.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), attn.ATTN_ERR_INVALID_ARG),
    (dict(q=None), attn.ATTN_ERR_INVALID_ARG),
    (dict(lse=None), attn.ATTN_ERR_INVALID_ARG),
    (dict(o=0x1008), attn.ATTN_ERR_INVALID_ARG),
    (dict(batch=-1, total=-8), attn.ATTN_ERR_INVALID_ARG),
    (dict(ws=None, wsb=0), attn.ATTN_ERR_INVALID_ARG),          # bf16 needs the 256-byte workspace
    (dict(ws=0x1008, wsb=256), attn.ATTN_ERR_INVALID_ARG),      # misaligned workspace
])
def test_fwd_rejects_bad_arguments_on_host(lib, kw, status):
    assert _fwd(lib, **kw) == status
    assert lib.attn_last_error_message() != b""


def test_empty_problem_is_a_no_op(lib):
    assert _fwd(lib, batch=0, seqlen=8, total=0, q=None, k=None, v=None, o=None, lse=None) == attn.ATTN_OK
    assert _fwd(lib, batch=3, seqlen=0, total=0, q=None, k=None, v=None, o=None, lse=None) == attn.ATTN_OK


def test_bwd_rejects_small_workspace(lib):
    vp = ctypes.c_void_p
    need = lib.attn_bwd_workspace_size(1, 8, 8, 2, 2, 64, 0)
    assert need == ((2 * 8 * 4 + 255) // 256) * 256 + 8 * 2 * 64 * 4 + 256   # D, dQ accumulator, item counter
    st = lib.attn_bwd(vp(16), vp(16), vp(16), vp(16), vp(16), vp(16), None, 1, 8, 8, 8, 2, 2, 64, 0.125, 0, 0,
                      vp(16), vp(16), vp(16), vp(16), need - 1, None)
    assert st == attn.ATTN_ERR_INVALID_ARG
    assert b"workspace" in lib.attn_last_error_message()


def test_workspace_sizes(lib):
    assert lib.attn_fwd_workspace_size(4, 2048, 8192, 16, 16, 128, 0) == 256   # the work-item counter
    assert lib.attn_fwd_workspace_size(4, 2048, 8192, 16, 16, 128, 1) == 0     # fp32 check mode
    assert lib.attn_fwd_workspace_size(0, 0, 0, 16, 16, 128, 0) == 0
    assert lib.attn_bwd_workspace_size(1, 0, 0, 4, 4, 64, 0) == 0
    assert lib.attn_bwd_workspace_size(2, 10, 20, 4, 2, 32, 1) == 4 * 20 * 4   # fp32 mode: D only


def _dec(lib, **kw):
    a = dict(q=16, k=16, v=16, cu_q=None, cu_k=None, batch=2, seqlen_q=1, seqlen_k=300, max_q=0, max_k=0,
             total_q=2, total_k=600, hq=8, hkv=2, d=128, scale=0.088, causal=0, splits=1, o=16, lse=16, ws=None,
             wsb=0, stream=None)
    a.update(kw)
    vp = ctypes.c_void_p
    return lib.attn_fwd_decode(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["cu_q"]), vp(a["cu_k"]), a["batch"],
                               a["seqlen_q"], a["seqlen_k"], a["max_q"], a["max_k"], a["total_q"], a["total_k"],
                               a["hq"], a["hkv"], a["d"], a["scale"], a["causal"], a["splits"], vp(a["o"]),
                               vp(a["lse"]), vp(a["ws"]), a["wsb"], vp(a["stream"]))


@pytest.mark.parametrize("kw,status", [
    (dict(d=48), attn.ATTN_ERR_UNSUPPORTED),
    (dict(hq=3, hkv=2), attn.ATTN_ERR_UNSUPPORTED),
    (dict(hq=64, hkv=1, seqlen_q=3, total_q=6), attn.ATTN_ERR_UNSUPPORTED),   # 64 heads x 3 rows > 128
    (dict(total_q=3), attn.ATTN_ERR_INVALID_ARG),
    (dict(total_k=599), attn.ATTN_ERR_INVALID_ARG),
    (dict(cu_q=0x1000), attn.ATTN_ERR_INVALID_ARG),                             # cu_k missing
    (dict(scale=0.0), attn.ATTN_ERR_INVALID_ARG),
    (dict(causal=3), attn.ATTN_ERR_INVALID_ARG),
    (dict(splits=-1), attn.ATTN_ERR_INVALID_ARG),
    (dict(q=None), attn.ATTN_ERR_INVALID_ARG),
    (dict(k=0x1004), attn.ATTN_ERR_INVALID_ARG),
    (dict(splits=3, ws=None, wsb=0), attn.ATTN_ERR_INVALID_ARG),                # needs a workspace
])
def test_decode_rejects_bad_arguments_on_host(lib, kw, status):
    assert _dec(lib, **kw) == status
    assert lib.attn_last_error_message() != b""


def test_decode_empty_problem_is_a_no_op(lib):
    assert _dec(lib, batch=0, total_q=0, total_k=0, q=None, k=None, v=None, o=None, lse=None) == attn.ATTN_OK


def test_decode_workspace_sizes(lib):
    # 1 sequence, 1 query row, 1024 keys = 8 key tiles in 4 splits of 2: partial O (fp32,
    # 256-byte aligned) + partial LSE
    assert lib.attn_fwd_decode_workspace_size(1, 1, 1024, 1, 1024, 8, 8, 128, 0, 4) == 4 * 8 * 128 * 4 + 4 * 8 * 4
    assert lib.attn_fwd_decode_workspace_size(1, 1, 1024, 1, 1024, 8, 8, 128, 0, 1) == 0
    # more splits than key tiles are clamped: 300 keys = 3 tiles
    assert lib.attn_fwd_decode_workspace_size(2, 1, 300, 2, 600, 8, 2, 64, 1, 16) == \
        ((3 * 2 * 8 * 64 * 4 + 255) // 256) * 256 + 3 * 8 * 2 * 4


def _fwd_fp8(lib, d=128, batch=1, seqlen=64, hq=2, hkv=2, ptr=0x1000, o=0x1000, ws=0x1000, wsb=256, causal=0):
    vp = ctypes.c_void_p
    return lib.attn_fwd_fp8(vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(ptr), batch, seqlen, hq, hkv, d,
                            ctypes.c_float(0.1), causal, vp(o), vp(ptr), vp(ws), wsb, None)


def test_fp8_calls_reject_bad_arguments_on_host(lib):
    assert _fwd_fp8(lib, d=32) == attn.ATTN_ERR_UNSUPPORTED            # e4m3 path is d = 64 or 128
    assert _fwd_fp8(lib, ptr=None) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8(lib, o=0x1008) == attn.ATTN_ERR_INVALID_ARG         # misaligned output
    assert _fwd_fp8(lib, wsb=0) == attn.ATTN_ERR_INVALID_ARG            # needs the 256-byte counter
    assert _fwd_fp8(lib, hq=3, hkv=2) == attn.ATTN_ERR_UNSUPPORTED
    assert _fwd_fp8(lib, causal=2) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8(lib, batch=0, ptr=None, o=None, ws=None, wsb=0) == attn.ATTN_OK   # empty: no-op
    vp = ctypes.c_void_p
    p = vp(0x1000)
    assert lib.attn_fp8_quantize(p, p, p, 1, 64, 2, 2, 32, p, p, p, p, p, p, None) == attn.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fp8_quantize(p, p, p, 1, 64, 2, 2, 128, p, None, p, p, p, p, None) == attn.ATTN_ERR_INVALID_ARG
    assert lib.attn_fp8_quantize(None, None, None, 0, 64, 2, 2, 128, None, None, None, None, None, None,
                                 None) == attn.ATTN_OK


def _fwd_fp8_varlen(lib, d=128, cu=0x2000, batch=2, max_seqlen=64, total=100, ptr=0x1000, o=0x1000, wsb=256):
    vp = ctypes.c_void_p
    return lib.attn_fwd_fp8_varlen(vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(ptr), vp(cu), batch, max_seqlen,
                                   total, 2, 2, d, ctypes.c_float(0.1), 1, vp(o), vp(ptr), vp(0x1000), wsb, None)


def test_fp8_varlen_calls_reject_bad_arguments_on_host(lib):
    assert _fwd_fp8_varlen(lib, cu=None) == attn.ATTN_ERR_INVALID_ARG              # the packed calls need it
    assert _fwd_fp8_varlen(lib, max_seqlen=101) == attn.ATTN_ERR_INVALID_ARG       # longer than all tokens
    assert _fwd_fp8_varlen(lib, total=-1) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(lib, d=32) == attn.ATTN_ERR_UNSUPPORTED
    assert _fwd_fp8_varlen(lib, o=0x1004) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(lib, wsb=8) == attn.ATTN_ERR_INVALID_ARG
    assert _fwd_fp8_varlen(lib, total=0, max_seqlen=0, ptr=None, o=None) == attn.ATTN_OK   # empty: no-op
    vp = ctypes.c_void_p
    p = vp(0x1000)
    q8v = lib.attn_fp8_quantize_varlen
    assert q8v(p, p, p, None, 2, 64, 100, 2, 2, 128, p, p, p, p, p, p, None) == attn.ATTN_ERR_INVALID_ARG
    assert q8v(p, p, p, vp(0x2000), 2, 64, 100, 2, 2, 64 + 32, p, p, p, p, p, p, None) == attn.ATTN_ERR_UNSUPPORTED
    assert q8v(p, p, p, vp(0x2000), 2, 64, 100, 2, 2, 128, p, p, None, p, p, p, None) == attn.ATTN_ERR_INVALID_ARG
    assert q8v(p, p, p, vp(0x2002), 2, 64, 100, 2, 2, 128, p, p, p, p, p, p, None) == attn.ATTN_ERR_INVALID_ARG
    assert q8v(None, None, None, vp(0x2000), 2, 0, 0, 2, 2, 128, None, None, None, None, None, None,
               None) == attn.ATTN_OK


def test_host_step_rejects_bad_arguments_on_host(lib):
    """attn_fwd_bwd_host checks its shapes, its host cu_seqlens and its scratch before it
    touches the GPU."""
    vp = ctypes.c_void_p
    p = vp(0x1000)

    def call(cu=None, batch=3, seqlen=100, max_seqlen=0, total=300, hq=4, hkv=2, d=128, ptr=p, scratch=p,
             scratch_bytes=1 << 40):
        return lib.attn_fwd_bwd_host(ptr, ptr, ptr, ptr, cu, batch, seqlen, max_seqlen, total, hq, hkv, d,
                                     ctypes.c_float(0.1), 1, ptr, ptr, ptr, ptr, ptr, scratch, scratch_bytes, None)

    assert call(hq=3) == attn.ATTN_ERR_UNSUPPORTED
    assert call(total=299) == attn.ATTN_ERR_INVALID_ARG                       # batch * seqlen mismatch
    assert call(ptr=None) == attn.ATTN_ERR_INVALID_ARG                        # NULL host arrays
    assert call(scratch_bytes=1000) == attn.ATTN_ERR_INVALID_ARG              # scratch too small
    assert b"scratch" in lib.attn_last_error_message()
    assert call(scratch=vp(0x1008)) == attn.ATTN_ERR_INVALID_ARG              # unaligned scratch
    cu_bad = [(0, 100, 50, 300), (0, 100, 200, 299), (1, 100, 200, 300), (0, 250, 260, 300)]
    for vals in cu_bad:                                # decreasing, wrong end, wrong start, > max
        arr = (ctypes.c_int32 * 4)(*vals)
        assert call(cu=ctypes.cast(arr, vp), seqlen=0, max_seqlen=200) == attn.ATTN_ERR_INVALID_ARG, vals
    assert call(batch=0, total=0, ptr=None, scratch=None, scratch_bytes=0) == attn.ATTN_OK   # empty: no-op
    need = lib.attn_fwd_bwd_host_scratch_size(3, 300, 4, 2, 128)
    assert need >= 300 * (4 * 4 + 4 * 2) * 128 * 2 + 300 * 4 * 4 * 128   # the tensors plus dQ's accumulator


def test_plain_c_client_compiles_links_and_runs(lib, tmp_path):
    """include/attn.h is a C header (C99, no C++), and a C program links libattn.so and
    gets the host-side answers (workspace sizes, validation statuses) without a GPU."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(attn.LIBRARY_PATH)
    exe = str(tmp_path / "c_abi_client")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi_client.c"), "-o", exe, "-L", libdir, "-lattn",
                        "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "unsupported configuration" in r.stdout and "invalid argument" in r.stdout
