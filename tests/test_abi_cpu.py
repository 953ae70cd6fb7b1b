"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/samba.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "samba.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(samba_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from sliding_window_attention_samba_b200 import _lib
    return _lib


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    h = lib.lib_handle()
    for n in names:
        assert hasattr(h, n), n


def test_status_strings_and_version(lib):
    assert lib.samba_status_string(0) == "SAMBA_OK"
    assert lib.samba_status_string(4) == "SAMBA_ERR_TIMEOUT"
    assert "sm_100a" in lib.samba_version()


def test_structs_match_header_layout(lib):
    # 10 ints + 2 floats + enum
    assert ctypes.sizeof(lib.BlockConfig) == 13 * 4
    assert ctypes.sizeof(lib.BlockWeights) == 23 * 8
    assert ctypes.sizeof(lib.DecodeState) == 5 * 8
    assert ctypes.sizeof(lib.BlockTaps) == 7 * 8


def test_workspace_sizes_host_only(lib):
    from sliding_window_attention_samba_b200 import inputs as I
    cfg = lib.make_config(I.WIDE)
    small = lib.samba_block_workspace_size(cfg, 1, 128)
    big = lib.samba_block_workspace_size(cfg, 4, 4096)
    assert 0 < small < big
    # tokens x (d_model*5 + 2 d_inner*... ) bytes: at least the in_proj output must fit
    assert big >= 4 * 4096 * 2 * I.WIDE.d_inner * 2
    bad = lib.make_config(I.WIDE)
    bad.d_state = 8
    assert lib.samba_block_workspace_size(bad, 1, 128) == 0
    assert lib.samba_selective_scan_workspace_size(1, 4096, 4096, 16) == 0
    assert lib.samba_swa_workspace_size(1, 4096, 32, 4, 64, 0.0, 1) == 0
    assert lib.samba_swa_workspace_size(1, 4096, 32, 4, 64, 10000.0, 1) >= 4096 * 36 * 64 * 2


def test_invalid_arguments_rejected_before_launch(lib):
    h = lib.lib_handle()
    # NULL inputs to the scan
    rc = h.samba_selective_scan(None, None, None, 1, None, None, None, None, None, None, None, None,
                                1, 16, 32, 16, 1, None, 0, None)
    assert rc == 1
    # unsupported state size (valid pointers are never dereferenced on this path)
    fake = ctypes.c_void_p(1 << 20)
    rc = h.samba_selective_scan(fake, fake, None, 1, fake, fake, fake, None, None, None, None, fake,
                                1, 16, 32, 8, 1, None, 0, None)
    assert rc == 2
    # GQA heads must divide
    rc = h.samba_swa_fwd(fake, fake, fake, fake, 1, 16, 6, 4, 64, 8, ctypes.c_float(0.0), 0,
                         ctypes.c_float(0.0), 1, None, 0, None)
    assert rc == 1
    # block: missing weights
    from sliding_window_attention_samba_b200 import inputs as I
    cfg = lib.make_config(I.TINY)
    w = lib.BlockWeights()
    with pytest.raises(lib.SambaError):
        lib.samba_block_fwd(cfg, w, 1 << 20, 2 << 20, None, None, 1, 8, 1 << 22, 1 << 30, 0)


def test_grid_limits_rejected_before_launch(lib):
    """Shapes beyond the launch grids (batch > 65535; more than 65535 conv runs of
    32 tokens in one call) come back as SAMBA_ERR_UNSUPPORTED from host-side
    validation, before any CUDA call (none can run on this machine)."""
    from sliding_window_attention_samba_b200 import inputs as I
    h = lib.lib_handle()
    fake = ctypes.c_void_p(1 << 20)
    big_b = 65536
    rc = h.samba_selective_scan(fake, fake, None, 1, fake, fake, fake, None, None, None, None, fake,
                                big_b, 16, 32, 16, 1, None, 0, None)
    assert rc == lib.SAMBA_ERR_UNSUPPORTED
    rc = h.samba_swa_fwd(fake, fake, fake, fake, big_b, 16, 4, 4, 64, 8, ctypes.c_float(0.0), 0,
                         ctypes.c_float(0.0), 1, None, 0, None)
    assert rc == lib.SAMBA_ERR_UNSUPPORTED
    # with RoPE on, the grid check still comes before the table and rotation launches
    # (a CUDA call here would return SAMBA_ERR_CUDA instead)
    rc = h.samba_swa_fwd(fake, fake, fake, fake, big_b, 1, 1, 1, 16, 8, ctypes.c_float(10000.0), 0,
                         ctypes.c_float(0.0), 1, fake, ctypes.c_size_t(1 << 40), None)
    assert rc == lib.SAMBA_ERR_UNSUPPORTED
    rc = h.samba_swa_fwd_noalloc(fake, fake, fake, fake, big_b, 1, 1, 1, 16, 8, ctypes.c_float(10000.0), 0,
                                 ctypes.c_float(0.0), 1, None)
    assert rc == lib.SAMBA_ERR_UNSUPPORTED
    rc = h.samba_swa_fwd_noalloc(fake, fake, fake, fake, 1, 1, big_b, 1, 16, 8, ctypes.c_float(0.0), 0,
                                 ctypes.c_float(0.0), 1, None)
    assert rc == lib.SAMBA_ERR_UNSUPPORTED
    cfg = lib.make_config(I.TINY)
    w = lib.BlockWeights()
    for i in range(4):
        w.norm_g[i] = 1 << 20
    for name, _ in lib.BlockWeights._fields_[1:]:
        setattr(w, name, 1 << 20)
    st = lib.make_state(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20)
    with pytest.raises(lib.SambaError) as e:
        lib.samba_step(cfg, w, 1 << 20, 2 << 20, st, big_b, 1 << 22, 1 << 40, 0)
    assert e.value.code == lib.SAMBA_ERR_UNSUPPORTED
    with pytest.raises(lib.SambaError) as e:
        lib.samba_block_fwd(cfg, w, 1 << 20, 2 << 20, None, None, 1, 65535 * 32 + 1, 1 << 22, 1 << 40, 0)
    assert e.value.code == lib.SAMBA_ERR_UNSUPPORTED
    # the largest accepted batch still gets as far as the workspace check
    with pytest.raises(lib.SambaError) as e:
        lib.samba_step(cfg, w, 1 << 20, 2 << 20, st, 65535, 1 << 22, 16, 0)
    assert e.value.code == lib.SAMBA_ERR_INVALID_ARG


def test_plain_c_consumer_builds_and_runs(tmp_path, lib):
    """The header is valid C99 (no C++ or torch types cross the boundary): a C
    program compiled with -std=c99 -Wall -Werror links libsamba.so and runs its
    host-side calls."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(lib.LIB_PATH)
    exe = str(tmp_path / "consumer")
    src = os.path.join(ROOT, "tests", "abi_c", "consumer.c")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                        "-L", libdir, "-lsamba", "-Wl,-rpath," + libdir, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("consumer ok")
    # the same header and program as C++ (extern "C" linkage)
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is not None:
        exe2 = str(tmp_path / "consumer_cxx")
        r = subprocess.run([cxx, "-x", "c++", "-std=c++17", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                            src, "-L", libdir, "-lsamba", "-Wl,-rpath," + libdir, "-o", exe2],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        assert subprocess.run([exe2], capture_output=True, text=True, timeout=60).returncode == 0


def test_gemm_timing_hook_host_side(lib):
    """The measurement hook validates its arguments and counts nothing until a
    projection launches (no device call happens in install/remove)."""
    h = lib.lib_handle()
    V = ctypes.c_void_p
    a = (V * 2)(1 << 20, 1 << 21)
    b = (V * 2)(1 << 22, 1 << 23)
    assert h.samba_set_gemm_timing(-1, None, None, 0) == 0
    assert h.samba_set_gemm_timing(2, None, None, 1) == lib.SAMBA_ERR_INVALID_ARG
    assert h.samba_set_gemm_timing(5, a, b, 2) == lib.SAMBA_ERR_INVALID_ARG
    assert h.samba_set_gemm_timing(2, a, b, 0) == lib.SAMBA_ERR_INVALID_ARG
    assert h.samba_set_gemm_timing(2, (V * 2)(1 << 20, None), b, 2) == lib.SAMBA_ERR_INVALID_ARG
    assert h.samba_set_gemm_timing(2, a, b, 2) == 0
    assert h.samba_gemm_timing_count() == 0
    assert h.samba_set_gemm_timing(-1, None, None, 0) == 0


def test_scan_stall_hook_arguments(lib):
    """The failure-detection hook validates its arguments on the host; setting and
    clearing it makes no device call."""
    h = lib.lib_handle()
    assert h.samba_debug_scan_stall(-2, 0) == lib.SAMBA_ERR_INVALID_ARG
    assert h.samba_debug_scan_stall(3, 10) == lib.SAMBA_ERR_INVALID_ARG          # below 1 ms
    assert h.samba_debug_scan_stall(3, 3_000_000_000) == lib.SAMBA_ERR_INVALID_ARG  # above 2 s
    assert h.samba_debug_scan_stall(3, 5_000_000) == 0
    assert h.samba_debug_scan_stall(-1, 0) == 0


def test_debug_check_build_exports_and_flags(lib):
    """libsamba_debug.so (built by __graft_entry__.build) exports the same
    symbols; only it reports the checks enabled, and the release library refuses
    the self-test before touching the device."""
    assert lib.samba_debug_checks_enabled() == 0
    assert lib.samba_debug_check_selftest(0, None, 0, 0) == lib.SAMBA_ERR_UNSUPPORTED
    assert lib.samba_debug_check_selftest(7, None, 0, 0) == lib.SAMBA_ERR_INVALID_ARG
    assert lib.samba_last_check_site() == ""
    assert lib.samba_status_string(lib.SAMBA_ERR_BOUNDS) == "SAMBA_ERR_BOUNDS"
    path = os.path.join(ROOT, "sliding_window_attention_samba_b200", "libsamba_debug.so")
    if not os.path.exists(path):
        pytest.skip("libsamba_debug.so not built")
    dbg = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(dbg, n), n
    dbg.samba_debug_checks_enabled.restype = ctypes.c_int
    assert dbg.samba_debug_checks_enabled() == 1
    # the guard bands are part of the workspace the size queries report
    dbg.samba_debug_selftest_workspace_size.restype = ctypes.c_size_t
    rel = ctypes.CDLL(lib.LIB_PATH)
    rel.samba_debug_selftest_workspace_size.restype = ctypes.c_size_t
    assert dbg.samba_debug_selftest_workspace_size() == rel.samba_debug_selftest_workspace_size() + 2 * 4096
