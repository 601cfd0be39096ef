"""The C-ABI library loads and exports every symbol include/moe_lowbit.h
declares; host-side validation works without a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_lowbit.h")


@pytest.fixture(scope="module")
def lib():
    from bit_quantized_moe_route_b200 import build
    build.build()
    from bit_quantized_moe_route_b200 import _lib
    return _lib.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(moe_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
                 "moe_workspace_size", "moe_read_device_error", "moe_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # also via the dynamic symbol table
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", os.path.join(ROOT, "bit_quantized_moe_route_b200",
                                                                       "libmoe_lowbit.so")],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(moe_\w+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


def test_status_strings(lib):
    from bit_quantized_moe_route_b200 import _lib
    for code in range(7):
        assert _lib.status_string(code) not in ("", "unknown status")
    assert _lib.status_string(99) == "unknown status"


def test_workspace_size_and_dims_validation(lib):
    from bit_quantized_moe_route_b200 import _lib
    d = _lib.make_dims(1, 4096, 2048, 256, 8, d_ff_shared=2048)
    n = lib.moe_workspace_size(ctypes.byref(d))
    assert n > 0 and n % 256 == 0
    big = _lib.make_dims(4096, 4096, 2048, 256, 8)
    assert lib.moe_workspace_size(ctypes.byref(big)) > n
    for bad in (_lib.make_dims(0, 4096, 2048, 256, 8), _lib.make_dims(1, 4010, 2048, 256, 8), _lib.make_dims(1, 16384, 2048, 256, 8),
                _lib.make_dims(1, 4096, 2048, 256, 300), _lib.make_dims(1, 4096, 2048, 2000, 8),
                _lib.make_dims(1, 4096, 2048, 8, 9), _lib.make_dims(1, 4096, 2048, 256, 8, hash_mode=1, vocab=0)):
        assert lib.moe_workspace_size(ctypes.byref(bad)) == 0


def test_host_validation_without_gpu(lib):
    from bit_quantized_moe_route_b200 import _lib
    d = _lib.make_dims(4, 256, 128, 8, 2)
    # NULL dims
    assert lib.moe_forward(None, None, None, None, None, None, None, None, None, None, None, None, None,
                           None, 0, None) == 1
    # NULL workspace
    st = lib.moe_route(ctypes.byref(d), None, None, None, None, None, None, None, None, 0, None)
    assert st == 1 and b"workspace" in lib.moe_last_error_detail()
    # expert slice outside [0, n_experts], include_shared not 0/1
    assert lib.moe_forward_partial(ctypes.byref(d), 3, 9, 1, *([None] * 13), 0, None) == 1
    assert b"expert range" in lib.moe_last_error_detail()
    assert lib.moe_forward_partial(ctypes.byref(d), 0, 8, 2, *([None] * 13), 0, None) == 1
    assert b"include_shared" in lib.moe_last_error_detail()
    # mxfp8 rows: n_in not a multiple of 32, negative rows
    assert lib.moe_dequant_mxfp8(None, None, 4, 48, None, None) == 1
    assert lib.moe_dequant_mxfp8(None, None, -1, 64, None, None) == 1
    assert lib.moe_dequant_mxfp8(None, None, 0, 64, None, None) == 0
    # bad dims
    bad = _lib.make_dims(4, 256, 128, 8, 0)
    assert lib.moe_permute(ctypes.byref(bad), None, None, None, None, None, 0, None) == 1
    assert b"top_k" in lib.moe_last_error_detail()
    # workspace too small is reported before any device access
    fake = ctypes.c_void_p(0x10000)
    assert lib.moe_route(ctypes.byref(d), None, None, None, None, None, None, None, fake, 16, None) == 3


def test_binding_fails_loudly_without_library(tmp_path):
    from bit_quantized_moe_route_b200 import _lib
    with pytest.raises(ImportError):
        _lib.load_library(str(tmp_path / "missing.so"))


def test_binding_rejects_unknown_pack_format():
    import types
    from bit_quantized_moe_route_b200 import _lib
    m = types.SimpleNamespace(fmt="mxfp8", bits=8, group=32, q=None, scales=None, biases=None)
    with pytest.raises(ValueError):
        _lib.qmat(m)


def test_plain_c_caller(lib, tmp_path):
    """The header compiles as strict C99 and a C program links and calls the library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.join(ROOT, "bit_quantized_moe_route_b200")
    exe = str(tmp_path / "abi_from_c")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi_from_c.c"), "-L", libdir, "-lmoe_lowbit",
                    f"-Wl,-rpath,{libdir}", "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("ok ")


def test_ffn_path_setting_is_per_thread(lib):
    """moe_set_ffn_path changes only the calling thread's setting."""
    import threading
    from bit_quantized_moe_route_b200 import _lib
    main_prev = _lib.set_ffn_path(_lib.FFN_TENSOR_CORE)
    seen = {}

    def other():
        seen["initial"] = _lib.set_ffn_path(_lib.FFN_GEMV)   # returns this thread's previous value
        seen["after"] = _lib.set_ffn_path(_lib.FFN_GEMV)

    th = threading.Thread(target=other)
    th.start()
    th.join()
    assert seen == {"initial": _lib.FFN_AUTO, "after": _lib.FFN_GEMV}
    assert _lib.set_ffn_path(main_prev) == _lib.FFN_TENSOR_CORE    # the other thread did not change it
