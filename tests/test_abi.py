"""The C-ABI library builds for sm_100a, loads without a GPU and exports every entry
point that include/ict.h declares (no compute calls here)."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ict.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ict_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("ict_linear_fwd", "ict_linear_bwd_data", "ict_linear_bwd_weight",
                     "ict_conv_implicit_gemm", "ict_requant", "ict_sgd_momentum_step"):
        assert required in names


def test_library_exports_every_declared_symbol():
    from integer_only_nn_02_b200.csrc.build import build

    path = build()
    lib = ctypes.CDLL(path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    lib.ict_status_string.restype = ctypes.c_char_p
    assert lib.ict_status_string(0) == b"ICT_OK"
    assert lib.ict_status_string(7) == b"ICT_ERR_DEVICE_TIMEOUT"


def test_binding_names_match_header():
    from integer_only_nn_02_b200 import ict

    assert sorted(ict.EXPORTED) == declared_functions()
    for name in ict.EXPORTED:
        assert callable(getattr(ict, name))


def test_library_shares_nothing_with_oracle():
    """The oracle and the CUDA path share no source: no include of one by the other."""
    csrc = os.path.join(ROOT, "integer_only_nn_02_b200", "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f)).read()
        assert "oracle" not in text.lower() or f == "build.py" and "oracle" not in text
    oracle_src = open(os.path.join(ROOT, "oracle", "ict_oracle.c")).read()
    assert "#include \"" not in oracle_src


def test_header_is_plain_c():
    """The boundary is a C ABI: the header compiles as C99 and as C++ without warnings,
    names no torch or CUDA type, and every entry point takes plain pointers and sizes."""
    import shutil
    import subprocess

    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for banned in ("torch", "at::", "cudaStream_t", "std::", "Tensor"):
        assert banned not in text, banned
    for compiler, lang, std in (("gcc", "c", "-std=c99"), ("g++", "c++", "-std=c++11")):
        if shutil.which(compiler) is None:
            continue
        r = subprocess.run([compiler, "-fsyntax-only", "-Wall", "-Wextra", "-Werror", "-x", lang, std, HEADER],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_c_program_links_and_gets_errors_without_a_gpu(tmp_path):
    """A plain C program includes ict.h, links libict.so and calls it.  The build host has
    no GPU: the version and status strings work, and a Product call returns an error
    code (no crash, no CPU fallback)."""
    import shutil
    import subprocess

    import pytest
    import torch

    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    if torch.cuda.is_available():  # the call below passes host buffers: never on a GPU host
        pytest.skip("meant for a host without a GPU")
    from integer_only_nn_02_b200.csrc.build import build

    lib = build()
    src = tmp_path / "use_ict.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "ict.h"
int main(void) {
    int8_t m[64 * 64], e[64];
    ict_tensor X = {m, e, 64, 64, 64, 1, 64}, W = X, Y = X;
    int32_t st = ict_linear_fwd(&X, &W, &Y, NULL, 0, NULL);
    printf("%s|%s|%d\n", ict_version(), ict_status_string(st), st != ICT_OK);
    return 0;
}
""")
    exe = tmp_path / "use_ict"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        lib, "-o", str(exe), f"-Wl,-rpath,{os.path.dirname(lib)}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    version, status, failed = out.stdout.strip().split("|")
    assert version.startswith("libict") and status.startswith("ICT_ERR") and failed == "1"
