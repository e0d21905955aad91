"""The boundary from plain C: the header compiles as C11 (and as C++), and a C
program linked against liblinattn.so gets the documented answers from the
host-side checks. No device is used."""
import os
import subprocess

import pytest

import __graft_entry__
from linear_attention_video_relu_b200 import _native as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INC = os.path.join(ROOT, "include")
LIBDIR = os.path.dirname(C.LIB_PATH)


@pytest.fixture(scope="module", autouse=True)
def built():
    __graft_entry__.build()


@pytest.mark.parametrize("lang,std", [("c", "-std=c11"), ("c++", "-std=c++17")])
def test_header_compiles_alone(lang, std, tmp_path):
    src = tmp_path / ("h." + ("c" if lang == "c" else "cpp"))
    src.write_text('#include "linattn.h"\nint main(void) { return 0; }\n')
    cc = "gcc" if lang == "c" else "g++"
    subprocess.check_call([cc, std, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INC,
                           "-c", str(src), "-o", str(tmp_path / "h.o")])


def test_c_program_gets_the_documented_answers(tmp_path):
    exe = tmp_path / "abi_consumer"
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", INC,
                           os.path.join(ROOT, "tests", "c", "abi_consumer.c"), "-L", LIBDIR,
                           "-llinattn", "-Wl,-rpath," + LIBDIR, "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60, check=True)
    got = dict(line.split(" ", 1) for line in out.stdout.strip().splitlines())
    assert got["workspace_size_bad_D"] == str(C.LA_ERR_INVALID_ARG)
    assert got["forward_empty"] == str(C.LA_OK)
    assert got["cross_no_keys"] == str(C.LA_ERR_INVALID_ARG)
    assert got["tconv_empty"] == str(C.LA_OK)
    assert got["tconv_bad_C"] == str(C.LA_ERR_INVALID_ARG)
    assert got["status_ok"] == C.status_string(C.LA_OK)
    assert got["status_limit"] == str(C.LA_WORKSPACE_CONTROL_BYTES)
