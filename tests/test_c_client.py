"""include/gdr.h is a C ABI: a C99 program (and a C++ one) compiles against the header
with warnings as errors, links against the built libgdr.so, and gets exact statuses
from the host-side checks.  Nothing here calls a kernel, so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from linear_attention_recurrence_10_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.dirname(_abi.LIB_PATH)

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "gdr.h"

int main(void) {
    gdr_decode_args d;
    gdr_prefill_args p;
    gdr_norm_args n;
    size_t bytes = 123;
    int s;
    memset(&d, 0, sizeof d);
    memset(&p, 0, sizeof p);
    memset(&n, 0, sizeof n);
    printf("version %d\n", gdr_version());
    for (s = GDR_OK; s <= GDR_ERR_TIMEOUT; ++s) printf("status %d %s\n", s, gdr_status_string((gdr_status)s));
    /* all-zero arguments: every check fails before anything is queued */
    printf("decode %d\n", (int)gdr_decode_step(&d, NULL));
    printf("decode_null %d\n", (int)gdr_decode_step(NULL, NULL));
    printf("workspace %d\n", (int)gdr_prefill_workspace_size(&p, &bytes));
    printf("prefill_null %d\n", (int)gdr_prefill_chunked(NULL, NULL, 0, NULL));
    printf("norm_null %d\n", (int)gdr_rmsnorm_gated(NULL, NULL));
    return 0;
}
"""


def _build_and_run(tmp_path, compiler, std, suffix):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    if not os.path.exists(_abi.LIB_PATH):
        pytest.skip("libgdr.so is not built")
    src = tmp_path / f"client.{suffix}"
    src.write_text(PROGRAM)
    exe = tmp_path / f"client_{suffix}"
    cmd = [compiler, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE,
           str(src), "-L", LIBDIR, "-lgdr", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    return dict(line.split(" ", 1) for line in r.stdout.strip().splitlines()
                if not line.startswith("status")), r.stdout


@pytest.mark.parametrize("compiler,std,suffix", [("gcc", "c99", "c"), ("g++", "c++17", "cpp")])
def test_c_client(tmp_path, compiler, std, suffix):
    got, raw = _build_and_run(tmp_path, compiler, std, suffix)
    assert int(got["version"]) == _abi.lib().gdr_version()
    for code in range(7):
        assert f"status {code} GDR_" in raw
    invalid = str(1)  # GDR_ERR_INVALID_ARG
    for key in ("decode", "decode_null", "workspace", "prefill_null", "norm_null"):
        assert got[key] == invalid, (key, raw)
