"""The boundary is a C ABI: a plain C99 program (gcc -std=c99 -pedantic, no C++ and no torch)
includes include/gdn.h, links libgdn.so, queries a workspace size and has a bad call rejected
on the host.  No GPU is needed: validation precedes any device access."""
import os
import subprocess

from gated_deltanet_linear_eqs_b200 import _abi
from gated_deltanet_linear_eqs_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "gdn.h"
int main(void) {
    size_t n = 0;
    int rc = gdn_workspace_bytes(GDN_OP_PREFILL, 1, 4096, 16, 128, 128, 0, &n);
    printf("%s|%d|%lu|%s\n", gdn_version(), rc, (unsigned long)n,
           gdn_status_string(GDN_ERR_WORKSPACE));
    rc = gdn_decode_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 64, 64, GDN_BF16,
                         1.0f, 1, NULL);
    printf("%d\n", rc);
    return 0;
}
"""


def test_plain_c_program_uses_the_library(tmp_path):
    lib = build()
    src = tmp_path / "main.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "main"
    libdir = os.path.dirname(lib)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lgdn",
                           f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    version, rc, nbytes, status = out[0].split("|")
    assert version.startswith("gdn-b200") and int(rc) == _abi.GDN_OK
    assert int(nbytes) == 64 * 16 * (128 * 128 + 8192 + 128 * 256 + 1024 + 8192)
    assert status.startswith("GDN_ERR_WORKSPACE")
    assert int(out[1]) == _abi.GDN_ERR_INVALID_ARG
