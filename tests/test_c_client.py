"""The C ABI as a C program sees it (no GPU): ``include/avq.h`` compiles as
plain C11 and as C++, and a C client linked against the library calls the
host-only entry points and gets argument errors back before any CUDA call."""
import os
import shutil
import subprocess

import pytest

from adaptive_vector_quantized_avq_b200 import build as bl

HEADER_DIR = os.path.join(bl.ROOT, "include")

CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "avq.h"

int main(void) {
    if (avq_version() < 100) return 10;
    if (strcmp(avq_status_string(AVQ_OK), "AVQ_OK") != 0) return 11;
    int32_t order[6 * 5];
    if (avq_gilbert_order(6, 5, order) != AVQ_OK) return 12;
    int seen[30] = {0};
    for (int i = 0; i < 30; ++i) {
        if (order[i] < 0 || order[i] >= 30 || seen[order[i]]++) return 13;
    }
    avq_shape s = {1, 2, 256, 48, 16, 4, AVQ_BF16};          /* d = 48: not supported */
    if (avq_precompute_workspace_bytes(&s) != 0) return 14;
    if (avq_precompute(&s, 0, 0, 0, 0, 0, 0, 0, 0, 0) != AVQ_EINVAL) return 15;
    s.d = 64;
    if (avq_attention(&s, 0, 0, 0, 0, 17, 128, 0.125f, 0, 0, 0, 0, 0) != AVQ_EINVAL) return 16;  /* P > M0 */
    if (avq_capture_workspace_bytes(&s, 4, 128) != 256) return 17;
    printf("ok\n");
    return 0;
}
"""


def _cc():
    return shutil.which("gcc") or shutil.which("cc")


@pytest.mark.skipif(_cc() is None, reason="no C compiler")
def test_header_is_plain_c_and_cxx(tmp_path):
    src = tmp_path / "inc.c"
    src.write_text('#include "avq.h"\nint main(void) { return 0; }\n')
    subprocess.run([_cc(), "-std=c11", "-Wall", "-Werror", "-fsyntax-only", "-I", HEADER_DIR, str(src)], check=True)
    cxx = shutil.which("g++")
    if cxx:
        srcx = tmp_path / "inc.cc"
        srcx.write_text('#include "avq.h"\nint main() { return 0; }\n')
        subprocess.run([cxx, "-std=c++17", "-Wall", "-Werror", "-fsyntax-only", "-I", HEADER_DIR, str(srcx)],
                       check=True)


@pytest.mark.skipif(_cc() is None, reason="no C compiler")
def test_c_client_links_and_calls_host_entry_points(tmp_path):
    lib = bl.build()
    src = tmp_path / "client.c"
    src.write_text(CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(lib)
    subprocess.run([_cc(), "-std=c11", "-Wall", "-Werror", "-I", HEADER_DIR, str(src), "-o", str(exe),
                    "-L", libdir, "-lavq_b200", "-Wl,-rpath," + libdir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
