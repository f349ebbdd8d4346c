"""The C ABI from C: a small C11 program that includes include/swimba.h (compiled with gcc, no
C++), links libswimba.so and calls the host-only entry points (workspace sizing, status strings,
argument checks). Needs no GPU."""
import os
import shutil
import subprocess
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = textwrap.dedent(r"""
    #include <stdio.h>
    #include <string.h>
    #include "swimba.h"

    int main(void) {
      swimba_dims d = {8, 4096, 4096, 16, 128, 8, 2, SWIMBA_BF16, SWIMBA_BF16};
      size_t layer = swimba_workspace_size(&d, SWIMBA_OP_LAYER);
      size_t scan = swimba_workspace_size(&d, SWIMBA_OP_SCAN);
      size_t proj = swimba_workspace_size(&d, SWIMBA_OP_PROJ);
      if (layer < 256 || layer < scan || layer < proj) return 1;
      swimba_block_dims bd = {d, 2048, 4};
      if (swimba_block_workspace_size(&bd) <= layer) return 2;
      swimba_dims bad = d;
      bad.top_k = 9;
      if (swimba_workspace_size(&bad, SWIMBA_OP_LAYER) != 0) return 3;
      if (strcmp(swimba_status_string(SWIMBA_OK), "ok") != 0) return 4;
      /* argument errors come back before anything is launched (no device needed) */
      if (swimba_route(&d, NULL, NULL, NULL, NULL, NULL) != SWIMBA_ERR_INVALID_ARG) return 5;
      if (swimba_get_device_status(NULL, NULL) != SWIMBA_ERR_INVALID_ARG) return 6;
      if (swimba_conv1d_fwd(&d, 9, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != SWIMBA_ERR_UNSUPPORTED) return 7;
      printf("layer=%zu block=%zu launches=%llu\n", layer, swimba_block_workspace_size(&bd),
             (unsigned long long)swimba_kernel_launches());
      return 0;
    }
""")


@pytest.fixture(scope="module")
def lib():
    from parameter_space_moe_swimba_b200 import build

    return build.build()


def test_header_compiles_as_c_and_the_library_links(lib, tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    cmd = [gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
           "-L", libdir, "-lswimba", f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("layer=")
