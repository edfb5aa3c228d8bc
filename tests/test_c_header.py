"""include/ep.h is a plain C header: a C11 program that includes it compiles
with warnings as errors, links against libep_b200.so and calls the entry
points whose host checks need no GPU."""

import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include "ep.h"

int main(void)
{
    ep_route_cfg cfg = {256, 8, 4, 8, 2.5f, 1};
    size_t ws = ep_workspace_size(8192, 8, 256, 8);
    if (ws == 0) return 1;
    if (ep_workspace_size(-1, 8, 256, 8) != 0) return 2;
    /* host checks fail before any CUDA call: no GPU is needed */
    if (ep_route(NULL, NULL, -1, cfg, NULL, NULL, NULL) != EP_ERR_INVALID) return 3;
    if (ep_silu_mul(NULL, 4, 100, NULL, NULL, 0, 1, NULL, NULL, 0, NULL) != EP_ERR_INVALID) return 4;
    if (ep_dispatch(NULL, -1, 256, 8, 0, NULL, 1, NULL, NULL, 0, NULL, NULL) != EP_ERR_INVALID)
        return 5;
    printf("%s|%zu\n", ep_status_string(EP_ERR_UNSUPPORTED), ws);
    return 0;
}
"""


def test_header_compiles_as_c_and_links(tmp_path):
    from combine_ep_route_02_b200.build import LIB
    if not os.path.exists(LIB):
        pytest.skip("library not built")
    src = tmp_path / "use_ep.c"
    src.write_text(C_SRC)
    exe = tmp_path / "use_ep"
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                           LIB, "-Wl,-rpath," + os.path.dirname(LIB)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stderr)
    name, ws = out.stdout.strip().split("|")
    assert name.startswith("EP_ERR_UNSUPPORTED")
    assert int(ws) > 0
