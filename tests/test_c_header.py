"""include/moe.h is a C header: a plain C11 program includes it, links
libmoe.so and calls the host-only entry points (sizes, capacity, status
strings, argument checks) -- no GPU involved."""
import os
import shutil
import subprocess

import pytest

from mixture_experts_layer_49_b200 import native as nat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "moe.h"

int main(void) {
    moe_config c = {0};
    c.T = 8192; c.d_model = 1024; c.E = 16; c.d_ff = 4096; c.top_k = 1;
    c.dtype = MOE_BF16; c.act = MOE_ACT_GELU_BIAS; c.score = MOE_SCORE_SOFTMAX;
    c.renorm = 0; c.capacity_factor = 1.25f; c.d_ff_shared = 0;
    size_t ws = moe_workspace_size(&c);
    int32_t cap = moe_capacity(&c);
    int64_t rows = moe_perm_rows(&c);
    moe_status bad = moe_forward(&c, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                                 NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
    printf("%zu %d %lld %d %s\n", ws, (int)cap, (long long)rows, (int)bad, moe_status_string(bad));
    return ws > 0 && cap == 640 && rows == 8192 && bad == MOE_ERR_INVALID_ARG ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c_and_links(tmp_path):
    lib = nat._build.build()
    src = tmp_path / "use_moe.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_moe"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    ws, cap, rows, status, _ = out.stdout.split(maxsplit=4)
    assert int(ws) == nat.workspace_size(nat.make_config(8192, 1024, 16, 4096, 1, act="gelu", renorm=0,
                                                         capacity_factor=1.25))
