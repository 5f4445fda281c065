"""include/moe.h is a C header: a C99 program that includes it and references every entry
point links against libmoe.so and runs its host-only calls (no GPU needed)."""
import os
import re
import shutil
import subprocess

import pytest

import moe_expert_layer_prefix_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"


def _entry_points():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:moe_status|size_t|const char\*|uint64_t)\s+(moe_\w+)\(", src, re.M)


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INC),
                    reason="needs gcc and the CUDA headers")
def test_c99_program_links_and_runs_host_calls(tmp_path):
    names = _entry_points()
    refs = "\n".join(f"    (void *)&{n}," for n in names)
    prog = f"""
#include <stdio.h>
#include "moe.h"
static void *const entry_points[] = {{
{refs}
}};
int main(void) {{
  printf("%s\\n", moe_status_string(MOE_ERR_WORKSPACE));
  printf("%zu\\n", moe_workspace_size(MOE_OP_FORWARD, 64, 256, 8, 2, 128, MOE_E4M3, MOE_E4M3));
  printf("%zu\\n", moe_workspace_size(MOE_OP_BACKWARD, 64, 256, 8, 2, 128, MOE_BF16, MOE_BF16));
  printf("%d\\n", (int)moe_route(NULL, NULL, 4, 8, 2, MOE_SCORE_SOFTMAX, 1, NULL, NULL, NULL));
  printf("%d\\n", (int)(sizeof(entry_points) / sizeof(entry_points[0])));
  return 0;
}}
"""
    c = tmp_path / "abi.c"
    c.write_text(prog)
    exe = tmp_path / "abi"
    lib_dir = os.path.dirname(M.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", str(c), "-o", str(exe),
                        "-I" + os.path.join(ROOT, "include"), "-I" + CUDA_INC, "-L" + lib_dir,
                        "-l:libmoe.so", "-Wl,-rpath," + lib_dir],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.split()
    assert lines[0] == "MOE_ERR_WORKSPACE"
    assert int(lines[1]) == M.moe_workspace_size("forward", 64, 256, 8, 2, 128, "e4m3", "e4m3")
    assert int(lines[2]) == M.moe_workspace_size("backward", 64, 256, 8, 2, 128, "bf16", "bf16")
    assert M.moe_status_string(int(lines[3])) == "MOE_ERR_INVALID_ARG"
    assert int(lines[4]) == len(names) == len(M.EXPORTS)
