"""The boundary is a C ABI: a plain C99 program (and a C++ one) compiles
against include/moba.h without warnings, links against libmoba.so and calls
the size queries and argument checks, which need no GPU."""
import os
import shutil
import subprocess

import pytest

from long_context_prefill_moba_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "long_context_prefill_moba_b200")

PROGRAM = r"""
#include <stdio.h>
#include "moba.h"
int main(void) {
  moba_shape_t s = {1, 1 << 20, 32, 8, 128, 4096, 12, MOBA_BF16, 0.0f, 0};
  if (moba_check_shape(&s) != MOBA_OK) return 1;
  if (moba_num_blocks(&s) != 256) return 2;
  if (moba_attn_workspace_size(&s) == 0 || moba_prefill_host_workspace_size(&s, 1) == 0) return 3;
  /* argument checks happen before anything is enqueued */
  if (moba_attn_fwd(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) != MOBA_ERR_INVALID_ARG)
    return 4;
  if (moba_last_launch_count() != 0) return 5;
  /* the pooled-gate variant's wide shape and the one-allocation sizes */
  moba_shape_t w;
  if (moba_pooled_wide_shape(&s, 2, &w) != MOBA_OK || w.topk != 16) return 6;
  if (moba_pooled_wide_shape(&s, 3, &w) != MOBA_ERR_UNSUPPORTED) return 7;
  if (moba_workspace_size(&s) != moba_gate_workspace_size(&s) + moba_attn_workspace_size(&s)) return 8;
  if (moba_rows_capacity(&s) != moba_rows_elems(&s)) return 9;
  if (moba_check_index(&s, 1, NULL, NULL, NULL, NULL, NULL) != MOBA_ERR_INVALID_ARG) return 10;
  printf("%s\n", moba_status_string(MOBA_ERR_WORKSPACE));
  return 0;
}
"""


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-std=c99", "-pedantic"]), ("g++", ["-std=c++17"])])
def test_header_is_a_c_abi(tmp_path, compiler, flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    B.build()
    src = tmp_path / ("prog.c" if compiler == "gcc" else "prog.cpp")
    src.write_text(PROGRAM)
    exe = tmp_path / "prog"
    cmd = [compiler, *flags, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           "-L", LIBDIR, "-lmoba", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    assert res.returncode == 0, (res.returncode, res.stdout, res.stderr)
    assert res.stdout.startswith("MOBA_ERR_WORKSPACE")


def test_every_declaration_is_documented():
    # each MOBA_API entry point in include/moba.h follows a comment block that
    # documents it (the header is the boundary's contract)
    import re
    text = open(os.path.join(ROOT, "include", "moba.h")).read()
    lines = text.splitlines()
    undocumented = []
    for i, ln in enumerate(lines):
        m = re.match(r"MOBA_API\s+[\w\s\*]*?\b(moba_\w+)\s*\(", ln)
        if not m:
            continue
        j = i - 1
        while j >= 0 and lines[j].startswith("MOBA_API"):      # a run of related declarations
            j -= 1
        while j >= 0 and (lines[j].startswith(" ") and not lines[j].lstrip().startswith(("*", "/*"))):
            j -= 1                                             # continuation of the previous declaration
        if j < 0 or not lines[j].rstrip().endswith("*/"):
            undocumented.append(m.group(1))
    assert not undocumented, undocumented
