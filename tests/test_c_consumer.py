"""The boundary is a plain C ABI: a C99 program that includes include/bsa.h
and links libbsa.so (no Python, no torch, no C++) compiles with -pedantic
-Werror, links, and runs the library's host-side calls (CPU only):
version and status names, the host interval-width function on a hand-worked
histogram, the reorder workspace size, and argument validation that returns
BSA_EINVAL before any device is touched."""

import os
import shutil
import subprocess

import pytest

from block_sparse_attention_logits_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "bsa.h"

int main(void) {
  /* histogram of runs per row: 5 rows with 1 run, 3 with 2, 2 with 3 */
  const int32_t hist[4] = {0, 5, 3, 2};
  const double qs[3] = {1.0, 0.8, 0.5};
  bsa_shape s = {1, 2, 256, 128, 128};
  int W = -1, i, r;
  printf("version %d\n", bsa_version());
  printf("einval %s\n", bsa_strerror(BSA_EINVAL));
  for (i = 0; i < 3; ++i) {
    r = bsa_interval_width_for_merge(hist, 4, qs[i], &W);
    printf("width %d %d\n", r, W);
  }
  r = bsa_interval_width_for_merge(hist, 4, 0.0, &W);
  printf("width_q0 %d\n", r == BSA_EINVAL);
  printf("workspace %d\n", bsa_reorder_workspace_bytes(21, 45, 80) > 0);
  r = bsa_sparse_attn_fwd(s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL);
  printf("null_q %d\n", r == BSA_EINVAL);
  return 0;
}
"""


def test_c99_program_links_and_runs(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(_lib.LIB_PATH):
        from block_sparse_attention_logits_b200 import build
        build.build()
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lbsa", f"-Wl,-rpath,{libdir}"],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, timeout=60).stdout.split("\n")
    lines = dict(line.split(" ", 1) for line in out if line)
    assert int(lines["version"]) >= 10000
    assert lines["einval"] == _lib.load().bsa_strerror(_lib.BSA_EINVAL).decode()
    widths = [line for line in out if line.startswith("width ")]
    # q = 1: the widest row (3); q = 0.8: 8 rows within 2; q = 0.5: 5 rows within 1
    assert widths == ["width 0 3", "width 0 2", "width 0 1"]
    assert lines["width_q0"] == "1"
    assert lines["workspace"] == "1"
    assert lines["null_q"] == "1"
