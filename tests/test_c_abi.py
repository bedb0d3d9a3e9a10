"""The boundary as a C program sees it: include/mls.h compiles as C99 (not
only C++), and a C program linked against libmls.so runs the host-side
paths that need no GPU: version, status strings, workspace queries and the
synchronous argument checks."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "lm_head_loss_junction_b200")
LIB = os.path.join(LIBDIR, "libmls.so")

PROGRAM = r"""
#include <stdio.h>
#include <stdint.h>
#include <string.h>
#include "mls.h"

int main(void) {
  int fails = 0;
  if (mls_version() <= 0) { printf("bad version\n"); ++fails; }
  if (strcmp(mls_status_string(MLS_OK), "ok") != 0 ||
      strcmp(mls_status_string(MLS_ERR_INVALID_ARG), mls_status_string(MLS_ERR_UNSUPPORTED)) == 0) {
    printf("bad status string\n"); ++fails;
  }

  size_t ws = 0;
  if (mls_junction_bwd_workspace(8192, 49152, &ws) != MLS_OK || ws == 0) { printf("junction ws\n"); ++fails; }
  if (mls_junction_bwd_workspace(0, 49152, &ws) != MLS_ERR_INVALID_ARG) { printf("junction ws T=0\n"); ++fails; }

  int64_t D[3] = {1024, 2304, 4352};
  size_t fb = 0, bb = 0;
  if (mls_multiexit_loss_workspace(3, 8192, D, 49152, MLS_BF16, &fb, &bb) != MLS_OK || fb == 0 || bb == 0) {
    printf("loss ws\n"); ++fails;
  }
  int64_t Dbad[2] = {2304, 1024};                       /* widths must increase */
  if (mls_multiexit_loss_workspace(2, 8192, Dbad, 49152, MLS_BF16, &fb, &bb) != MLS_ERR_INVALID_ARG) {
    printf("loss ws widths\n"); ++fails;
  }
  if (mls_multiexit_loss_workspace(3, 8192, D, 49151, MLS_BF16, &fb, &bb) != MLS_ERR_UNSUPPORTED) {
    printf("loss ws V\n"); ++fails;
  }

  /* argument errors are synchronous and launch nothing: NULL pointers */
  mls_status st = mls_junction_fwd(NULL, 16, NULL, 64, NULL, 32, 64, NULL, NULL, MLS_BF16, NULL, NULL);
  if (st != MLS_ERR_INVALID_ARG) { printf("junction fwd NULL -> %d\n", (int)st); ++fails; }
  mls_loss_options opts;
  memset(&opts, 0, sizeof(opts));
  opts.distill = 9;                                      /* unknown distillation kind */
  const void* ptrs[3] = {NULL, NULL, NULL};
  st = mls_multiexit_loss_fwd_opts(3, 256, 1024, D, NULL, ptrs, ptrs, 0.3f, MLS_BF16, NULL, NULL, NULL, 0,
                                   &opts, NULL, NULL);
  if (st != MLS_ERR_INVALID_ARG) { printf("loss fwd opts -> %d\n", (int)st); ++fails; }

  printf("%s\n", fails == 0 ? "C ABI OK" : "C ABI FAILED");
  return fails;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_a_c_program_links_and_runs(tmp_path):
    if not os.path.exists(LIB):
        pytest.skip("libmls.so not built")
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                         str(src), "-o", str(exe), "-L", LIBDIR, "-lmls", f"-Wl,-rpath,{LIBDIR}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "C ABI OK" in run.stdout, run.stdout + run.stderr
