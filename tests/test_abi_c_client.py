"""The boundary from plain C: include/bsa.h compiles as strict C99 and a C
program linked against libbsa.so gets the sizes of the 720p workload and
the validation errors without a GPU (no call here reaches the device)."""
import os
import shutil
import subprocess

import pytest

import block_sparse_attention_47_b200 as bsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include "bsa.h"

int main(void) {
  bsa_problem p = {0};
  bsa_sizes s;
  p.B = 2; p.heads = 24; p.head_dim = 128;
  p.T = 32; p.H = 48; p.W = 80; p.T_valid = 32; p.H_valid = 48; p.W_valid = 80;
  p.keep_blocks = bsa_keep_count(1920, 0.25);
  p.block_mode = BSA_BLOCK_FIXED_444;
  p.dyn_tau = 1.25f;
  p.softmax_scale = 0.08838834764831845f;
  if (bsa_query_sizes(&p, &s) != BSA_OK) return 1;
  if (s.n_tokens != 122880 || s.n_blocks != 1920 || s.list_capacity != 480) return 2;
  p.head_dim = 96;  /* unsupported: rejected on the host, nothing launched */
  if (bsa_query_sizes(&p, &s) != BSA_ERR_UNSUPPORTED) return 3;
  if (bsa_last_error()[0] == '\0') return 4;
  printf("%s\n", bsa_status_string(BSA_ERR_UNSUPPORTED));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_client(tmp_path):
    from block_sparse_attention_47_b200 import build
    build.build()
    src = tmp_path / "client.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "client"
    libdir = os.path.dirname(bsa.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lbsa",
                         "-Wl,-rpath," + libdir, "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert run.stdout.strip() == "BSA_ERR_UNSUPPORTED"
