"""A plain C program (gcc, C99) includes include/lserve.h, links
liblserve.so and calls the host-side entry points: the header is valid C and
the exported symbols carry the declared C signatures."""
import os
import shutil
import subprocess

import pytest

import block_sparse_attention_page_b200 as lserve

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "lserve.h"

int main(void) {
  int32_t lo, hi, n;
  lserve_paged_desc d = {1, 32, 8, 128, 16, 128, 2048, 2048};
  if (strcmp(lserve_status_string(LSERVE_OK), "ok") != 0) return 1;
  if (lserve_seqshard_bounds(262144, 128, 3, 4, &lo, &hi, &n) != LSERVE_OK) return 2;
  if (lo != 1536 || hi != 2048 || n != 65536) return 3;
  if (lserve_seqshard_bounds(10, 0, 0, 1, &lo, &hi, &n) != LSERVE_ERR_INVALID_ARG) return 4;
  if (lserve_seqshard_sel_stride(&d, 4, 128, 1024) != 10) return 5;
  /* validation happens before any device work: a null q is rejected */
  if (lserve_page_select(&d, NULL, NULL, NULL, NULL, NULL, 8, NULL, NULL, NULL, NULL, 0, NULL)
      != LSERVE_ERR_INVALID_ARG) return 6;
  /* the prefill with the paged hand-over: a null block table is rejected */
  {
    lserve_prefill_desc pf = {1024, 32, 8, 128, 128, 128, 1, 4};
    uint8_t kinds[8] = {0, 0, 0, 0, 1, 1, 1, 1};
    if (lserve_blocksparse_prefill_paged(&pf, &d, NULL, NULL, NULL, kinds, 0.088f, NULL, NULL, NULL,
                                         NULL, NULL, NULL, NULL, 0, NULL) != LSERVE_ERR_INVALID_ARG)
      return 7;
  }
  printf("c client ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_links_and_calls_the_library():
    bdir = os.path.join(ROOT, "tests", "_build")
    os.makedirs(bdir, exist_ok=True)
    src = os.path.join(bdir, "c_client.c")
    exe = os.path.join(bdir, "c_client")
    with open(src, "w") as f:
        f.write(PROGRAM)
    libdir = os.path.dirname(lserve.library_path())
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                        "-L", libdir, "-llserve", "-Wl,-rpath," + libdir, "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "c client ok" in r.stdout, (r.returncode, r.stdout, r.stderr)
