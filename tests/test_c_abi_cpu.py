"""The C ABI from plain C, without a GPU: a C11 program that includes only
include/kin.h compiles with gcc -Wall -Werror, links libkin.so, and gets the
documented answers from the calls that need no device (status names,
workspace sizes, arguments rejected before any launch)."""
import os
import shutil
import subprocess

import pytest

from block_top_sparse_kin_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include "kin.h"

int main(void) {
  kin_dims d = {2, 2, 8, 128, 16, 256};
  kin_dims bad = {2, 2, 8, 64, 16, 256};  /* head_dim must be 128 */
  void* p = (void*)(uintptr_t)(1u << 20); /* aligned, never dereferenced */
  size_t ws = kin_workspace_bytes(&d, 8);
  printf("%s\n", kin_status_string(KIN_ERR_WORKSPACE));
  printf("%zu %zu\n", ws, kin_workspace_bytes(&bad, 8));
  printf("%zu\n", kin_token_topk_workspace_bytes(&d, 8));
  /* k_blocks = 1, then a missing workspace: rejected on the host */
  printf("%d %d\n",
         (int)kin_block_topk_select(&d, p, (const float*)p, (const int32_t*)p, 1, (int32_t*)p, (int32_t*)p,
                                    p, ws, NULL, NULL),
         (int)kin_sparse_decode_attn(&d, p, p, p, (const int32_t*)p, (const int32_t*)p, (const int32_t*)p, 8,
                                     0.0f, p, NULL, NULL, ws, NULL, NULL));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_links_and_calls_the_library(tmp_path):
    srcs = [os.path.join(kbuild.CSRC, s) for s in kbuild.SOURCES]
    if not os.path.exists(kbuild.LIB) or os.path.getmtime(kbuild.LIB) < max(map(os.path.getmtime, srcs)):
        kbuild.build()
    libdir = os.path.dirname(kbuild.LIB)
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", libdir, "-lkin", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    assert out[0] == "KIN_ERR_WORKSPACE"
    ws, ws_bad = map(int, out[1].split())
    assert ws > 0 and ws % 256 == 0 and ws_bad == 0
    assert int(out[2]) >= 2 * 8 * 256 * 4     # at least the fp32 logits of every query head
    assert out[3].split() == ["1", "2"]        # KIN_ERR_INVALID_ARG, KIN_ERR_WORKSPACE
