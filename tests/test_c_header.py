"""The C ABI from plain C: include/fa.h compiles as C99 with gcc, a program
links libfa.so, and the argument checks answer as the header documents
(no device is needed: every call here fails before anything is launched)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "exact_io_aware_84_b200")

C_PROGRAM = r"""
#include <stdio.h>
#include "fa.h"

#define EXPECT(call, want)                                                  \
  do {                                                                      \
    int got_ = (call);                                                      \
    if (got_ != (want)) {                                                   \
      printf("FAIL %s -> %d (%s), want %d\n", #call, got_,                  \
             fa_status_string(got_), (int)(want));                          \
      return 1;                                                             \
    }                                                                       \
  } while (0)

int main(void) {
  char buf[64] = {0};
  void* p = (void*)(buf + (16 - ((size_t)buf & 15)) % 16);  /* any 16-byte aligned address */
  float* f = (float*)p;
  EXPECT(fa_fwd(NULL, p, p, p, f, 1, 1, 128, 64, 0.125f, 0, FA_BF16, NULL), FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd(p, p, p, p, f, 1, 1, 128, 96, 0.125f, 0, FA_BF16, NULL), FA_ERR_UNSUPPORTED);
  EXPECT(fa_fwd(p, p, p, p, f, 1, 1, 0, 64, 0.125f, 0, FA_BF16, NULL), FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd(p, p, p, (char*)p + 2, f, 1, 1, 128, 64, 0.125f, 0, FA_BF16, NULL), FA_ERR_MISALIGNED);
  EXPECT(fa_bwd(p, p, p, p, p, f, p, p, p, NULL, 0, 1, 1, 128, 64, 0.125f, 1, FA_FP16, NULL), FA_ERR_WORKSPACE);
  EXPECT(fa_fwd_gqa(p, p, p, p, f, 1, 6, 4, 128, 64, 0.125f, 0, FA_BF16, NULL), FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd_blocksparse(p, p, p, p, f, NULL, 0, 1, 1, 128, 64, 0.125f, 0, FA_BF16, NULL), FA_ERR_INVALID_ARG);
  EXPECT(fa_fwd_fp8(p, p, p, p, f, NULL, NULL, 0, 1, 1, 128, 64, 0.1f, 0, FA_BF16, NULL), FA_ERR_UNSUPPORTED);
  EXPECT(fa_merge(f, f, f, f, NULL, -1, 0, 64, NULL), FA_OK);
  if (fa_bwd_workspace_size(1, 1, 128, 64) != (size_t)(128 * 64 * 4 + 2 * 512)) {
    printf("FAIL workspace size %zu\n", fa_bwd_workspace_size(1, 1, 128, 64));
    return 1;
  }
  if (fa_fwd_fp8_workspace_size(1, 1, 128, 64) != 0) { printf("FAIL fp8 size\n"); return 1; }
  printf("OK %s\n", fa_version());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_compiles_as_c_and_argument_checks_answer(tmp_path):
    lib = os.path.join(LIB_DIR, "libfa.so")
    if not os.path.exists(lib):
        pytest.skip("libfa.so not built")
    src = tmp_path / "abi_check.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           "-L", LIB_DIR, "-lfa", "-Wl,-rpath," + LIB_DIR, "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("OK"), r.stdout + r.stderr
