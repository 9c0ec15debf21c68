"""The boundary is a C ABI: include/fa.h must compile as plain C (C99) and a C
program must be able to link libfa.so and call it.  CPU only: the calls made
here (status strings, workspace sizes, argument checks) never reach a GPU."""
import os
import shutil
import subprocess

import pytest

import exact_io_aware_50_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include "fa.h"

int main(void) {
  char buf[16];
  printf("%s\n", fa_strerror(FA_OK));
  printf("%zu\n", fa_bwd_workspace_size(4, 16, 4096, 128));
  printf("%zu\n", fa_fwd_splitkv_workspace_size(1, 8, 512, 128, 9));
  printf("%d\n", fa_fwd_splitkv_num_splits(1, 8, 512, 16384, 128));
  /* null pointers are refused before anything touches a device */
  printf("%d\n", fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 8, 8, 64, 0.125f, 0, NULL));
  printf("%d\n", fa_fwd_dropout(buf, buf, buf, buf, (float *)buf, 1, 1, 1, 8, 8, 64, 0.125f, 0,
                                1.5f, 1ULL, 0ULL, (fa_stream_t)0));
  /* e4m3 forward: a zero dequantisation factor, then an unsupported head dim */
  printf("%d\n", fa_fwd_fp8(buf, buf, buf, buf, (float *)buf, 1, 1, 1, 8, 128, 0.125f, 0.0f,
                            1.0f, 1.0f, 0, (fa_stream_t)0));
  printf("%d\n", fa_fwd_fp8(buf, buf, buf, buf, (float *)buf, 1, 1, 1, 8, 64, 0.125f, 1.0f,
                            1.0f, 1.0f, 0, (fa_stream_t)0));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c_and_library_links(tmp_path):
    F.lib()   # builds nothing; fails loudly if the library is missing
    src = tmp_path / "use_fa.c"
    src.write_text(C_SRC)
    exe = tmp_path / "use_fa"
    libdir = os.path.dirname(F.lib_path)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lfa", "-Wl,-rpath," + libdir, "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert out[0] == "ok"
    assert int(out[1]) == F.fa_bwd_workspace_size(4, 16, 4096, 128)
    assert int(out[2]) == F.fa_fwd_splitkv_workspace_size(1, 8, 512, 128, 9)
    assert int(out[3]) == 9
    assert int(out[4]) == F.FA_ERR_INVALID_ARG
    assert int(out[5]) == F.FA_ERR_INVALID_ARG      # p_drop outside [0, 1)
    assert int(out[6]) == F.FA_ERR_INVALID_ARG      # descale_q = 0
    assert int(out[7]) == F.FA_ERR_UNSUPPORTED      # e4m3 at d = 64
