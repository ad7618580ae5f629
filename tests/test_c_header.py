"""The boundary as a C user sees it: include/mxc.h compiles as strict C99, and a
plain C program links against the library and runs its host-only entry points
(no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from vector_quantized_mx_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "mxc.h"

int main(void) {
  static uint8_t idx[256 * 128], scales[4];
  static uint16_t cb[4 * 256];
  mxc_weight_host w;
  mxc_packed_sizes sz;
  memset(&w, 0, sizeof w);
  w.strategy = MXC_POSTSCALE_QB;
  w.fmt = MXC_FMT_E4M3_B16;
  w.N = 256; w.K = 512; w.qn = 128; w.qk = 256;
  w.idx = idx; w.cb = cb; w.scales = scales; w.w_tscale = 1.0f;
  if (mxc_packed_weight_sizes(&w, &sz) != MXC_OK) return 1;
  printf("%zu %zu %zu %zu\n", sz.idx, sz.cb, sz.scales, mxc_sf_bytes(16, 4096, MXC_FMT_E4M3_B16));
  printf("%s|%s|%d\n", mxc_status_string(MXC_OK), mxc_status_string(MXC_ERR_ALIGNMENT), mxc_version());
  w.K = 500;                                   /* not a multiple of 256 */
  printf("%d\n", (int)mxc_packed_weight_sizes(&w, &sz));
  return 0;
}
"""


def test_header_is_strict_c99_and_links(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = build.build()
    src = tmp_path / "use_mxc.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_mxc"
    libdir = os.path.dirname(lib)
    # the library is libmxc.so next to the package: link it by path, find it at run time by rpath
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), lib, f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert out[0].split() == [str(256 * 128), str(2 * 2 * 256 * 2), str(2 * 2), str(128 * 4096 // 16)]
    assert out[1] == "ok|shape or alignment requirement not met|100"
    assert out[2] == "3"                          # MXC_ERR_ALIGNMENT
