"""The boundary is a plain C ABI: a C11 program compiled with -pedantic
against include/tp_layer.h links against libtplayer.so and calls it.  Only
calls that need no GPU are made (version, status names, workspace sizes, and
argument checks that return before any device work)."""
import os
import shutil
import subprocess

import pytest

import tensor_transformer_layer_column_b200 as tl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include "tp_layer.h"

int main(void) {
  tp_dims d = {1, 8, 256, 1024, 2, 128, 2, 1, 1e-5f};
  tp_dims bad = d;
  tp_status st;
  bad.t = 3;
  printf("%s\n", tp_version());
  printf("%s\n", tp_status_string(TP_ERR_WORKSPACE));
  printf("%d %d\n", tp_workspace_size(TP_OP_LAYER_BWD, &d) > 0,
         (int)tp_workspace_size(TP_OP_LAYER_BWD, &bad));
  st = tp_mlp_fwd(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%d\n", (int)st);
  st = tp_mlp_fwd(&bad, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%d\n", (int)st);
  return 0;
}
"""


def test_c_program_links_and_calls_the_library(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    tl.lib()                                   # builds are checked by test_abi; must exist here
    src = tmp_path / "consumer.c"
    exe = tmp_path / "consumer"
    src.write_text(C_SRC)
    libdir = os.path.dirname(tl.lib_path)
    subprocess.run([cc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), str(src), "-L", libdir, "-ltplayer",
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert out[0].startswith("tplayer-b200")
    assert out[1] == "TP_ERR_WORKSPACE"
    assert out[2] == "1 0"
    assert out[3] == "1"        # TP_ERR_INVALID_ARG: null pointers
    assert out[4] == "2"        # TP_ERR_UNSUPPORTED: t = 3
