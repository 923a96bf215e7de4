"""The C ABI from a C program (no GPU): a C99 translation unit includes
include/thrift.h, links libthrift.so and calls the entry points that need no
device — sizes, status strings and argument checks — and its results agree
with the Python binding's."""
import os
import shutil
import subprocess

import pytest

import fp16_block_attention_b200 as thrift

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "fp16_block_attention_b200")

PROGRAM = r"""
#include <stdio.h>
#include "thrift.h"

int main(void) {
  thrift_shape s = {1, 32, 8, 32768, 128, 128, 1, 0.08838834764831845f};
  size_t c = 0, sc = 0, c8 = 0, s8 = 0, ws = 0, fw = 0, fw8 = 0;
  if (thrift_quant_bytes(&s, THRIFT_Q, &c, &sc) != THRIFT_OK) return 1;
  if (thrift_quant8_bytes(&s, THRIFT_V, &c8, &s8) != THRIFT_OK) return 2;
  if (thrift_select_workspace_bytes(&s, &ws) != THRIFT_OK) return 3;
  if (thrift_fused_workspace_bytes(&s, &fw) != THRIFT_OK) return 4;
  if (thrift_fused_tiered_workspace_bytes(&s, 0.1, &fw8) != THRIFT_OK) return 5;
  thrift_shape bad = s;
  bad.D = 96;
  printf("%zu %zu %zu %zu %zu %zu %zu %d %d %d %s\n", c, sc, c8, s8, ws, fw, fw8,
         (int)thrift_quant_bytes(&bad, THRIFT_Q, &c, &sc),
         (int)thrift_select_blocks(NULL, NULL, &s, 0.05, NULL, NULL, 0, NULL),
         (int)thrift_attention_fused_tiered(NULL, NULL, NULL, &s, 0.05, 2.0, 0.0, NULL, NULL, 0, NULL),
         thrift_strerror(THRIFT_ERR_WORKSPACE));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_links_and_calls_the_library(tmp_path):
    src = tmp_path / "consumer.c"
    exe = tmp_path / "consumer"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", LIBDIR, "-lthrift", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    c, sc, c8, s8, ws, fw, fw8 = (int(v) for v in out[:7])
    sh = thrift.Shape(1, 32, 8, 32768, 128, 128, True, 0.08838834764831845)
    assert (c, sc) == thrift.quant_bytes(sh, thrift.Q)
    assert (c8, s8) == thrift.quant8_bytes(sh, thrift.V)
    assert ws == thrift.select_workspace_bytes(sh)
    assert fw == thrift.fused_workspace_bytes(sh)
    assert fw8 == thrift.fused_tiered_workspace_bytes(sh, 0.1)
    assert [int(v) for v in out[7:10]] == [2, 1, 1]          # unsupported D, null pointers, rho8 > 1
    assert " ".join(out[10:]) == thrift.lib().thrift_strerror(5).decode()
