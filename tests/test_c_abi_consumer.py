"""The boundary is a plain C ABI: a C99 program that includes include/gptq.h
(no CUDA or C++ headers) compiles with gcc, links against the built library,
and calls the host-only parts (status strings, workspace sizes, argument
checks that return before any device work).  No GPU is touched."""

import os
import shutil
import subprocess
import tempfile

import pytest

from post_weight_quantization_23_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "gptq.h"

int main(void) {
  gptq_config cfg = {4, 128, 128, 0.01f, 0, 0, 0};
  size_t q = gptq_workspace_size(GPTQ_OP_QUANTIZE, 4096, 4096, 0, &cfg);
  if (q < (size_t)4 * 4096 * 4096) return 1;
  if (strcmp(gptq_status_string(GPTQ_ERR_NOT_PD), "GPTQ_ERR_NOT_PD") != 0) return 2;
  /* rejected on the host: bad bit width, before anything is enqueued */
  if (gptq_pack((const uint8_t*)256, 4, 32, 5, (int32_t*)256, NULL) != GPTQ_ERR_UNSUPPORTED) return 3;
  if (gptq_gemm((const void*)256, GPTQ_F32, 1, 256, 256, (const int32_t*)256, (const float*)256,
                (const int32_t*)256, NULL, 8, 4, 128, 2, (void*)256, 8, NULL) != GPTQ_ERR_UNSUPPORTED)
    return 4;
  if (gptq_rotate((const void*)256, GPTQ_F16, 0, 512, 512, (const int8_t*)256, 256, 0,
                  (void*)4096, 512, NULL) != GPTQ_OK)
    return 5;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c99_program_includes_header_and_links():
    if not os.path.exists(_lib.LIB_PATH):
        from post_weight_quantization_23_b200 import build
        build.build()
    libdir = os.path.dirname(_lib.LIB_PATH)
    libname = os.path.basename(_lib.LIB_PATH)
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "consumer.c")
        exe = os.path.join(d, "consumer")
        open(src, "w").write(PROGRAM)
        cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src,
               "-o", exe, os.path.join(libdir, libname), f"-Wl,-rpath,{libdir}"]
        subprocess.run(cmd, check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=60)
        assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
        assert out.stdout.strip() == "ok"
