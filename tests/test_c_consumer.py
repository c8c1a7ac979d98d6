"""The C ABI from a plain C program (no GPU needed).

Compiles a C99 program against include/sage.h with gcc, links it to the
in-tree libsage.so, and runs it: sage_npad and sage_workspace_bytes return the
documented sizes, and every call that gets an invalid argument returns its
documented status with a message from sage_last_error() before touching a
device.  This is what a C or C++ caller without PyTorch sees.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "action_diffusion_transformers_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "sage.h"

static int fails = 0;
#define CHECK(cond, what) do { if (!(cond)) { printf("FAIL %s\n", what); ++fails; } } while (0)

int main(void) {
  CHECK(sage_npad(1) == 128 && sage_npad(128) == 128 && sage_npad(129) == 256 && sage_npad(0) == 0, "npad");
  sage_shape s;
  memset(&s, 0, sizeof(s));
  s.B = 1; s.N = 1000; s.H = 4; s.D = 128;
  size_t ws = sage_workspace_bytes(s);
  CHECK(ws >= 1000 / 64 * 4 * 128 * 8, "workspace covers the FP64 partial sums");
  CHECK(ws % 256 == 0, "workspace is a multiple of 256 bytes");

  char dummy[64] __attribute__((aligned(256)));
  /* a NULL input: invalid argument, with a message naming it */
  sage_status st = sage_quant_qk(NULL, dummy, s, (int8_t*)dummy, (float*)dummy, (int8_t*)dummy, (float*)dummy,
                                 NULL, dummy, ws, NULL);
  CHECK(st == SAGE_ERR_INVALID_ARG, "quant_qk NULL q -> INVALID_ARG");
  CHECK(strstr(sage_last_error(), "q") != NULL, "message names q");
  /* an unsupported head dimension */
  sage_shape bad = s;
  bad.D = 96;
  st = sage_quant_v(dummy, bad, (uint8_t*)dummy, (float*)dummy, (float*)dummy, dummy, ws, NULL);
  CHECK(st == SAGE_ERR_UNSUPPORTED || st == SAGE_ERR_INVALID_ARG, "quant_v D = 96 rejected");
  /* a workspace that is too small */
  st = sage_quant_v(dummy, s, (uint8_t*)dummy, (float*)dummy, (float*)dummy, dummy, 16, NULL);
  CHECK(st == SAGE_ERR_WORKSPACE, "quant_v small workspace -> WORKSPACE");
  /* cu_seqlens that do not end at N */
  int32_t cu[3] = {0, 400, 999};
  sage_shape rag = s;
  rag.cu_seqlens = cu;
  rag.n_seg = 2;
  st = sage_attn_fwd((const int8_t*)dummy, (const float*)dummy, (const int8_t*)dummy, (const float*)dummy,
                     (const uint8_t*)dummy, (const float*)dummy, (const float*)dummy, rag, 0.f, dummy, 0, NULL,
                     NULL);
  CHECK(st == SAGE_ERR_INVALID_ARG, "attn_fwd bad cu_seqlens -> INVALID_ARG");
  printf("%s\n", fails ? "FAILED" : "OK");
  return fails ? 1 : 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_against_the_header_and_library(tmp_path):
    if not os.path.exists(os.path.join(LIBDIR, "libsage.so")):
        pytest.skip("libsage.so is not built")
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", LIBDIR, "-lsage", "-Wl,-rpath," + LIBDIR, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr
