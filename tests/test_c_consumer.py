"""A plain C program uses the library through include/misa.h alone: the header
compiles as strict C11, the program links against libmisa.so and runs the calls
that need no GPU (version, status strings, workspace sizes, host-side argument
rejection)."""
import os
import shutil
import subprocess

import pytest

import sparse_attention_token_misa_b200 as pkg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "misa.h"

int main(void) {
  if (misa_abi_version() != MISA_ABI_VERSION) return 1;
  if (strcmp(misa_status_string(MISA_OK), "ok") != 0) return 2;
  /* router scratch for 32 queries, 64 heads, L = 32768, B = 128 (documented formula) */
  size_t ws = misa_workspace_bytes(MISA_OP_ROUTE_HEADS, 32, 64, 32768, 128, 0, 0);
  if (ws != 256 + 32 * 8 * 64 * 4 + 4 * 32) return 3;
  /* k = 0 is rejected on the host, before anything is launched */
  unsigned char fake[512];
  int st = misa_topk((const float*)(fake + 0), 2, 64, 64, NULL, NULL, 0, 0, (int32_t*)(fake + 256),
                     fake, sizeof(fake), NULL);
  if (st != MISA_ERR_INVALID_ARG) return 4;
  printf("ok %zu\n", ws);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_uses_the_abi(tmp_path):
    lib = pkg.lib()  # builds nothing; fails loudly if the library is missing
    del lib
    src = tmp_path / "consumer.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.join(ROOT, "sparse_attention_token_misa_b200")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lmisa", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("ok ")
