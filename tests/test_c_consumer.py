"""A plain C99 program compiles against include/ttt.h alone, links libttt.so and calls the
entry points that need no GPU: the boundary is a C ABI, not a C++ or Python one."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "ttt.h"

int main(void) {
  ttt_config cfg;
  ttt_state* st = NULL;
  if (ttt_config_init(&cfg, TTT_RULE_INPLACE_HEBBIAN) != TTT_OK) return 1;
  printf("abi=%d chunk=%d io=%d taps=%d\n", (int)ttt_abi_version(), (int)cfg.chunk, (int)cfg.io_dtype,
         (int)cfg.conv_taps);
  if (ttt_config_init(&cfg, 9) != TTT_ERR_INVALID_ARG) return 2;
  if (strstr(ttt_last_error_string(), "unknown rule") == NULL) return 3;
  if (ttt_chunk_scan(st, NULL, NULL, NULL, 0, NULL, NULL, NULL) != TTT_ERR_INVALID_ARG) return 4;
  if (ttt_state_create(&cfg, NULL, NULL, NULL, NULL, NULL) != TTT_ERR_INVALID_ARG) return 5;
  if (ttt_state_destroy(NULL) != TTT_OK) return 6;
  if (ttt_state_launch_count(NULL) != 0) return 7;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_uses_the_abi(tmp_path):
    from chunked_weight_layers_b200 import build
    lib = build.build()
    src = tmp_path / "consumer.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lttt", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.splitlines() == ["abi=2 chunk=1024 io=1 taps=3", "ok"]
