"""The boundary from C: a plain C program compiled against include/attn.h and linked to
libattn_b200.so calls the entry points that need no GPU -- status strings, workspace
sizes, the checking-build flag, and argument validation that rejects a call before any
launch -- and prints what it gets.  No CUDA header, no torch, no Python in the client."""
import os
import subprocess

import __graft_entry__

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "io_aware_exact_26_b200")

CLIENT = r"""
#include <stdio.h>
#include "attn.h"

int main(void) {
  /* statuses and their texts */
  printf("ok=%s\n", attn_status_string(ATTN_OK));
  printf("conflict=%d\n", ATTN_ERR_SCHED_CONFLICT);
  printf("checks=%d\n", attn_checks_enabled());
  /* 8 bytes per query row, rows padded to whole 128-row tiles, 256-byte aligned parts */
  printf("ws=%zu\n", attn_bwd_workspace_size(2, 4, 2, 1000, 128, 1));
  printf("ws_bad=%zu\n", attn_bwd_workspace_size(2, 4, 3, 1000, 128, 1));
  /* rejected before any launch: NULL pointers, unsupported head size, bad GQA split */
  printf("null=%d\n", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 1, 128, 128, 0.088f, 1, NULL));
  printf("d96=%d\n", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 1, 128, 96, 0.088f, 1, NULL));
  printf("gqa=%d\n", attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 3, 2, 128, 128, 0.088f, 1, NULL));
  return 0;
}
"""


def test_c_program_links_the_library_and_calls_the_boundary(tmp_path):
    __graft_entry__.build()
    src = tmp_path / "client.c"
    src.write_text(CLIENT)
    exe = tmp_path / "client"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-L", LIBDIR, "-lattn_b200", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    got = dict(line.split("=", 1) for line in out.stdout.strip().splitlines())
    assert got["ok"] == "ok"
    assert int(got["conflict"]) == -9
    assert got["checks"] == "0"
    rows = 2 * 4 * 1024                                   # B * Hq * N padded to 1024
    assert int(got["ws"]) == 2 * rows * 4                 # -lse2 and -D, fp32, 256-byte aligned parts
    assert int(got["ws_bad"]) == 0
    assert int(got["null"]) == -1                         # ATTN_ERR_INVALID_ARG
    assert int(got["d96"]) == -2                          # ATTN_ERR_UNSUPPORTED
    assert int(got["gqa"]) == -1
