"""The C ABI from plain C (no Python, no GPU): a C99 program compiled against include/fd.h and
linked to libfd.so calls the host-only entry points (the split planner, status strings, argument
checks that return before any device work) and prints what it gets."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "split_kv_decode_flashdecoding_b200")

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "fd.h"

int main(void) {
  /* the host planner: 3 sequences, 2 KV heads, capacity 4096, planner splits, 148 CTAs */
  const int32_t lens[3] = {4096, 10, 0};
  int32_t splits[3] = {0, 0, 0};
  int32_t items[5 * 64];
  fd_plan_info info;
  fd_status s = fd_split_plan(lens, 3, 2, 4096, 0, 148, 1, splits, items, 64, &info);
  printf("plan %s %d %d %d %d\n", fd_status_string(s), info.total_items, splits[0], splits[1],
         splits[2]);
  /* the first item: (sequence, KV head, split, key start, key end) */
  printf("item0 %d %d %d %d %d\n", items[0], items[1], items[2], items[3], items[4]);
  /* an argument error returns before any device work, with a message */
  s = fd_split_plan(lens, 3, 0, 4096, 0, 148, 1, NULL, NULL, 0, &info);
  printf("bad %s %d\n", fd_status_string(s), (int)(strlen(fd_last_error_message()) > 0));
  /* a decode call whose q is NULL is refused on the host */
  s = fd_decode_attention(NULL, NULL, NULL, NULL, 0, NULL, NULL, NULL);
  printf("decode %s\n", fd_status_string(s));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_abi():
    lib = os.path.join(PKG, "libfd.so")
    assert os.path.exists(lib), "build libfd.so first"
    work = os.path.join(ROOT, "_build", "c_abi_test")   # build products, ignored by git
    os.makedirs(work, exist_ok=True)
    src = os.path.join(work, "abi.c")
    with open(src, "w") as f:
        f.write(C_SRC)
    exe = os.path.join(work, "abi")
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                         str(src), "-L", PKG, "-lfd", "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    env = dict(os.environ, LD_LIBRARY_PATH=PKG + os.pathsep + os.environ.get("LD_LIBRARY_PATH", ""))
    run = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=60)
    assert run.returncode == 0, run.stderr
    out = dict((l.split()[0], l.split()[1:]) for l in run.stdout.splitlines())
    assert out["plan"][0] == "FD_OK"
    # the same plan as the host planner's Python tests: 4096 keys cut into equal splits
    n0 = int(out["plan"][2])
    assert n0 >= 1 and out["plan"][3] == "1" and out["plan"][4] == "1"
    assert int(out["plan"][1]) == 2 * (n0 + 1 + 1)
    assert out["item0"][:3] == ["0", "0", "0"] and out["item0"][3] == "0"
    assert out["bad"] == ["FD_ERR_INVALID_ARGUMENT", "1"]
    assert out["decode"] == ["FD_ERR_INVALID_ARGUMENT"]
