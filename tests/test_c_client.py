"""The boundary from plain C: a C99 program that includes only
include/sparse_attn.h and links only libsparse_attn.so sizes the workspaces
of every configuration's policy, gets a host-side argument error and its
message, all without a GPU. It shows the header is plain C (no C++ or torch
types) and that the library's exported names are the header's."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "sparse_attention_video_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "sparse_attn.h"

int main(void) {
  sa_problem pr;
  sa_policy po;
  size_t mask = 0, scratch = 0;
  memset(&pr, 0, sizeof pr);
  memset(&po, 0, sizeof po);
  pr.batch = 1; pr.heads = 12; pr.T = 21; pr.H = 30; pr.W = 52; pr.head_dim = 128;
  po.kind = SA_MASK_STA; po.block = 128;
  po.tile[0] = 4; po.tile[1] = 4; po.tile[2] = 8;
  po.window[0] = 3; po.window[1] = 3; po.window[2] = 3;
  int e = sparse_attn_workspace_size(&pr, &po, &mask, &scratch);
  printf("sta %d %zu %zu\n", e, mask, scratch);
  po.window[0] = 2;                                   /* even window: refused */
  e = sparse_attn_workspace_size(&pr, &po, &mask, &scratch);
  printf("even %d %s\n", e, sparse_attn_strerror(e));
  e = sparse_attn_forward(&pr, &po, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL);
  printf("null %d\n", e);
  return 0;
}
"""


def test_plain_c_client_links_and_sizes_workspaces(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = os.path.join(LIBDIR, "libsparse_attn.so")
    assert os.path.exists(lib), "build the library first (build.py)"
    src = tmp_path / "client.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "client"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", LIBDIR, "-lsparse_attn", "-Wl,-rpath," + LIBDIR], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    sta = out[0].split()
    assert sta[0] == "sta" and sta[1] == "0" and int(sta[2]) > 0 and int(sta[3]) > 0, out
    even = out[1].split(maxsplit=2)
    assert even[0] == "even" and int(even[1]) != 0 and len(even[2]) > 0, out
    null = out[2].split()
    assert null[0] == "null" and int(null[1]) != 0, out
