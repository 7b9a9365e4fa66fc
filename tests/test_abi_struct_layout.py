"""The C structs of include/stq.h and the Python binding's ctypes mirrors agree field by
field (offsets and sizes), checked by compiling a small C program against the header
with the host compiler (no GPU)."""
import ctypes
import os
import shutil
import subprocess

import pytest

from quantized_linear_attention_02_b200 import stq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stddef.h>
#include <stdio.h>
#include "stq.h"
#define F(T, f) printf(#T " " #f " %zu %zu\n", offsetof(T, f), sizeof(((T*)0)->f))
int main(void) {
  printf("stq_pool_desc size %zu\n", sizeof(stq_pool_desc));
  F(stq_pool_desc, kind); F(stq_pool_desc, n_slots); F(stq_pool_desc, H); F(stq_pool_desc, d);
  F(stq_pool_desc, unit_bits); F(stq_pool_desc, omega); F(stq_pool_desc, scheme);
  F(stq_pool_desc, scale_bits);
  printf("stq_pool_sizes size %zu\n", sizeof(stq_pool_sizes));
  F(stq_pool_sizes, codes_bytes); F(stq_pool_sizes, scales_bytes); F(stq_pool_sizes, pivots_bytes);
  F(stq_pool_sizes, meta_bytes); F(stq_pool_sizes, slot_code_bytes); F(stq_pool_sizes, n_pivot_rows);
  F(stq_pool_sizes, max_head_bytes);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a host C compiler")
def test_ctypes_mirrors_match_the_header(tmp_path):
    src = tmp_path / "layout.c"
    exe = tmp_path / "layout"
    src.write_text(PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    lines = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    c_sizes, c_fields = {}, {}
    for ln in lines:
        parts = ln.split()
        if parts[1] == "size":
            c_sizes[parts[0]] = int(parts[2])
        else:
            c_fields[(parts[0], parts[1])] = (int(parts[2]), int(parts[3]))
    for cname, py in (("stq_pool_desc", stq._Desc), ("stq_pool_sizes", stq._Sizes)):
        assert ctypes.sizeof(py) == c_sizes[cname], cname
        for fname, ftype in py._fields_:
            off = getattr(py, fname).offset
            assert (off, ctypes.sizeof(ftype)) == c_fields[(cname, fname)], (cname, fname)
        assert len(py._fields_) == sum(1 for k in c_fields if k[0] == cname), cname
