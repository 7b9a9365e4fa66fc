"""The C structs of include/stq.h and the Python binding's ctypes mirrors agree field by
field (offsets and sizes), checked by compiling a small C program against the header
with the host compiler (no GPU); and a plain C program links the library and calls it."""
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


CALLER = r"""
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#include "stq.h"
int main(void) {
  uint8_t bits[2] = {6, 16};
  float omega[2 * STQ_D];
  for (int i = 0; i < 2 * STQ_D; ++i) omega[i] = 1.0f;
  stq_pool_desc d;
  memset(&d, 0, sizeof d);
  d.kind = STQ_GDN; d.n_slots = 3; d.H = 2; d.d = STQ_D; d.unit_bits = bits; d.omega = omega;
  stq_pool_sizes s;
  stq_status st = stq_pool_layout(&d, &s);
  printf("version %s\n", stq_version());
  printf("ok %d %zu %zu %zu %d\n", (int)st, s.codes_bytes, s.scales_bytes, s.pivots_bytes, s.n_pivot_rows);
  bits[0] = 5;                                   /* not a width */
  st = stq_pool_layout(&d, &s);
  printf("bad %d %s\n", (int)st, stq_last_error());
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a host C compiler")
def test_plain_c_caller(tmp_path):
    # the library as a C program uses it: no Python, no torch in the process
    from quantized_linear_attention_02_b200 import build
    build.build()
    libdir = os.path.dirname(os.path.abspath(stq.__file__))
    src = tmp_path / "caller.c"
    exe = tmp_path / "caller"
    src.write_text(CALLER)
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lstq", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    assert out[0].startswith("version ") and "sm_100a" in out[0]
    ok = out[1].split()
    assert ok[1] == "0"
    # 3 slots: one 6-bit head (128 rows x 96 B) and one FP16 pivot head (128 rows)
    assert int(ok[2]) == 3 * 128 * 96
    assert int(ok[3]) == 3 * 2 * 2 * 128 * 4
    assert int(ok[4]) == 3 * 128 * 128 * 2 and int(ok[5]) == 128
    bad = out[2].split(maxsplit=2)
    assert bad[1] == "1" and len(bad) == 3 and bad[2]     # STQ_ERR_INVALID_ARG with a message


def test_static_staging_size_matches_header():
    import re
    txt = open(os.path.join(ROOT, "include", "stq.h")).read()
    m = re.search(r"#define\s+STQ_STATIC_STAGING_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", txt)
    assert m, "STQ_STATIC_STAGING_BYTES not found in include/stq.h"
    assert int(m.group(1)) << int(m.group(2)) == stq.STATIC_STAGING_BYTES
