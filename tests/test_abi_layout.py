"""The host structs of include/csla.h, compiled by the C compiler, against
the ctypes mirrors in the Python binding: same size, same field offsets.
(A field added on one side only would shift every later argument.)"""
import ctypes
import os
import shutil
import subprocess
import tempfile

import pytest

from conftest import ROOT

STRUCTS = ("csla_cfg", "csla_cache", "csla_state", "csla_compress_params", "csla_queries", "csla_token_rows")


def _c_layout():
    from compressed_sparse_long_append_b200 import csla as C
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "csla.h"', "int main(void) {"]
    for name in STRUCTS:
        lines.append('printf("%s size %%zu\\n", sizeof(%s));' % (name, name))
        for field, _ in getattr(C, name)._fields_:
            lines.append('printf("%s.%s %%zu\\n", offsetof(%s, %s));' % (name, field, name, field))
    lines += ["return 0;", "}"]
    with tempfile.TemporaryDirectory() as d:
        src, exe = os.path.join(d, "layout.c"), os.path.join(d, "layout")
        with open(src, "w") as f:
            f.write("\n".join(lines))
        subprocess.run([cc, "-I", os.path.join(ROOT, "include"), "-o", exe, src], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    return dict(line.rsplit(" ", 1) for line in out.splitlines())


def test_ctypes_structs_match_the_header():
    from compressed_sparse_long_append_b200 import csla as C
    got = _c_layout()
    for name in STRUCTS:
        S = getattr(C, name)
        assert int(got["%s size" % name]) == ctypes.sizeof(S), name
        for field, _ in S._fields_:
            assert int(got["%s.%s" % (name, field)]) == getattr(S, field).offset, (name, field)
