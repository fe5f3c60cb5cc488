"""The binding's ctypes structures agree with the C header field by field: a host C
compiler builds a program against include/csa2.h that prints each struct's size and
every field's offset, and the ctypes layout must match (no GPU, no CUDA)."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _c_layout(tmp_path, structs):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "csa2.h"', "int main(void) {"]
    for cname, fields in structs:
        lines.append(f'    printf("{cname} size %zu\\n", sizeof({cname}));')
        for f in fields:
            lines.append(f'    printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    table = {}
    for line in out.splitlines():
        cname, key, value = line.split()
        table[(cname, key)] = int(value)
    return table


def test_struct_layouts_match_the_header(tmp_path):
    from __graft_entry__ import build
    build()
    from fp4_kv_cache_04_b200 import csa2
    pairs = [("csa2_index_args", csa2.IndexArgs), ("csa2_layer_args", csa2.LayerArgs)]
    table = _c_layout(tmp_path, [(c, [f for f, _ in py._fields_]) for c, py in pairs])
    import ctypes
    for cname, py in pairs:
        assert table[(cname, "size")] == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert table[(cname, f)] == getattr(py, f).offset, f"{cname}.{f}"


def test_noalloc_scratch_constant_matches_the_header(tmp_path):
    """The binding's NOALLOC_POOL_SCRATCH_BYTES is the header's macro, read by a host C
    build of include/csa2.h (the GPU test sizes its calls from the Python constant)."""
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    src = tmp_path / "macro.c"
    src.write_text('#include <stdio.h>\n#include "csa2.h"\n'
                   'int main(void) { printf("%llu\\n", (unsigned long long)CSA2_NOALLOC_POOL_SCRATCH_BYTES); '
                   'return 0; }\n')
    exe = tmp_path / "macro"
    subprocess.run([cc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe)], check=True, capture_output=True)
    value = int(subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout)
    from __graft_entry__ import build
    build()
    from fp4_kv_cache_04_b200 import csa2
    assert value == csa2.NOALLOC_POOL_SCRATCH_BYTES
