"""The Python binding's ctypes structures match include/moe.h field for field (names,
offsets, sizes), checked by compiling a C program against the header (CPU only)."""
import ctypes
import os
import shutil
import subprocess
import tempfile

import pytest

import routing_grouped_expert_softmax_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STRUCTS = {
    "moe_config": (moe.MoeConfig, ["T", "d", "E", "k", "f", "dtype", "prec"]),
    "moe_layer_weights": (moe.LayerWeights, list(moe.WEIGHT_FIELDS)),
    "moe_layer_saved": (moe.LayerSaved, list(moe.SAVED_FIELDS)),
    "moe_layer_grads": (moe.LayerGrads, list(moe.GRAD_FIELDS)),
}


def _cc():
    for c in ("gcc", "cc"):
        if shutil.which(c):
            return c
    return None


@pytest.mark.skipif(_cc() is None, reason="needs a C compiler")
def test_ctypes_structures_match_the_header():
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "moe.h"', "int main(void) {"]
    for cname, (_, fields) in STRUCTS.items():
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for f in fields:
            lines.append(f'  printf("{cname} {f} %zu %zu\\n", offsetof({cname}, {f}), sizeof((({cname} *)0)->{f}));')
    lines += ["  return 0;", "}"]
    with tempfile.TemporaryDirectory() as tmp:
        src, exe = os.path.join(tmp, "layout.c"), os.path.join(tmp, "layout")
        with open(src, "w") as fh:
            fh.write("\n".join(lines))
        r = subprocess.run([_cc(), "-I", os.path.join(ROOT, "include"), src, "-o", exe], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    c = {}
    for line in out:
        parts = line.split()
        if len(parts) == 3 and parts[1] == "sizeof":
            c[(parts[0], "sizeof")] = int(parts[2])
        elif len(parts) == 4:
            c[(parts[0], parts[1])] = (int(parts[2]), int(parts[3]))
    for cname, (cls, fields) in STRUCTS.items():
        assert [f[0] for f in cls._fields_] == fields, cname
        assert ctypes.sizeof(cls) == c[(cname, "sizeof")], cname
        for f in fields:
            desc = getattr(cls, f)
            assert (desc.offset, desc.size) == c[(cname, f)], (cname, f)


def _prototypes():
    """name -> number of parameters, from the MOE_API declarations in moe.h."""
    import re
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(([^)]*)\)\s*;", src):
        params = [p for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(1)] = len(params)
    return out


def test_binding_signatures_match_the_prototypes():
    lib = moe.lib() if os.path.exists(moe.LIB_PATH) else None
    if lib is None:
        pytest.skip("library not built")
    protos = _prototypes()
    assert sorted(protos) == sorted(moe.EXPORTED)
    for name, n in protos.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None and len(fn.argtypes) == n, (name, n, fn.argtypes)
