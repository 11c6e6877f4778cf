"""The boundary as a plain C caller sees it (no GPU): ``include/fa.h`` compiles
as strict C99 and as C++17 without warnings, every entry point it declares
links against the built library under its unmangled name, and a C program
gets the documented status for a call with an invalid argument (no CUDA call
is made for it)."""

import os
import shutil
import subprocess
import tempfile

import pytest

from tests.test_abi_cpu import ROOT, _declared_functions

LIBDIR = os.path.join(ROOT, "exact_io_aware_49_b200")


@pytest.fixture(scope="module")
def built():
    from exact_io_aware_49_b200 import build
    build.build()
    tmp = tempfile.mkdtemp(prefix="fa_cabi_")
    yield tmp
    shutil.rmtree(tmp, ignore_errors=True)


def _program(names):
    refs = ",\n    ".join(f"(fa_fn)&{n}" for n in names)
    return f"""#include "fa.h"
#include <stdio.h>

typedef void (*fa_fn)(void);

int main(void) {{
  fa_fn all[] = {{
    {refs}
  }};
  /* null pointers: rejected before any CUDA call */
  fa_status st = fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 64, 1, 0.125f, 0.0f, 0, NULL);
  printf("%d %d %zu %s\\n", (int)(sizeof(all) / sizeof(all[0])), (int)st,
         fa_bwd_workspace_size(1, 2, 256, 128), fa_status_string(st));
  return 0;
}}
"""


@pytest.mark.parametrize("lang", ["c99", "c++17"])
def test_header_compiles_links_and_reports_status(built, lang):
    names = _declared_functions()
    src = os.path.join(built, "caller.c" if lang == "c99" else "caller.cpp")
    exe = os.path.join(built, f"caller_{lang.replace('+', 'p')}")
    with open(src, "w") as f:
        f.write(_program(names))
    cc = ["gcc", "-std=c99"] if lang == "c99" else ["g++", "-std=c++17"]
    subprocess.run(cc + ["-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), src,
                         "-o", exe, "-L", LIBDIR, "-lfa_sm100", f"-Wl,-rpath,{LIBDIR}"], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split(maxsplit=3)
    assert int(out[0]) == len(names)
    assert int(out[1]) == 1  # FA_ERR_INVALID_ARG
    assert int(out[2]) > 0
    assert out[3].startswith("FA_ERR_INVALID_ARG")
