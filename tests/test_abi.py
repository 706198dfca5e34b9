"""The C-ABI library builds for sm_100a, loads without a GPU, exports every
symbol that include/mhc_birkhoff.h declares, and validates arguments on the
host before touching CUDA.  No call here launches a kernel."""
import ctypes
import os
import re

import pytest

from doubly_stochastic_projection_b200 import build

HEADER = os.path.join(build.ROOT, "include", "mhc_birkhoff.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MHC_API\s+[\w\s\*]*?\b(mhc_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("mhc_birkhoff_fwd", "mhc_birkhoff_bwd", "mhc_residual_mix_fwd", "mhc_residual_mix_bwd",
              "mhc_proj_mix_fwd", "mhc_proj_mix_bwd", "mhc_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    import subprocess
    out = subprocess.check_output(["nm", "-D", "--defined-only", build.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        getattr(L, n)  # resolvable through the dynamic loader


def test_host_only_calls(L):
    L.mhc_status_string.restype = ctypes.c_char_p
    L.mhc_status_string.argtypes = [ctypes.c_int]
    assert L.mhc_status_string(0) == b"MHC_OK"
    assert b"ALIGN" in L.mhc_status_string(2)
    assert L.mhc_status_string(99) == b"unknown mhc status"
    assert L.mhc_version() >= 100


def test_validation_rejects_before_any_cuda_call(L):
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.mhc_birkhoff_fwd.argtypes = [p, p, i64, i32, i32, p]
    L.mhc_residual_mix_fwd.argtypes = [p, p, p, p, p, i64, i64, p]
    L.mhc_birkhoff_bwd.argtypes = [p, p, p, p, i64, p]
    fake = 1 << 20  # never dereferenced: every call below returns before launching
    assert L.mhc_birkhoff_fwd(fake, fake, -5, 1, 0, None) == 3
    assert L.mhc_birkhoff_fwd(fake, fake, 10, 4, 0, None) == 4
    assert L.mhc_birkhoff_fwd(fake, fake, 10, 0, -1, None) == 4
    assert L.mhc_birkhoff_fwd(fake, fake, 10, 1, 1001, None) == 4
    assert L.mhc_birkhoff_fwd(None, fake, 10, 1, 0, None) == 1
    assert L.mhc_birkhoff_fwd(fake + 4, fake, 10, 1, 0, None) == 2
    assert L.mhc_birkhoff_fwd(None, None, 0, 1, 0, None) == 0      # empty batch: nothing to do
    assert L.mhc_birkhoff_bwd(None, None, fake, fake, 3, None) == 1
    assert L.mhc_residual_mix_fwd(fake, fake, fake, fake, fake, 4, 12, None) == 3
    assert L.mhc_residual_mix_fwd(fake, fake, fake, fake, fake, 4, 0, None) == 3
    assert L.mhc_residual_mix_fwd(fake, fake, fake, fake, fake + 8, 4, 16, None) == 2
    assert L.mhc_residual_mix_fwd(None, None, None, None, None, 0, 16, None) == 0
    L.mhc_birkhoff_fwd_n.argtypes = [p, p, i64, i32, i32, i32, p]
    assert L.mhc_birkhoff_fwd_n(fake, fake, 10, 9, 1, 0, None) == 3
    assert L.mhc_birkhoff_fwd_n(fake, fake, 10, 5, 2, 0, None) == 4
    assert L.mhc_birkhoff_fwd_n(None, None, 0, 5, 1, 0, None) == 0


def test_validation_of_the_remaining_entry_points(L):
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    fake = 1 << 20  # never dereferenced: every call below returns before launching
    L.mhc_birkhoff_fwd_n.argtypes = [p, p, i64, i32, i32, i32, p]
    L.mhc_birkhoff_bwd_n.argtypes = [p, p, p, i64, i32, p]
    assert L.mhc_birkhoff_fwd_n(fake, fake, 10, 0, 1, 0, None) == 3
    assert L.mhc_birkhoff_bwd_n(fake, fake, fake, 10, 9, None) == 3
    assert L.mhc_birkhoff_bwd_n(fake, None, fake, 10, 3, None) == 1
    L.mhc_composite_gain.argtypes = [p, p, p, p, i64, i64, p]
    assert L.mhc_composite_gain(fake, None, fake, fake, 0, 10, None) == 3        # L >= 1
    assert L.mhc_composite_gain(fake, None, fake, fake, 2, -1, None) == 3
    assert L.mhc_composite_gain(fake, None, fake, fake, (1 << 20) + 1, 10, None) == 3
    assert L.mhc_composite_gain(None, None, fake, fake, 2, 10, None) == 1
    assert L.mhc_composite_gain(fake + 4, None, fake, fake, 2, 10, None) == 2
    assert L.mhc_composite_gain(fake, None, fake + 4, fake, 2, 10, None) == 2     # gain_rows
    assert L.mhc_composite_gain(fake, None, fake, fake + 8, 2, 10, None) == 2     # gain_cols
    assert L.mhc_composite_gain(None, None, None, None, 2, 0, None) == 0       # no tokens
    L.mhc_exp_shifted.argtypes = [p, p, i64, p]
    assert L.mhc_exp_shifted(fake, fake, -1, None) == 3
    assert L.mhc_exp_shifted(None, fake, 10, None) == 1
    assert L.mhc_exp_shifted(None, None, 0, None) == 0
    assert L.mhc_exp_shifted(fake + 1, fake, 10, None) == 2                      # odd byte offset
    assert L.mhc_exp_shifted(fake, fake + 2, 10, None) == 2
    L.mhc_premap_bwd.argtypes = [p, p, p, p, p, i32, i64, i64, p]
    assert L.mhc_premap_bwd(fake, fake, fake, fake, fake, 2, 4, 16, None) == 4     # accumulate is 0 or 1
    L.mhc_birkhoff_fwd_layout.argtypes = [p, p, i64, i32, i32, i32, p]
    assert L.mhc_birkhoff_fwd_layout(fake, fake, 10, 1, 0, 4, None) == 4          # unknown layout
    assert L.mhc_birkhoff_fwd_layout(fake, fake, 10, 0, 0, 3, None) == 4          # lane pair is Newton only
    assert L.mhc_birkhoff_fwd_layout(fake, fake, 10, 0, 0, 2, None) == 4          # row group is Newton only
    assert L.mhc_birkhoff_fwd_layout(fake, fake, -1, 1, 0, 2, None) == 3
    assert L.mhc_birkhoff_fwd_layout(None, fake, 10, 1, 0, 2, None) == 1
    assert L.mhc_birkhoff_fwd_layout(fake + 4, fake, 10, 1, 0, 2, None) == 2
    L.mhc_birkhoff_fwd_bwd_host.argtypes = [p, p, p, p, p, p, p, p, i64, i32, p]
    assert L.mhc_birkhoff_fwd_bwd_host(*[fake] * 8, -1, 4, None) == 3
    assert L.mhc_birkhoff_fwd_bwd_host(*[fake] * 8, 10, 0, None) == 4            # pieces >= 1
    assert L.mhc_birkhoff_fwd_bwd_host(*[fake] * 8, 10, 65, None) == 4           # pieces <= 64
    assert L.mhc_birkhoff_fwd_bwd_host(*[None] * 8, 0, 4, None) == 0             # nothing to do
    assert L.mhc_birkhoff_fwd_bwd_host(None, *[fake] * 7, 10, 4, None) == 1
    assert L.mhc_birkhoff_fwd_bwd_host(*[fake] * 7, fake + 4, 10, 4, None) == 2
    L.mhc_birkhoff_fwd_bwd_mapped.argtypes = [p, p, p, p, p, i64, p]
    assert L.mhc_birkhoff_fwd_bwd_mapped(*[fake] * 5, -1, None) == 3
    assert L.mhc_birkhoff_fwd_bwd_mapped(*[None] * 5, 0, None) == 0
    assert L.mhc_birkhoff_fwd_bwd_mapped(fake, fake, fake, fake, None, 10, None) == 1
    assert L.mhc_birkhoff_fwd_bwd_mapped(fake, fake, fake + 8, fake, fake, 10, None) == 2
    L.mhc_residual_mix_bwd.argtypes = [p, p, p, p, p, p, p, p, p, p, i64, i64, p]
    assert L.mhc_residual_mix_bwd(fake, fake, fake, fake, fake, fake, None, None, fake, None, 1 << 36, 1 << 24,
                                  None) == 3                                    # T * 4 * C above 2^40


def test_validation_of_the_no_alloc_entry_point(L):
    p, i64 = ctypes.c_void_p, ctypes.c_int64
    fake = 1 << 20  # never dereferenced: every call below returns before any CUDA call
    cap = int(re.search(r"#define\s+MHC_NOALLOC_MAX_MATS\s+(\d+)", open(HEADER).read()).group(1))
    f = L.mhc_birkhoff_fwd_bwd_mapped_static
    f.argtypes = [p, p, p, p, i64, p]
    assert f(*[fake] * 4, cap + 1, None) == 3                                    # beyond the fixed array
    assert f(*[fake] * 4, -1, None) == 3
    assert f(*[None] * 4, 0, None) == 0
    assert f(fake, fake, None, fake, 10, None) == 1
    assert f(fake, fake, fake, fake + 8, 10, None) == 2


def test_header_is_plain_c(tmp_path):
    # the boundary is usable from C: the header compiles as strict C99 and a C
    # program links the library and runs a host-only call
    import shutil
    import subprocess

    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "t.c"
    src.write_text('#include <stdio.h>\n#include "mhc_birkhoff.h"\n'
                   "int main(void) {\n"
                   "    if (mhc_version() < 100) return 2;\n"
                   "    return mhc_birkhoff_fwd(NULL, NULL, -1, MHC_NEWTON, 0, NULL) == MHC_ERR_SIZE ? 0 : 1;\n"
                   "}\n")
    inc = os.path.join(build.ROOT, "include")
    libdir = os.path.dirname(build.LIB_PATH)
    exe = tmp_path / "t"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, str(src),
                           "-L", libdir, "-lmhc_b200", "-Wl,-rpath," + libdir, "-o", str(exe)])
    assert subprocess.call([str(exe)]) == 0


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    # no CPU or torch fallback: a missing library is an error, not a slow path
    from doubly_stochastic_projection_b200 import api

    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api._build, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        api.lib()
