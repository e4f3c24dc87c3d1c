"""CPU checks of the C ABI: the library loads, exports every symbol that
include/mpq.h declares, and rejects bad arguments before touching the GPU."""
import ctypes as C
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mpq():
    from post_weight_quantization_row_b200 import _lib
    return _lib


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "mpq.h")).read()
    return sorted(set(re.findall(r"^MPQ_API\s+[\w\s\*]+?\b(mpq_\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_abi():
    syms = declared_symbols()
    assert "mpq_solve" in syms and "mpq_plan_create_from_x" in syms
    assert len(syms) >= 18


def test_library_exports_every_declared_symbol(mpq):
    for name in declared_symbols():
        assert hasattr(mpq.lib, name), name
    assert set(declared_symbols()) == set(mpq.EXPORTED)


def test_params_default(mpq):
    p = mpq.Params()
    mpq.lib.mpq_params_default(C.byref(p), 1, 8)
    assert p.d == 1 and p.K == 8 and p.beta0 == 1.0 and p.damping == 0.5
    assert p.tau == 0.2 and p.gamma_lo_rel == 1e-10 and p.gamma_hi_rel == 1e10
    assert p.alpha_min == 1e-10 and p.alpha_max == 0.99
    assert p.vec_engine == 0 and p.cd_panel == 0 and p.solve_graphs == 1 and p.group_size == 0
    assert p.cd_skip_precision == 0.0
    assert p.greedy_init == 0 and p.greedy_damp == 0.01


@pytest.mark.parametrize("field,value", [("d", 3), ("K", 1), ("damping", 1.5), ("beta0", -1.0),
                                         ("tau", 0.0), ("alpha_max", 1.0), ("vec_engine", 3),
                                         ("cd_panel", 100), ("cd_panel", -128),
                                         ("solve_graphs", 2), ("group_size", 100),
                                         ("group_size", -128), ("cd_skip_precision", -1.0),
                                         ("greedy_init", 2), ("greedy_damp", -0.5),
                                         ("greedy_damp", math.inf)])
def test_bad_params_rejected_without_a_device(mpq, field, value):
    p = mpq.Params()
    mpq.lib.mpq_params_default(C.byref(p), 1, 8)
    setattr(p, field, value)
    h = C.c_void_p()
    dummy = C.c_void_p(16)
    st = mpq.lib.mpq_plan_create_from_spectrum(dummy, dummy, 64, 8, C.byref(p), None, C.byref(h))
    assert st == 1, mpq.lib.mpq_last_error()
    assert h.value is None


def test_null_plan_rejected(mpq):
    assert mpq.lib.mpq_solve(None, None, 0, None, None, 1, 1, None, None, None, None, None) == 1
    assert b"plan" in mpq.lib.mpq_last_error()
    assert mpq.lib.mpq_plan_destroy(None) == 0


def test_codebook_required_for_vector_plans(mpq):
    p = mpq.Params()
    mpq.lib.mpq_params_default(C.byref(p), 8, 16)
    h = C.c_void_p()
    st = mpq.lib.mpq_plan_create_from_spectrum(C.c_void_p(16), C.c_void_p(16), 64, 8, C.byref(p),
                                               None, C.byref(h))
    assert st == 1


def test_streamed_gram_and_rht_reject_bad_arguments_without_a_device(mpq):
    lib, h = mpq.lib, C.c_void_p()
    dummy = C.c_void_p(16)
    assert lib.mpq_gram_create(0, None, C.byref(h)) == 1 and h.value is None
    assert lib.mpq_gram_create(1 << 18, None, C.byref(h)) == 1
    assert lib.mpq_gram_create(64, None, None) == 1
    assert lib.mpq_gram_accumulate(None, dummy, 4, None) == 1
    assert lib.mpq_gram_info(None, None, None) == 1
    assert lib.mpq_gram_get(None, dummy, None) == 1
    assert lib.mpq_gram_destroy(None) == 0
    p = mpq.Params()
    lib.mpq_params_default(C.byref(p), 1, 8)
    assert lib.mpq_plan_create_from_gram(None, C.byref(p), None, C.byref(h)) == 1
    assert h.value is None
    # n not a power of two, above the shared-memory limit, negative rows, NULL X
    for rows, n, x in [(4, 3, dummy), (4, 65536, dummy), (4, 0, dummy), (-1, 64, dummy),
                       (4, 64, None)]:
        assert lib.mpq_rht(x, rows, n, dummy, None) == 1, (rows, n)
    assert "power of two" in lib.mpq_last_error().decode() or "device" in lib.mpq_last_error().decode()


@pytest.mark.parametrize("c_name,py_name", [("mpq_params", "Params"), ("mpq_row_stats", "RowStats")])
def test_struct_layout_matches_the_c_header(mpq, tmp_path, c_name, py_name):
    # the ctypes mirrors of the ABI structs must have the C compiler's size and
    # field offsets, or every call would read shifted fields
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    cls = getattr(mpq, py_name)
    fields = [f[0] for f in cls._fields_]
    src = ['#include <stdio.h>', '#include <stddef.h>', '#include "mpq.h"', "int main(void) {",
           f'  printf("%zu\\n", sizeof({c_name}));']
    src += [f'  printf("%zu\\n", offsetof({c_name}, {f}));' for f in fields]
    src += ["  return 0;", "}"]
    c_file = tmp_path / "layout.c"
    c_file.write_text("\n".join(src) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(c_file), "-o", str(exe)],
                   check=True)
    out = [int(x) for x in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    assert out[0] == C.sizeof(cls)
    assert out[1:] == [getattr(cls, f).offset for f in fields]


def test_binding_argument_counts_match_the_header(mpq):
    # every ctypes signature takes as many arguments as its C declaration
    txt = open(os.path.join(ROOT, "include", "mpq.h")).read()
    decls = re.findall(r"^MPQ_API\s+[\w\s\*]+?\b(mpq_\w+)\s*\(([^;]*?)\)\s*;", txt, flags=re.M | re.S)
    assert len(decls) == len(declared_symbols())
    for name, params in decls:
        params = " ".join(params.split())
        n_c = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(mpq.lib, name).argtypes) == n_c, name
