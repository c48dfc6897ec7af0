"""The C ABI library loads and exports every entry point its header declares.
No compute calls: this runs without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tdm.h")
LIB = os.path.join(ROOT, "tiled_distance_maps_b200", "libtdm.so")


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tdm_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        import __graft_entry__
        __graft_entry__._build_module().build(quiet=True)
    return ctypes.CDLL(LIB)


def test_header_declares_the_boundary():
    names = declared()
    for need in ("tdm_init_schedule", "tdm_ddim_step", "tdm_ddim_run", "tdm_seam_project", "tdm_mds_recover",
                 "tdm_pairwise_dist", "tdm_seam_discrepancy", "tdm_eps_standin", "tdm_init_noise"):
        assert need in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared() if not hasattr(lib, n)]
    assert not missing, missing
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (tdm_[a-z0-9_]+)\b", out))
    assert set(declared()) <= exported


def test_binding_covers_the_header():
    import tiled_distance_maps_b200 as tdm
    assert set(declared()) == set(tdm.EXPORTED)


def test_status_strings_need_no_device(lib):
    lib.tdm_status_str.restype = ctypes.c_char_p
    assert lib.tdm_status_str(0) == b"ok"
    assert lib.tdm_status_str(1) == b"invalid argument"
    assert lib.tdm_status_str(7) == b"eigen-solve did not converge"
    assert lib.tdm_status_str(99) == b"unknown status"


def test_null_context_is_rejected_before_any_cuda_call(lib):
    # argument checks come first: a NULL context returns TDM_EINVAL
    assert lib.tdm_ddim_run(None, None, None, None, ctypes.c_float(0), ctypes.c_float(0), ctypes.c_float(0),
                            ctypes.c_uint64(0), 1, None, None) == 1
    assert lib.tdm_mds_recover(None, None, ctypes.c_int64(0), None, None, None) == 1


C_PROG = r"""
#include <stdio.h>
#include <string.h>
#include "tdm.h"
int main(void) {
    /* host-only calls: status strings, argument checks, the cosine table */
    double ab[4];
    if (strcmp(tdm_status_str(TDM_OK), "ok") != 0) return 1;
    if (tdm_ddim_run(NULL, NULL, NULL, NULL, 0.f, 0.f, 0.f, 0u, 1, NULL, NULL) != TDM_EINVAL) return 2;
    if (tdm_cosine_alphas_bar(4, 0.008, ab) != TDM_OK) return 3;
    if (!(ab[0] < 1.0 && ab[3] < ab[2] && ab[3] > 0.0)) return 4;
    if (tdm_cosine_alphas_bar(0, 0.008, ab) != TDM_EINVAL) return 5;
    printf("%.17g\n", ab[1]);
    return 0;
}
"""


def test_header_is_c99_and_links_from_c(tmp_path):
    # the boundary is plain C: the header compiles as strict C99 and a C
    # program links against the library and calls its host entry points
    src = tmp_path / "abi.c"
    src.write_text(C_PROG)
    exe = tmp_path / "abi"
    inc = os.path.join(ROOT, "include")
    libdir = os.path.dirname(LIB)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", inc, str(src), "-o", str(exe),
                    "-L", libdir, "-ltdm", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out
    from oracle.schedule import cosine_alphas_bar
    assert abs(float(out.stdout) - cosine_alphas_bar(4, 0.008)[1]) <= 1e-15
