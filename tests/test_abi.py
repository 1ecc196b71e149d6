"""C-ABI checks that need no GPU: the library loads, exports every function
that include/muon.h declares, the ctypes structs match the C layout, and
host-side validation rejects bad arguments before any launch."""

import ctypes as C
import os
import re
import subprocess

import pytest

from newton_schulz_10_b200 import build as nbuild
from newton_schulz_10_b200 import muon as mu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "muon.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(mu.LIB_PATH):
        nbuild.build()
    return mu.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_exports_every_declared_function(L):
    names = declared_functions()
    assert len(names) >= 12, names
    out = subprocess.run(["nm", "-D", "--defined-only", mu.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if " T " in line)
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)
    assert set(mu.EXPORTS) == set(names)


def test_struct_layout_matches_c(tmp_path):
    src = tmp_path / "sizes.c"
    src.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "muon.h"\n'
        "int main(void){printf(\"%zu %zu %zu %zu %zu %zu\\n\", sizeof(muon_ns_params), sizeof(muon_matrix),"
        " sizeof(muon_params), offsetof(muon_params, ns), offsetof(muon_params, dev_status),"
        " offsetof(muon_ns_params, compute)); return 0;}\n")
    exe = tmp_path / "sizes"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()))
    want = [C.sizeof(mu.NsParams), C.sizeof(mu.Matrix), C.sizeof(mu.Params), mu.Params.ns.offset,
            mu.Params.dev_status.offset, mu.NsParams.compute.offset]
    assert got == want


def test_status_strings(L):
    for code in range(10):
        assert mu.status_str(code).startswith("MUON_")
    assert mu.status_str(1234) == "MUON_ERR_UNKNOWN"


def test_rows_for_fraction(L):
    assert mu.rows_for_fraction(8192, 1, 4) == 2048
    assert mu.rows_for_fraction(10, 1, 3) == 4
    assert mu.rows_for_fraction(7, 1, 1) == 7
    assert mu.rows_for_fraction(7, 2, 1) == -1
    assert mu.rows_for_fraction(7, 0, 1) == -1


def test_default_params(L):
    p = mu.ns_params()
    assert p.T == 5 and p.restart_at == 3 and p.compute == mu.BF16
    assert abs(p.coeffs[4][0] - 3.4445) < 1e-6 and abs(p.coeffs[0][1] + 4.775) < 1e-6
    assert abs(p.norm_eps - 1e-7) < 1e-12


FAKE = 1 << 20  # a 16-byte aligned non-NULL address; never dereferenced on these paths


def test_polar_validation(L):
    p = mu.ns_params()
    ws = mu.ns_workspace_size(64, 256, p)
    assert ws > 64 * 256 * 2 * 2
    call = lambda X, O, xd, od, r, c, pp, w, nb: L.ns_polar(X, xd, O, od, r, c, C.byref(pp), w, nb, None)
    assert call(None, FAKE, mu.F32, mu.F32, 64, 256, p, FAKE, ws) == mu.ERR_INVALID_ARG
    assert call(FAKE, FAKE, mu.F16, mu.F32, 64, 256, p, FAKE, ws) == mu.ERR_DTYPE
    assert call(FAKE + 4, FAKE, mu.F32, mu.F32, 64, 256, p, FAKE, ws) == mu.ERR_ALIGN
    assert call(FAKE, FAKE, mu.F32, mu.F32, 64, 256, p, FAKE, 4096) == mu.ERR_WORKSPACE
    assert call(FAKE, FAKE, mu.F32, mu.F32, 64, 256, p, None, ws) == mu.ERR_WORKSPACE
    assert call(FAKE, FAKE, mu.F32, mu.F32, -1, 256, p, FAKE, ws) == mu.ERR_SHAPE
    assert call(None, None, mu.F32, mu.F32, 0, 256, p, None, 0) == mu.OK  # empty: nothing to do
    bad = mu.ns_params(T=0)
    assert call(FAKE, FAKE, mu.F32, mu.F32, 64, 256, bad, FAKE, ws) == mu.ERR_INVALID_ARG
    bad = mu.ns_params(T=mu.MAX_T + 1)
    assert call(FAKE, FAKE, mu.F32, mu.F32, 64, 256, bad, FAKE, ws) == mu.ERR_INVALID_ARG
    bad = mu.ns_params()
    bad.compute = 7
    assert call(FAKE, FAKE, mu.F32, mu.F32, 64, 256, bad, FAKE, ws) == mu.ERR_DTYPE
    assert mu.ns_workspace_size(64, 256, bad) == 0


def test_step_validation(L):
    mats = (mu.Matrix * 2)()
    mats[0] = mu.Matrix(FAKE, FAKE, FAKE, None, 32, 64)
    mats[1] = mu.Matrix(FAKE, FAKE, FAKE, None, 64, 32)
    p = mu.step_params()
    n = L.muon_workspace_size(mats, 2, C.byref(p))
    assert n > 0
    assert L.muon_step(mats, 2, C.byref(p), FAKE, n - 1, None) == mu.ERR_WORKSPACE
    assert L.muon_step(mats, 2, C.byref(p), None, n, None) == mu.ERR_WORKSPACE
    assert L.muon_step(mats, -1, C.byref(p), FAKE, n, None) == mu.ERR_INVALID_ARG
    pn = mu.step_params(normuon=True)  # NorMuon needs v
    assert L.muon_step(mats, 2, C.byref(pn), FAKE, n, None) == mu.ERR_INVALID_ARG
    pd = mu.step_params(dion3=True, frac=(3, 2))
    assert L.muon_step(mats, 2, C.byref(pd), FAKE, n, None) == mu.ERR_INVALID_ARG
    mis = (mu.Matrix * 1)()
    mis[0] = mu.Matrix(FAKE + 8, FAKE, FAKE, None, 32, 64)
    assert L.muon_step(mis, 1, C.byref(p), FAKE, n, None) == mu.ERR_ALIGN
    empty = (mu.Matrix * 1)()
    empty[0] = mu.Matrix(None, None, None, None, 0, 64)
    assert L.muon_step(empty, 1, C.byref(p), None, 0, None) == mu.OK
    assert L.muon_step(empty, 0, C.byref(p), None, 0, None) == mu.OK


def test_select_and_normuon_validation(L):
    assert L.select_rows(FAKE, 10, 4, 0, 0, FAKE, FAKE, 1 << 20, None) == mu.ERR_SHAPE
    assert L.select_rows(FAKE, 10, 4, 11, 0, FAKE, FAKE, 1 << 20, None) == mu.ERR_SHAPE
    assert L.select_rows(FAKE, 10, 4, 3, 5, FAKE, FAKE, 1 << 20, None) == mu.ERR_INVALID_ARG
    assert L.select_rows(FAKE, 10, 4, 3, 0, FAKE, FAKE, 8, None) == mu.ERR_WORKSPACE
    assert L.normuon_scale(FAKE, mu.F16, 4, 8, FAKE, None, 0.95, 1e-8, FAKE, None, None) == mu.ERR_DTYPE
    assert L.normuon_scale(FAKE, mu.F32, 4, 8, None, None, 0.95, 1e-8, FAKE, None, None) == mu.ERR_INVALID_ARG
    assert L.normuon_scale(None, mu.F32, 0, 8, None, None, 0.95, 1e-8, None, None, None) == mu.OK


def test_workspace_grows_with_batch(L):
    p = mu.step_params()
    one = (mu.Matrix * 1)()
    one[0] = mu.Matrix(FAKE, FAKE, FAKE, None, 768, 768)
    four = (mu.Matrix * 4)()
    for i in range(4):
        four[i] = mu.Matrix(FAKE, FAKE, FAKE, None, 768, 768)
    a = L.muon_workspace_size(one, 1, C.byref(p))
    b = L.muon_workspace_size(four, 4, C.byref(p))
    assert b > 3 * (a - 4096)
