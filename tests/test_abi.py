"""The C-ABI library loads and exports every entry point its header declares;
host-side validation answers without touching a GPU."""
import ctypes
import os

import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from clustered_sparse_attention_flash_b200.build import build


@pytest.fixture(scope="module")
def L():
    build()
    return sv.lib()


def test_every_header_symbol_is_exported(L):
    names = sv.header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(sv._SIGS), set(names) ^ set(sv._SIGS)


def test_params_struct_matches_header(tmp_path):
    """The ctypes mirror of svgear_params has the C struct's size and field
    offsets (compiled with the host C compiler against the header)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = [n for n, _ in sv.svgear_params._fields_]
    src = tmp_path / "p.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "svgear.h"\nint main(void){printf("%zu", sizeof(svgear_params));'
                   + "".join(f'printf(" %zu", offsetof(svgear_params, {n}));' for n in fields) + "return 0;}\n")
    exe = tmp_path / "p"
    subprocess.run([cc, "-I", os.path.dirname(sv.HEADER), str(src), "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(sv.svgear_params)
    assert got[1:] == [getattr(sv.svgear_params, n).offset for n in fields]


def test_version_and_status_strings(L):
    assert "sm_100a" in sv.svgear_version()
    for code in (0, -1, -2, -3, -4, -5):
        assert sv.status_string(code) != "unknown status"
    assert sv.status_string(42) == "unknown status"


def test_workspace_sizes_are_host_only(L):
    p = sv.params(40, 75600, 75600, 128, 100, 500, 10, 0.15)
    ws = sv.svgear_workspace_size(p)
    assert ws > 3 * 40 * 75600 * 128 * 2
    assert sv.svgear_block_error_workspace_size(p) >= 40 * 100 * 500 * 4
    assert sv.svgear_hybrid_attn_workspace_size(p) > 0
    assert sv.svgear_kmeans_workspace_size(40, 75600, 128, 500) > 40 * 75600 * 4
    assert sv.svgear_permute_workspace_size(40, 75600, 500) > 0
    bad = sv.params(1, 100, 100, 96, 4, 4, 1, 0.5)      # d = 96 unsupported
    assert sv.svgear_workspace_size(bad) == 0
    assert sv.svgear_kmeans_workspace_size(1, 10, 64, 11) == 0  # C > N


def test_validation_rejects_before_any_launch(L):
    p = sv.params(1, 256, 256, 64, 4, 8, 2, 0.3, 0.0, sv.SVGEAR_F32)
    f = L.svgear_forward
    assert f(None, None, None, ctypes.byref(p), None, None, None, None, 0, None, None) == sv.SVGEAR_ERR_INVALID
    bad = sv.params(1, 256, 256, 64, 4, 8, 2, 1.5)      # rho > 1
    assert f(16, 16, 16, ctypes.byref(bad), None, None, 16, 16, 1 << 30, None, None) == sv.SVGEAR_ERR_INVALID
    bad = sv.params(1, 256, 256, 64, 4, 8, 2, 0.5, 0.0, 7)
    assert f(16, 16, 16, ctypes.byref(bad), None, None, 16, 16, 1 << 30, None, None) == sv.SVGEAR_ERR_UNSUPPORTED
    # missing workspace
    assert f(16, 16, 16, ctypes.byref(p), None, None, 16, None, 0, None, None) == sv.SVGEAR_ERR_WORKSPACE
    # misaligned pointer
    assert f(18, 16, 16, ctypes.byref(p), None, None, 16, 16, 1 << 30, None, None) == sv.SVGEAR_ERR_INVALID
    assert L.svgear_kmeans(16, 0, 1, 10, 64, 0, 1, None, 16, 16, 16, 16, 1 << 20, None) == sv.SVGEAR_ERR_INVALID
    assert L.svgear_route(None, None, None, ctypes.byref(p), None, None, None, None, None) == sv.SVGEAR_ERR_INVALID
    # routing signal outside svgear_router
    for r in (-1, 3):
        bad = sv.params(1, 256, 256, 64, 4, 8, 2, 0.5, router=r)
        assert f(16, 16, 16, ctypes.byref(bad), None, None, 16, 16, 1 << 30, None, None) == sv.SVGEAR_ERR_INVALID
        assert sv.svgear_workspace_size(bad) == 0
    for r in (sv.SVGEAR_ROUTE_MASS, sv.SVGEAR_ROUTE_ERROR_NOV):
        assert sv.svgear_workspace_size(sv.params(1, 256, 256, 64, 4, 8, 2, 0.5, router=r)) > 0
    # budget form outside svgear_budget
    for b in (-1, 2):
        bad = sv.params(1, 256, 256, 64, 4, 8, 2, 0.5, budget=b)
        assert sv.svgear_workspace_size(bad) == 0
    g = sv.params(1, 256, 256, 64, 4, 8, 2, 0.5, budget=sv.SVGEAR_BUDGET_GLOBAL)
    assert sv.svgear_workspace_size(g) > 0
    assert L.svgear_route_global(16, None, 16, 16, ctypes.byref(g), 16, 16, 16, 16, None) == sv.SVGEAR_ERR_INVALID
