"""CPU-side checks of the C-ABI library: it builds for sm_100a, loads, and
exports every entry point include/eblc.h declares; argument and option
validation that happens before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def E():
    from error_bounded_lossy_encode_b200 import build

    build.build()
    import error_bounded_lossy_encode_b200 as E

    return E


def _declared():
    src = open(os.path.join(ROOT, "include", "eblc.h")).read()
    return sorted(set(re.findall(r"EBLC_API[^;(]*?\b(eblc_\w+)\s*\(", src)))


def test_header_declares_entry_points():
    names = _declared()
    assert {"eblc_abi_version", "eblc_status_string", "eblc_plan_create", "eblc_plan_get_limits", "eblc_compress",
            "eblc_decompress", "eblc_check", "eblc_plan_kernel_times", "eblc_plan_destroy"} <= set(names)


def test_library_exports_every_declared_symbol(E):
    L = ctypes.CDLL(E.LIB_PATH)
    for name in _declared():
        assert hasattr(L, name), name


def test_only_api_symbols_exported(E):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", E.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {s for s in exported if s.startswith("eblc_")} == set(_declared())


def test_version_and_status_strings(E):
    assert E.eblc_abi_version() == 1
    assert E.eblc_status_string(E.EBLC_OK) == "ok"
    assert E.eblc_status_string(E.EBLC_CORRUPT) == "corrupt stream"
    assert E.eblc_status_string(99) == "unknown status"


def test_struct_sizes(E):
    assert ctypes.sizeof(E.eblc_sidecar_t) == 64
    assert ctypes.sizeof(E.eblc_limits_t) == 72  # matches the static_assert in plan.cu
    assert ctypes.sizeof(E.eblc_async_result_t) == 32  # matches the static_assert in plan.cu


@pytest.mark.parametrize("opts,status", [
    ("rel=-1", 2), ("abs=nan", 2), ("rel=1e-3,abs=1e-3", 2), ("block=48", 1), ("bogus=1", 1), ("rel", 2),
    ("block=x", 2), ("outlier_cap=-3", 2), ("wait_ms=0", 2)])
def test_option_errors_need_no_gpu(E, opts, status):
    st, plan = E.eblc_plan_create([100], None, opts)
    assert st == status and plan is None


def test_shape_errors_need_no_gpu(E):
    assert E.eblc_plan_create([], None, None)[0] == E.EBLC_INVALID_ARG
    assert E.eblc_plan_create([-1], None, None)[0] == E.EBLC_INVALID_ARG
    assert E.eblc_plan_create([1 << 20, 1 << 11], None, None)[0] == E.EBLC_UNSUPPORTED
    assert E.eblc_plan_create([4, 5], [1, 4], None)[0] == E.EBLC_UNSUPPORTED


def test_null_arguments(E):
    assert E.lib().eblc_plan_create(None, 1, None, None, None) == E.EBLC_INVALID_ARG
    assert E.lib().eblc_plan_get_limits(None, None) == E.EBLC_INVALID_ARG
    assert E.lib().eblc_compress(None, None, None, None, 0, None, None) == E.EBLC_INVALID_ARG
    assert E.lib().eblc_decompress(None, None, None, 0, None, None) == E.EBLC_INVALID_ARG
    E.eblc_plan_destroy(None)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import error_bounded_lossy_encode_b200 as E

    monkeypatch.setattr(E, "_lib", None)
    monkeypatch.setattr(E, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        E.lib()


def test_product_path_never_touches_the_oracle():
    """The library and its binding neither import, load nor execute anything
    under oracle/: only the tests, the smoke check and the benchmark's CPU
    legs may.  Python: no import of it and no string naming it outside
    docstrings; C/CUDA: no reference to its symbols or files outside comments."""
    import ast
    import pathlib
    import re

    root = pathlib.Path(__file__).resolve().parents[1]
    pkg = root / "error_bounded_lossy_encode_b200"
    offenders = []
    for path in pkg.rglob("*.py"):
        tree = ast.parse(path.read_text())
        docstrings = set()
        for node in ast.walk(tree):
            if isinstance(node, (ast.Module, ast.FunctionDef, ast.ClassDef, ast.AsyncFunctionDef)):
                body = getattr(node, "body", [])
                if body and isinstance(body[0], ast.Expr) and isinstance(getattr(body[0], "value", None), ast.Constant):
                    docstrings.add(id(body[0].value))
        for node in ast.walk(tree):
            if isinstance(node, ast.Import) and any("oracle" in a.name for a in node.names):
                offenders.append(f"{path.name}:{node.lineno} import")
            if isinstance(node, ast.ImportFrom) and "oracle" in (node.module or ""):
                offenders.append(f"{path.name}:{node.lineno} from-import")
            if isinstance(node, ast.Constant) and isinstance(node.value, str) and id(node) not in docstrings \
                    and re.search(r"oracle|eblc_oracle", node.value):
                offenders.append(f"{path.name}:{node.lineno} string {node.value[:40]!r}")
    pattern = re.compile(r"eblc_oracle|\borc_\w+|oracle/")
    for path in list(pkg.rglob("*.cu")) + list(pkg.rglob("*.cuh")) + list(pkg.rglob("*.h")) + \
            list((root / "include").rglob("*.h")):
        text = re.sub(r"/\*.*?\*/", "", path.read_text(), flags=re.S)
        for ln, line in enumerate(text.splitlines(), 1):
            if pattern.search(line.split("//")[0]):
                offenders.append(f"{path.name}:{ln}: {line.strip()}")
    assert not offenders, offenders


def test_header_compiles_as_c99_and_links(tmp_path):
    """A plain C program (C99, -Wall -Werror) includes the header, links
    against the library and exercises the calls that need no GPU."""
    import shutil
    import subprocess

    import error_bounded_lossy_encode_b200 as E

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    E.lib()  # fails loudly when the library is not built
    src = tmp_path / "abi.c"
    src.write_text(r"""
#include <stdio.h>
#include <string.h>
#include "eblc.h"
int main(void) {
    if (eblc_abi_version() != EBLC_ABI_VERSION) return 1;
    if (strcmp(eblc_status_string(EBLC_OK), "ok") != 0) return 2;
    eblc_plan_t plan = (eblc_plan_t)1;
    int64_t dims[1] = {100};
    if (eblc_plan_create(&plan, 1, dims, NULL, "block=48") != EBLC_UNSUPPORTED || plan != NULL) return 3;
    if (eblc_plan_create(&plan, 0, dims, NULL, NULL) != EBLC_INVALID_ARG) return 4;
    if (eblc_compress(NULL, NULL, NULL, NULL, 0, NULL, NULL) != EBLC_INVALID_ARG) return 5;
    if (sizeof(eblc_sidecar_t) != 64 || sizeof(eblc_async_result_t) != 32) return 6;
    eblc_plan_destroy(NULL);
    puts("c abi ok");
    return 0;
}
""")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(E.LIB_PATH)
    inc = os.path.join(os.path.dirname(libdir), "include")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", inc, str(src), "-o", str(exe),
                    "-L", libdir, "-leblc", "-Wl,-rpath," + libdir], check=True, capture_output=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)
