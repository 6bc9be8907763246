"""The C-ABI library loads and exports every entry point include/dms.h declares (CPU only).

No compute call is made here: there is no GPU in this environment.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dms.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dms_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from learned_kv_cache_decode_b200 import build
    build.build()   # nvcc cross-compiles sm_100a without a GPU
    from learned_kv_cache_decode_b200 import _native
    return _native.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("dms_cache_create", "dms_append", "dms_decode_attention", "dms_stats"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    from learned_kv_cache_decode_b200 import _native
    names = declared_functions()
    assert set(names) == set(_native.EXPORTS)
    for name in names:
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr), name


def test_status_strings(lib):
    from learned_kv_cache_decode_b200 import _native
    for code in range(8):
        s = _native.status_string(code)
        assert s and "unknown" not in s
    assert "unknown" in _native.status_string(99)


def test_config_struct_layout_matches_header():
    from learned_kv_cache_decode_b200 import _native
    # 7 int32 fields + 2 enums (int) = 9 * 4 bytes, no padding
    assert ctypes.sizeof(_native.DmsConfig) == 36
    text = open(HEADER).read()
    block = text[text.index("typedef struct {"):text.index("} dms_config;")]
    block = re.sub(r"/\*.*?\*/", "", block, flags=re.S)
    fields = re.findall(r"\b(\w+);", block)
    assert fields == [f for f, _ in _native.DmsConfig._fields_]


def test_product_package_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "learned_kv_cache_decode_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "dms_oracle" not in src, f


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from learned_kv_cache_decode_b200 import _native
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(ImportError):
        _native.load()


def test_a_c_program_compiles_against_the_header_links_and_calls_the_library(lib, tmp_path):
    """The boundary is plain C: dms.h compiles as strict C11, and a C program links
    against libdms.so and calls it (a host-only call: there is no GPU here)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_dms.c"
    src.write_text(
        '#include <stdio.h>\n#include <string.h>\n#include "dms.h"\n'
        "int main(void) {\n"
        '  if (strcmp(dms_status_string(DMS_OK), "ok") != 0) return 1;\n'
        "  if (dms_launch_count(NULL) != 0) return 2;\n"
        "  if (dms_cache_destroy(NULL) != DMS_OK) return 3;\n"
        '  printf("%s\\n", dms_status_string(DMS_ERR_TIMEOUT));\n'
        "  return 0;\n}\n")
    pkg = os.path.join(ROOT, "learned_kv_cache_decode_b200")
    exe = tmp_path / "use_dms"
    cuda_inc = "/usr/local/cuda/include"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, str(src), "-o", str(exe), "-L", pkg, "-ldms", f"-Wl,-rpath,{pkg}"],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True)
    assert out.stdout.strip() == "bounded wait timed out inside a kernel"
