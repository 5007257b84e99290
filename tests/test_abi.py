"""The C-ABI library builds, loads and exports every entry point include/cf.h declares (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "cf.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(cf_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def libcf():
    from activation_residual_compression_02_b200 import build

    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["cf_create", "cf_compress", "cf_decompress", "cf_lowrank", "cf_destroy", "cf_check",
                 "cf_workspace_bytes", "cf_set_workspace", "cf_payload_bytes", "cf_last_error",
                 "cf_lowrank_workspace_bytes"]:
        assert want in names


def test_library_exports_every_declared_symbol(libcf):
    for name in declared_functions():
        assert hasattr(libcf, name), name


def test_binding_names_match_header():
    import activation_residual_compression_02_b200 as cf

    assert set(cf.EXPORTED) == set(declared_functions())


def test_library_is_sm100a_only():
    """The library carries sm_100a code only (checked from the build flags)."""
    from activation_residual_compression_02_b200 import build

    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "use_fast_math" not in flags


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "activation_residual_compression_02_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), f
                assert "cf_oracle" not in text, f


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import activation_residual_compression_02_b200._cf as b

    monkeypatch.setattr(b, "_lib", None)
    monkeypatch.setattr(b, "_LIB_PATH", str(tmp_path / "libcf.so"))
    with pytest.raises(ImportError):
        b.lib()


def test_every_call_names_its_source():
    """Each function declared in include/cf.h carries, in the comment right
    above it, a "Source:" line: the passage of the pages that defines the
    operation, or the statement that it is library plumbing."""
    src = open(os.path.join(ROOT, "include", "cf.h")).read()
    missing = []
    for m in re.finditer(r"/\*(?:(?!\*/).)*\*/\s*(?:typedef[^;]*;\s*|#define[^\n]*\n\s*)*"
                         r"(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(cf_\w+)\s*\(", src, flags=re.S):
        comment = m.group(0)[:m.group(0).rindex("*/")]
        if "Source:" not in comment:
            missing.append(m.group(1))
    found = {m.group(1) for m in re.finditer(r"/\*(?:(?!\*/).)*\*/\s*(?:typedef[^;]*;\s*|#define[^\n]*\n\s*)*"
                                             r"(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(cf_\w+)\s*\(", src, flags=re.S)}
    assert found == set(declared_functions()), set(declared_functions()) ^ found
    assert not missing, missing
