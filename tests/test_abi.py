"""The C-ABI library on the CPU: it loads, exports what include/larosa.h
declares, and rejects bad arguments on the host before touching a device.

No call here launches work: every call fails validation first.
"""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "larosa.h")


@pytest.fixture(scope="module")
def lib():
    from activation_sparsity_b200 import build_lib
    path = build_lib.build()
    lib = ctypes.CDLL(path)
    return lib


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(larosa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("larosa_prepare_weights", "larosa_rotate", "larosa_topk", "larosa_rotate_topk",
                 "larosa_sparse_linear",
                 "larosa_rotate_topk_linear", "larosa_dense_linear", "larosa_workspace_bytes",
                 "larosa_threshold", "larosa_rotate_threshold_linear", "larosa_fold_rotation",
                 "larosa_sparse_lowrank_linear", "larosa_check"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    path = lib._name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s+(larosa_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert getattr(lib, n) is not None


def test_status_strings_and_version(lib):
    lib.larosa_status_string.restype = ctypes.c_char_p
    for code in range(11):
        s = lib.larosa_status_string(code).decode()
        assert s.startswith("LAROSA_")
    assert b"unknown" in lib.larosa_status_string(99)
    assert lib.larosa_version() == 100


def test_debug_and_split_k_settings_validate_and_restore(lib):
    """Host-only settings: out-of-range values change nothing; each setter
    returns the setting it replaced."""
    prev = ctypes.c_int(-7)
    assert lib.larosa_set_debug(2, ctypes.byref(prev)) == 1 and prev.value == -7
    assert lib.larosa_set_split_k(-1, None) == 1
    assert lib.larosa_set_split_k(9, None) == 1
    assert lib.larosa_set_split_k(3, ctypes.byref(prev)) == 0
    first = prev.value
    assert lib.larosa_set_split_k(first, ctypes.byref(prev)) == 0 and prev.value == 3
    assert lib.larosa_set_debug(1, ctypes.byref(prev)) == 0
    was = prev.value
    assert lib.larosa_set_debug(was, ctypes.byref(prev)) == 0 and prev.value == 1


@pytest.mark.parametrize("env,expect", [
    ({"LAROSA_SPLIT_K": "5", "LAROSA_DEBUG": "1"}, (5, 1)),
    ({"LAROSA_SPLIT_K": "12", "LAROSA_DEBUG": "0"}, (0, 0)),   # out of range: chosen per shape
    ({"LAROSA_SPLIT_K": "x", "LAROSA_DEBUG": ""}, (0, 0)),
])
def test_settings_read_from_the_environment_at_first_use(lib, env, expect):
    code = (
        "import ctypes, sys; lib = ctypes.CDLL(sys.argv[1]); p = ctypes.c_int(-1); q = ctypes.c_int(-1);"
        "lib.larosa_set_split_k(0, ctypes.byref(p)); lib.larosa_set_debug(0, ctypes.byref(q));"
        "print(p.value, q.value)")
    e = dict(os.environ)
    e.pop("LAROSA_SPLIT_K", None)
    e.pop("LAROSA_DEBUG", None)
    e.update(env)
    out = subprocess.run([sys.executable, "-c", code, lib._name], capture_output=True, text=True, env=e,
                         check=True).stdout.split()
    assert (int(out[0]), int(out[1])) == expect


P = ctypes.c_void_p
FAKE = P(0x10000)          # aligned, never dereferenced: validation fails first
MISALIGNED = P(0x10008)


def test_host_validation_rejects_bad_arguments(lib):
    BF16, F32 = 1, 0
    z = ctypes.c_size_t(1 << 20)
    # unsupported dtype
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 1, 64, 7, None) == 4
    assert lib.larosa_prepare_weights(FAKE, FAKE, FAKE, 64, 64, 9, None) == 4
    # NULL pointers
    assert lib.larosa_rotate(None, FAKE, FAKE, 1, 64, BF16, None) == 1
    assert lib.larosa_topk(None, 1, 64, 3, FAKE, FAKE, None, None) == 1
    assert lib.larosa_topk(FAKE, 1, 64, 3, None, FAKE, None, None) == 1
    assert lib.larosa_sparse_linear(FAKE, FAKE, 1, 4, None, 64, 64, FAKE, FAKE, z, BF16, None, None) == 1
    assert lib.larosa_prepare_weights(FAKE, None, FAKE, 64, 64, BF16, None) == 1
    # sizes
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 0, 64, BF16, None) == 2
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 17, 64, BF16, None) == 2
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 1, 32769, BF16, None) == 2
    assert lib.larosa_topk(FAKE, 1, 64, 65, FAKE, FAKE, None, None) == 2
    assert lib.larosa_topk(FAKE, 1, 64, -1, FAKE, FAKE, None, None) == 2
    assert lib.larosa_sparse_linear(FAKE, FAKE, 1, 65, FAKE, 64, 64, FAKE, FAKE, z, BF16, None, None) == 2
    assert lib.larosa_rotate_topk_linear(FAKE, FAKE, FAKE, 1, 64, 64, 65, FAKE, FAKE, z, None, BF16, None) == 2
    assert lib.larosa_dense_linear(FAKE, FAKE, 1, 64, 0, FAKE, BF16, None) == 2
    # alignment: base pointers and row lengths (bf16 rows a multiple of 8 elements)
    assert lib.larosa_rotate(FAKE, MISALIGNED, FAKE, 1, 64, BF16, None) == 3
    assert lib.larosa_rotate(MISALIGNED, FAKE, FAKE, 1, 64, BF16, None) == 3
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 1, 60, BF16, None) == 3
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 1, 62, F32, None) == 3
    assert lib.larosa_rotate(FAKE, FAKE, FAKE, 1, 12, F32, None) == 3  # rows a multiple of 8
    assert lib.larosa_sparse_linear(FAKE, FAKE, 1, 4, MISALIGNED, 64, 64, FAKE, FAKE, z, BF16, None, None) == 3
    assert lib.larosa_sparse_linear(FAKE, FAKE, 1, 4, FAKE, 64, 36, FAKE, FAKE, z, BF16, None, None) == 3
    assert lib.larosa_rotate_topk_linear(FAKE, FAKE, FAKE, 1, 64, 12, 5, FAKE, FAKE, z, None, BF16, None) == 3
    assert lib.larosa_dense_linear(FAKE, MISALIGNED, 1, 64, 64, FAKE, BF16, None) == 3
    assert lib.larosa_dense_linear(FAKE, FAKE, 1, 60, 64, FAKE, BF16, None) == 3
    # rotation + Top-K for one token
    assert lib.larosa_rotate_topk(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 3, FAKE, z, None, 7, None) == 4
    assert lib.larosa_rotate_topk(None, FAKE, FAKE, FAKE, FAKE, 64, 3, FAKE, z, None, BF16, None) == 1
    assert lib.larosa_rotate_topk(FAKE, FAKE, FAKE, None, FAKE, 64, 3, FAKE, z, None, BF16, None) == 1
    assert lib.larosa_rotate_topk(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 65, FAKE, z, None, BF16, None) == 2
    assert lib.larosa_rotate_topk(FAKE, FAKE, FAKE, FAKE, FAKE, 32776, 3, FAKE, z, None, BF16, None) == 2
    assert lib.larosa_rotate_topk(FAKE, FAKE, MISALIGNED, FAKE, FAKE, 64, 3, FAKE, z, None, BF16, None) == 3
    assert lib.larosa_rotate_topk(FAKE, FAKE, FAKE, FAKE, FAKE, 60, 3, FAKE, z, None, BF16, None) == 3
    # threshold selection and the threshold path (t is a float; NaN is refused)
    f = ctypes.c_float
    nan = f(float("nan"))
    assert lib.larosa_threshold(None, 1, 64, f(0.5), FAKE, FAKE, FAKE, None, None) == 1
    assert lib.larosa_threshold(FAKE, 1, 64, f(0.5), FAKE, FAKE, None, None, None) == 1
    assert lib.larosa_threshold(FAKE, 1, 64, nan, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.larosa_threshold(FAKE, 0, 64, f(0.5), FAKE, FAKE, FAKE, None, None) == 2
    assert lib.larosa_threshold(FAKE, 1, 32769, f(0.5), FAKE, FAKE, FAKE, None, None) == 2
    rtl = lib.larosa_rotate_threshold_linear
    assert rtl(FAKE, FAKE, FAKE, 1, 64, 64, f(0.5), FAKE, FAKE, z, None, 7, None) == 4
    assert rtl(None, FAKE, FAKE, 1, 64, 64, f(0.5), FAKE, FAKE, z, None, BF16, None) == 1
    assert rtl(FAKE, FAKE, FAKE, 1, 64, 64, nan, FAKE, FAKE, z, None, BF16, None) == 1
    assert rtl(FAKE, FAKE, FAKE, 17, 64, 64, f(0.5), FAKE, FAKE, z, None, BF16, None) == 2
    assert rtl(FAKE, FAKE, FAKE, 1, 64, 12, f(0.5), FAKE, FAKE, z, None, BF16, None) == 3
    assert rtl(MISALIGNED, None, FAKE, 1, 64, 64, f(0.5), FAKE, FAKE, z, None, BF16, None) == 3
    assert rtl(FAKE, None, FAKE, 1, 60, 64, f(0.5), FAKE, FAKE, z, None, BF16, None) == 3
    # the identity rotation (no Qt) is checked like the rotated path
    assert lib.larosa_rotate_topk_linear(MISALIGNED, None, FAKE, 1, 64, 64, 5, FAKE, FAKE, z, None, BF16, None) == 3
    assert lib.larosa_rotate_topk_linear(FAKE, None, FAKE, 1, 64, 64, 65, FAKE, FAKE, z, None, BF16, None) == 2
    off = ctypes.c_size_t()
    assert lib.larosa_workspace_nnz_offset(1, 64, 64, 65, ctypes.byref(off)) == 2
    # folding the rotation into a producer is validated as the counter-rotation
    assert lib.larosa_fold_rotation(FAKE, None, FAKE, 64, 64, BF16, None) == 1
    assert lib.larosa_fold_rotation(FAKE, FAKE, FAKE, 64, 64, 9, None) == 4
    assert lib.larosa_fold_rotation(FAKE, FAKE, FAKE, 0, 64, BF16, None) == 2
    # sparse + low rank
    slr = lib.larosa_sparse_lowrank_linear
    assert slr(None, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, 64, 64, 16, FAKE, FAKE, z, BF16, None, None) == 1
    assert slr(FAKE, FAKE, FAKE, 1, 4, FAKE, None, FAKE, 64, 64, 16, FAKE, FAKE, z, BF16, None, None) == 1
    assert slr(FAKE, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, 64, 64, 0, FAKE, FAKE, z, BF16, None, None) == 2
    assert slr(FAKE, FAKE, FAKE, 1, 65, FAKE, FAKE, FAKE, 64, 64, 16, FAKE, FAKE, z, BF16, None, None) == 2
    assert slr(FAKE, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, 64, 64, 12, FAKE, FAKE, z, BF16, None, None) == 3
    assert slr(FAKE, FAKE, FAKE, 1, 4, FAKE, MISALIGNED, FAKE, 64, 64, 16, FAKE, FAKE, z, BF16, None, None) == 3
    assert slr(FAKE, FAKE, FAKE, 1, 4, FAKE, FAKE, FAKE, 64, 64, 16, FAKE, FAKE, z, 7, None, None) == 4
    # in-place counter-rotation is refused
    assert lib.larosa_prepare_weights(FAKE, P(0x20000), P(0x20000), 64, 64, BF16, None) == 1
    # status check needs a status word
    assert lib.larosa_check(None, None, None) == 1


def _prototypes():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//.*", "", text)
    out = {}
    for ret, name, args in re.findall(r"([A-Za-z_][\w \*]*?)\b(larosa_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text,
                                      flags=re.S):
        params = [a.strip() for a in args.replace("\n", " ").split(",")] if args.strip() not in ("", "void") else []
        out[name] = (ret.strip(), params)
    return out


def _kind_of_c(decl: str) -> str:
    """'ptr', 'int', 'size', 'float' or 'str' for one C parameter or return type."""
    if decl.startswith("const char") and "*" in decl:
        return "str"
    if "*" in decl or decl.startswith("larosa_stream_t"):
        return "ptr"
    t = decl.split()[0] if not decl.startswith("const ") else decl.split()[1]
    # uint64_t and size_t are the same 64-bit unsigned integer on this ABI
    # (ctypes.c_uint64 is ctypes.c_size_t)
    return {"int": "int", "size_t": "size", "uint64_t": "size", "float": "float"}[t]


def _kind_of_ctypes(t) -> str:
    if t is ctypes.c_char_p:
        return "str"
    if t is ctypes.c_void_p or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    return {ctypes.c_int: "int", ctypes.c_size_t: "size", ctypes.c_float: "float"}[t]


def test_binding_signatures_match_the_header(lib):
    """Every entry point the binding calls has the header's arity and
    argument kinds (pointer, int, size_t, float), so the marshalling cannot
    drift from the C ABI unnoticed."""
    from activation_sparsity_b200 import larosa as binding
    protos = _prototypes()
    for name, (args, ret) in binding._SIGNATURES.items():
        assert name in protos, name
        c_ret, c_params = protos[name]
        assert [_kind_of_c(p) for p in c_params] == [_kind_of_ctypes(a) for a in args], name
        assert _kind_of_c(c_ret) == _kind_of_ctypes(ret), name
    # and the binding covers every declared entry point
    assert set(protos) == set(binding._SIGNATURES)


def test_binding_constants_match_the_header():
    """The status codes, device bits and limits the binding names have the
    header's values."""
    from activation_sparsity_b200 import larosa as binding
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    values = {m.group(1): int(m.group(2), 0)
              for m in re.finditer(r"#define\s+(LAROSA_\w+)\s+(0x[0-9a-fA-F]+|\d+)", text)}
    values.update({m.group(1): int(m.group(2)) for m in re.finditer(r"\b(LAROSA_[A-Z0-9_]+)\s*=\s*(\d+)", text)})
    values.update({m.group(1): int(m.group(2)) << int(m.group(3))
                   for m in re.finditer(r"#define\s+(LAROSA_\w+)\s+\((\d+)u?\s*<<\s*(\d+)\)", text)})
    checked = 0
    for name in dir(binding):
        if name.startswith("LAROSA_") and name in values:
            assert getattr(binding, name) == values[name], name
            checked += 1
    assert checked >= 15
