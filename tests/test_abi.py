"""The C ABI without a GPU: the library loads, exports what include/*.h
declares, and rejects invalid arguments with status codes (no device call)."""

import ctypes
import os
import re

import pytest

from rank_structured_matmul_b200 import dyra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(dyra_[a-z_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = dyra.lib()
    names = declared_functions()
    assert {"dyra_plan_create", "dyra_load_factors", "dyra_forward", "dyra_plan_destroy"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), "libdyra.so does not export %s" % n
    assert set(dyra.SIGNATURES) <= names


def test_debug_library_exports_every_declared_symbol():
    """The bounds-checked build (compiled with DYRA_DEBUG) has the same ABI."""
    import ctypes
    from rank_structured_matmul_b200.build import build
    build(debug=True)  # incremental: rebuilt only when a source is newer
    lib = ctypes.CDLL(dyra.DEBUG_LIB_PATH)
    for n in sorted(declared_functions()):
        assert hasattr(lib, n), "libdyra_debug.so does not export %s" % n


def test_error_strings():
    for code in range(0, -9, -1):
        s = dyra.error_string(code)
        assert s and s != "unknown error"
    assert dyra.error_string(-99) == "unknown error"


def _create(*args):
    lib = dyra.lib()
    h = ctypes.c_void_p()
    rc = lib.dyra_plan_create(ctypes.byref(h), *args)
    return rc, h


@pytest.mark.parametrize("args,code", [
    ((0, 256, 32, 8, dyra.DYRA_F32), dyra.DYRA_ERR_INVALID_ARG),      # d_in < 1
    ((256, -1, 32, 8, dyra.DYRA_F32), dyra.DYRA_ERR_INVALID_ARG),     # d_out < 1
    ((256, 256, 0, 8, dyra.DYRA_F32), dyra.DYRA_ERR_INVALID_ARG),     # r < 1
    ((256, 256, 32, -1, dyra.DYRA_F32), dyra.DYRA_ERR_INVALID_ARG),   # k < 0
    ((256, 256, 32, 129, dyra.DYRA_F32), dyra.DYRA_ERR_INVALID_ARG),  # k > 128
    ((64, 256, 60, 8, dyra.DYRA_F32), dyra.DYRA_ERR_INVALID_ARG),     # r + k > min(d_in, d_out)
    ((256, 256, 32, 8, 7), dyra.DYRA_ERR_INVALID_ARG),                # bad dtype
    ((260, 256, 32, 8, dyra.DYRA_BF16), dyra.DYRA_ERR_ALIGNMENT),     # d_in % 8
    ((256, 252, 32, 8, dyra.DYRA_BF16), dyra.DYRA_ERR_ALIGNMENT),     # d_out % 8
    ((256, 256, 30, 8, dyra.DYRA_BF16), dyra.DYRA_ERR_ALIGNMENT),     # r % 8
    ((256, 256, 32, 12, dyra.DYRA_BF16), dyra.DYRA_ERR_ALIGNMENT),    # k % 8
])
def test_plan_create_rejects(args, code):
    rc, h = _create(*args)
    assert rc == code
    assert h.value is None


def test_null_handles():
    lib = dyra.lib()
    assert lib.dyra_plan_create(None, 256, 256, 32, 8, dyra.DYRA_F32) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_forward(None, None, None, 10, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_forward_batched(None, None, None, 2, 3, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_forward_weight_only(None, None, None, 1, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_load_factors(None, None, None, None, None, 0.0, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_reserve(None, 1, 1) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_set_linear(None, None, 1.0, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_set_als_steps(None, 2) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_forward_batched_host(None, None, None, 2, 3, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_plan_create_monarch(None, 12, 3, 4, 2, dyra.DYRA_F32) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_load_monarch(None, None, None, None, None, 0.0, None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_last_status(None) == dyra.DYRA_ERR_INVALID_ARG
    assert lib.dyra_plan_destroy(None) == dyra.DYRA_OK
    assert lib.dyra_plan_device_bytes(None) == 0


def test_python_wrapper_raises():
    with pytest.raises(dyra.DyraError) as e:
        dyra.dyra_plan_create(256, 256, 32, 12, dyra.DYRA_BF16)
    assert e.value.code == dyra.DYRA_ERR_ALIGNMENT


def test_plan_create_without_gpu_fails_cleanly():
    """A valid shape needs a B200; on a machine without one the call returns
    an error code (CUDA or UNSUPPORTED), never crashes."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc, h = _create(256, 256, 32, 8, dyra.DYRA_BF16)
    assert rc in (dyra.DYRA_ERR_CUDA, dyra.DYRA_ERR_UNSUPPORTED)
    assert h.value is None


def _declared_signatures():
    """name -> list of parameter type strings, from include/*.h."""
    sigs = {}
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if not f.endswith(".h"):
            continue
        text = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, f)).read(), flags=re.S)
        for m in re.finditer(r"\b(dyra_[a-z_]+)\s*\(([^;{)]*)\)\s*;", text):
            params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
            sigs[m.group(1)] = params
    return sigs


def _kind(c_param):
    """The ctypes class a C parameter declaration needs."""
    t = re.sub(r"\b[A-Za-z_][A-Za-z_0-9]*$", "", c_param).strip()  # drop the parameter name
    if "*" in t or t.endswith("_t") and t not in ("int64_t", "uint64_t", "size_t", "dyra_dtype_t"):
        return "ptr"
    # uint64_t and size_t are the same 64-bit unsigned type on LP64 Linux
    # (ctypes.c_uint64 is ctypes.c_size_t there)
    return {"int": "int", "dyra_dtype_t": "int", "int64_t": "int64", "uint64_t": "size",
            "float": "float", "size_t": "size"}[t]


def test_binding_signatures_match_the_header():
    """Every call the binding declares has the header's parameter count and
    kinds (pointer, int, int64, float, size), so a changed header cannot
    silently misalign the ctypes arguments."""
    kinds = {ctypes.c_void_p: "ptr", ctypes.c_int: "int", ctypes.c_int64: "int64",
             ctypes.c_float: "float", ctypes.c_size_t: "size"}
    declared = _declared_signatures()
    for name, (_, args) in dyra.SIGNATURES.items():
        assert name in declared, name
        want = [_kind(p) for p in declared[name]]
        got = ["ptr" if getattr(a, "_type_", None) is not None and a is not ctypes.c_void_p
               and issubclass(a, ctypes._Pointer) else kinds[a] for a in args]
        assert got == want, "%s: binding %s, header %s" % (name, got, want)
