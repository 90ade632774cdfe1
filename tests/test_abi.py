"""The C-ABI library: it loads, exports every function include/sa.h
declares, and rejects bad host-side arguments before touching the GPU.
No compute call is made here (this runs without a GPU)."""

import ctypes
import os
import re
import subprocess

import pytest

from sketch_attention_compression_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from sketch_attention_compression_b200 import build
        build.build()
    return binding.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("sa_prepare_query", "sa_sketch_forward", "sa_sketch_free"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (sa_\w+)", out))
    for name in declared_functions():
        assert name in exported, f"{name} declared in sa.h but not exported"
        assert getattr(lib, name) is not None


def test_binding_covers_header():
    assert sorted(binding.SIGNATURES) == declared_functions()


def test_status_strings(lib):
    for code in range(6):
        assert lib.sa_status_string(code)
    assert b"workspace" in lib.sa_status_string(binding.SA_ERR_WORKSPACE)


def test_null_and_range_arguments_rejected_on_host(lib):
    out = ctypes.c_void_p(123)
    st = lib.sa_prepare_query(None, None, None, 16, 64, 0.125, binding.SA_FP32, None,
                              ctypes.byref(out))
    assert st == binding.SA_ERR_INVALID_ARG and out.value is None
    dummy = ctypes.c_void_p(256)
    for k, d in [(0, 64), (1025, 64), (16, 96), (16, 512)]:
        st = lib.sa_prepare_query(dummy, dummy, dummy, k, d, 0.1, binding.SA_BF16, None,
                                  ctypes.byref(out))
        assert st == binding.SA_ERR_INVALID_ARG
    st = lib.sa_prepare_query(dummy, dummy, dummy, 16, 64, float("nan"), binding.SA_BF16, None,
                              ctypes.byref(out))
    assert st == binding.SA_ERR_INVALID_ARG
    st = lib.sa_prepare_query(dummy, dummy, dummy, 16, 64, 0.1, 7, None, ctypes.byref(out))
    assert st == binding.SA_ERR_INVALID_ARG
    assert lib.sa_sketch_forward(None, None, None, 1, 1, None, None, None, 0, None) == \
        binding.SA_ERR_INVALID_ARG
    assert lib.sa_workspace_bytes(None, 1, 1) == 0
    lib.sa_sketch_free(None)  # NULL-safe
    assert lib.sa_read_device_status(None, 0, None, None) == binding.SA_ERR_INVALID_ARG


def test_host_path_rejects_bad_offsets_before_any_copy(lib):
    # q == NULL is checked first; the offsets checks need a real query and
    # run in the GPU suite.
    offs = (ctypes.c_int64 * 3)(0, 5, 3)
    assert lib.sa_sketch_forward_host(None, None, offs, 2, 3, None, None, None, 0, None) == \
        binding.SA_ERR_INVALID_ARG


def declared_signatures():
    """name -> (return type, [parameter types]) parsed from include/sa.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"#[^\n]*", "", text)
    out = {}
    for m in re.finditer(r"([A-Za-z_][\w \*]*?)\b(sa_[a-z_]+)\s*\(([^;{]*?)\)\s*;", text):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        plist = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        out[name] = (ret, plist)
    return out


def _kind(ctype_decl):
    """Coarse class of a C parameter or return type: pointer, 64-bit integer,
    32-bit integer/enum, float, size_t or void."""
    t = " ".join(ctype_decl.replace("*", " * ").split())
    if "*" in t or t.startswith(("sa_query", "sa_refine", "sa_cache", "sa_adapter", "sa_action")):
        return "ptr"
    if t == "double":
        return "f64"
    if "int64_t" in t:
        return "i64"
    if "size_t" in t:
        return "size"
    if "float" in t:
        return "f32"
    if t == "void":
        return "void"
    return "i32"  # int, sa_dtype, sa_status


def _ctypes_kind(ct):
    if ct is None:
        return "void"
    if ct in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(ct, "_type_") and ct.__name__.startswith("LP_"):
        return "ptr"
    if ct is ctypes.c_int64:
        return "i64"
    if ct is ctypes.c_size_t:
        return "size"
    if ct is ctypes.c_float:
        return "f32"
    if ct is ctypes.c_double:
        return "f64"
    return "i32"


def test_binding_signatures_match_header():
    """Every ctypes declaration has the header's parameter count and, class
    by class (pointer, int64, size_t, float, 32-bit int), its types."""
    decl = declared_signatures()
    assert sorted(decl) == declared_functions()
    for name, (ret, params) in decl.items():
        res, args = binding.SIGNATURES[name]
        # names of parameters are stripped: keep the type part of "type name"
        ptypes = [p.rsplit(" ", 1)[0] if not p.endswith("*") else p for p in params]
        got = [_ctypes_kind(a) for a in args]
        want = [_kind(p) for p in ptypes]
        assert got == want, f"{name}: binding {got} vs header {want}"
        assert _ctypes_kind(res) == _kind(ret), f"{name}: return {res} vs {ret}"


def test_refine_entry_points_reject_bad_arguments_on_the_host(lib):
    """The refinement entry points check their arguments before touching the
    device (null handles and pointers, unsupported widths)."""
    out = ctypes.c_void_p()
    dummy = ctypes.c_void_p(256)
    args7 = [dummy] * 7
    assert lib.sa_prepare_refine(*args7, 128, 512, None, None) == binding.SA_ERR_INVALID_ARG
    assert lib.sa_prepare_refine(None, *args7[1:], 128, 512, None, ctypes.byref(out)) == \
        binding.SA_ERR_INVALID_ARG
    for d, h, want in [(128, 100, binding.SA_ERR_INVALID_ARG), (128, 64, binding.SA_ERR_INVALID_ARG),
                       (96, 128, binding.SA_ERR_INVALID_ARG), (256, 128, binding.SA_ERR_UNSUPPORTED)]:
        assert lib.sa_prepare_refine(*args7, d, h, None, ctypes.byref(out)) == want
        assert out.value is None
    lib.sa_refine_free(None)  # NULL-safe
    assert lib.sa_refine_update(None, dummy, 0, dummy, dummy, 1, 4, dummy, None, None) == \
        binding.SA_ERR_INVALID_ARG
    assert lib.sa_refine_layer_forward(None, None, None, None, None, None, 1, 1, None, None, 0,
                                       None) == binding.SA_ERR_INVALID_ARG
    assert lib.sa_refine_stack_forward(0, None, None, None, None, None, 1, 1, None, None, 0,
                                       None) == binding.SA_ERR_INVALID_ARG
    assert lib.sa_workspace_bytes_refine_layer(None, 1, 1) == 0
    assert lib.sa_workspace_bytes_refine_stack(None, 1, 1) == 0


def test_backward_rejects_bad_arguments_on_the_host(lib):
    dummy = ctypes.c_void_p(256)
    assert lib.sa_sketch_backward(None, None, dummy, dummy, dummy, dummy, dummy, 1, 1, dummy, None,
                                  dummy, dummy, dummy, dummy, dummy, 1 << 20, None) == \
        binding.SA_ERR_INVALID_ARG
    assert lib.sa_workspace_bytes_backward(None, 1, 1) == 0


def test_cache_and_adapter_reject_bad_arguments_on_the_host(lib):
    out = ctypes.c_void_p(123)
    # ... the last: capacity * k * (d + 1) * 4 bytes would not fit in size_t
    for k, d, cap, ttl in [(0, 128, 4, 1.0), (16, 6, 4, 1.0), (16, 128, 0, 1.0), (16, 128, 4, 0.0),
                           (16, 128, 4, float("nan")), (1024, 1024, 1 << 50, 1.0)]:
        assert lib.sa_cache_create(k, d, cap, ttl, ctypes.byref(out)) == binding.SA_ERR_INVALID_ARG
        assert out.value is None
    lib.sa_cache_free(None)  # NULL-safe
    dummy = ctypes.c_void_p(256)
    assert lib.sa_cache_lookup(None, dummy, 1, 0.0, dummy, dummy, dummy, None) == \
        binding.SA_ERR_INVALID_ARG
    assert lib.sa_cache_insert(None, dummy, 1, 0.0, dummy, dummy, None) == \
        binding.SA_ERR_INVALID_ARG
    assert lib.sa_cache_stats(None, None, None, None, None) == binding.SA_ERR_INVALID_ARG
    assert lib.sa_cache_forward(None, None, dummy, 0.0, dummy, dummy, 1, 1, dummy, dummy, dummy,
                                dummy, 1 << 20, None) == binding.SA_ERR_INVALID_ARG
    assert lib.sa_cache_forward_workspace_bytes(None, 1, 1) == 0
    for d, D in [(96, 256), (128, 0), (128, 300), (256, 256)]:
        assert lib.sa_prepare_adapter(dummy, d, D, None, ctypes.byref(out)) == \
            binding.SA_ERR_INVALID_ARG
    assert lib.sa_prepare_adapter(None, 128, 256, None, ctypes.byref(out)) == \
        binding.SA_ERR_INVALID_ARG
    lib.sa_adapter_free(None)  # NULL-safe
    assert lib.sa_adapter_forward(None, dummy, 1, dummy, None, None) == binding.SA_ERR_INVALID_ARG


def test_action_entry_points_reject_bad_arguments_on_the_host(lib):
    out = ctypes.c_void_p(123)
    dummy = ctypes.c_void_p(256)
    for d, da, h, nt in [(96, 8, 128, 4), (128, 0, 128, 4), (128, 8, 100, 4), (128, 8, 0, 4),
                         (128, 8, 128, 0), (128, 8, 128, 17), (128, 8, 8192, 4)]:
        assert lib.sa_prepare_action(dummy, dummy, dummy, dummy, d, da, h, nt, None,
                                     ctypes.byref(out)) == binding.SA_ERR_INVALID_ARG
        assert out.value is None
    assert lib.sa_prepare_action(None, dummy, dummy, dummy, 128, 8, 128, 4, None,
                                 ctypes.byref(out)) == binding.SA_ERR_INVALID_ARG
    lib.sa_action_free(None)  # NULL-safe
    assert lib.sa_action_fuse(None, dummy, dummy, 1, dummy, None, None) == \
        binding.SA_ERR_INVALID_ARG
    assert lib.sa_action_sketch_forward(None, None, dummy, dummy, dummy, 1, 1, dummy, dummy, dummy,
                                        1 << 20, None) == binding.SA_ERR_INVALID_ARG
    assert lib.sa_workspace_bytes_action_sketch(None, 1, 1) == 0
