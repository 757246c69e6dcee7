"""The C ABI library loads and exports every symbol include/atlaskv.h
declares; host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

from hierarchical_kv_pruning_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "atlaskv.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(atlaskv_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("atlaskv_create_tree", "atlaskv_attend", "atlaskv_destroy"):
        assert name in syms
    assert sorted(binding.EXPORTED) == syms


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def _desc(**kw):
    d = binding.atlaskv_tree_desc()
    d.dtype = kw.get("dtype", binding.ATLASKV_BF16)
    d.n_kv_heads = kw.get("n_kv_heads", 1)
    d.head_dim = kw.get("head_dim", 128)
    d.fanout[:] = kw.get("fanout", (4, 4, 4))
    for f in ("root_keys", "mid_keys", "leaf_keys", "leaf_values"):
        setattr(d, f, kw.get(f, 4096))
    d.leaf_location = kw.get("leaf_location", binding.ATLASKV_LEAVES_DEVICE)
    d.mid_location = kw.get("mid_location", binding.ATLASKV_LEAVES_DEVICE)
    return d


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), binding.ATLASKV_EUNSUPPORTED),
    (dict(dtype=7), binding.ATLASKV_EINVAL),
    (dict(n_kv_heads=0), binding.ATLASKV_EINVAL),
    (dict(fanout=(4, 0, 4)), binding.ATLASKV_EINVAL),
    (dict(root_keys=None), binding.ATLASKV_EINVAL),
    (dict(mid_keys=4100), binding.ATLASKV_EINVAL),            # not 16-byte aligned
    (dict(leaf_location=5), binding.ATLASKV_EINVAL),
    (dict(mid_location=5), binding.ATLASKV_EINVAL),
    (dict(mid_location=binding.ATLASKV_LEAVES_HOST_PINNED), binding.ATLASKV_EINVAL),   # mids on host, leaves not
    (dict(fanout=(2000, 2000, 2000)), binding.ATLASKV_EUNSUPPORTED),
])
def test_create_tree_rejects_bad_descriptions(lib, kw, status):
    out = ctypes.c_void_p()
    st = lib.atlaskv_create_tree(ctypes.byref(_desc(**kw)), None, ctypes.byref(out))
    assert st == status
    assert out.value is None
    assert binding.atlaskv_last_error() != ""


def test_null_arguments(lib):
    out = ctypes.c_void_p()
    assert lib.atlaskv_create_tree(None, None, ctypes.byref(out)) == binding.ATLASKV_EINVAL
    p = binding.atlaskv_params(1, 1, 1, 0.0)
    sz = ctypes.c_size_t()
    assert lib.atlaskv_workspace_size(None, ctypes.byref(p), 1, 1, 1, 1, ctypes.byref(sz)) == binding.ATLASKV_EINVAL
    io = binding.atlaskv_io()
    assert lib.atlaskv_attend(None, ctypes.byref(p), ctypes.byref(io), None, 0, None) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_attend(None, ctypes.byref(p), None, None, 0, None) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_sync_status(None, None) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_set_profiling(None, 1) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_set_descent(None, binding.ATLASKV_DESCENT_FUSED) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_set_leaf_cache(None, 8, None) == binding.ATLASKV_EINVAL
    cnt = (ctypes.c_uint64 * 3)()
    assert lib.atlaskv_leaf_cache_stats(None, cnt, 3) == binding.ATLASKV_EINVAL
    buf = (ctypes.c_float * 3)()
    assert lib.atlaskv_stage_times(None, buf, 3) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_destroy(None) == binding.ATLASKV_OK
    trees = (ctypes.c_void_p * 2)(None, None)
    ios = (binding.atlaskv_io * 2)()
    assert lib.atlaskv_workspace_size_layers(2, trees, ctypes.byref(p), ios, ctypes.byref(sz)) == \
        binding.ATLASKV_EINVAL                                         # null trees
    assert lib.atlaskv_workspace_size_layers(0, trees, ctypes.byref(p), ios, ctypes.byref(sz)) == \
        binding.ATLASKV_EINVAL                                         # no layers
    assert lib.atlaskv_workspace_size_layers(binding.MAX_LAYERS + 1, trees, ctypes.byref(p), ios,
                                             ctypes.byref(sz)) == binding.ATLASKV_EINVAL
    assert lib.atlaskv_attend_layers(2, trees, ctypes.byref(p), ios, None, 0, None) == binding.ATLASKV_EINVAL


def test_error_wrapper_raises(lib):
    with pytest.raises(binding.AtlaskvError) as ei:
        binding.atlaskv_create_tree(_desc(head_dim=32))
    assert ei.value.status == binding.ATLASKV_EUNSUPPORTED
    assert "head_dim" in str(ei.value)


def test_missing_library_fails_loudly(tmp_path):
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(OSError):
            binding.load_library(str(tmp_path / "nope.so"))
    finally:
        binding._lib = saved


def test_product_path_never_reaches_the_oracle():
    # The library and its binding compute everything in CUDA; no file of the
    # package imports, loads or links the oracle (test infrastructure only).
    import ast
    import glob
    pkg = os.path.join(ROOT, "hierarchical_kv_pruning_b200")
    for path in glob.glob(os.path.join(pkg, "*.py")):
        tree = ast.parse(open(path).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                assert not any(a.name.split(".")[0] == "oracle" for a in node.names), path
            if isinstance(node, ast.ImportFrom):
                assert (node.module or "").split(".")[0] != "oracle", path
            if isinstance(node, ast.Constant) and isinstance(node.value, str):
                assert "hikvp_oracle" not in node.value, path
    for path in glob.glob(os.path.join(pkg, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*")):
        text = open(path).read()
        assert "hikvp_oracle" not in text and "oracle/" not in text, path
