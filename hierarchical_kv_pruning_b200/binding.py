"""ctypes binding of libatlaskv.so (the C ABI in include/atlaskv.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  The ``atlaskv_*`` functions mirror the C entry points one to one;
``HikvpTree`` is a thin convenience layer that takes torch tensors (torch is
used for device memory and streams), keeps them alive, and allocates outputs
and the workspace.  If the library is missing or fails to load, every call
raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libatlaskv.so")

ATLASKV_OK, ATLASKV_EINVAL, ATLASKV_ENOMEM, ATLASKV_ECUDA, ATLASKV_EUNSUPPORTED, ATLASKV_ETIMEOUT, ATLASKV_EDEVICE = range(7)
STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ENOMEM", 3: "ECUDA", 4: "EUNSUPPORTED", 5: "ETIMEOUT", 6: "EDEVICE"}
ATLASKV_F32, ATLASKV_BF16 = 0, 1
ATLASKV_LEAVES_DEVICE, ATLASKV_LEAVES_HOST_PINNED = 0, 1
ATLASKV_PROFILE_TIMES, ATLASKV_PROFILE_COUNTERS = 1, 2
ATLASKV_DESCENT_AUTO, ATLASKV_DESCENT_FUSED, ATLASKV_DESCENT_PARENT_MAJOR = 0, 1, 2
STAGE_NAMES = ("descend", "staging", "attend", "attend_seq", "attend_leaf")

# Every symbol include/atlaskv.h declares.
EXPORTED = ("atlaskv_create_tree", "atlaskv_workspace_size", "atlaskv_attend", "atlaskv_sync_status",
            "atlaskv_set_profiling", "atlaskv_stage_times", "atlaskv_refine_stats", "atlaskv_attend_static",
            "atlaskv_probe_wait_timeout", "atlaskv_destroy", "atlaskv_last_error", "atlaskv_workspace_size_layers",
            "atlaskv_attend_layers", "atlaskv_create_tree_csr", "atlaskv_workspace_size_csr", "atlaskv_attend_csr",
            "atlaskv_set_descent", "atlaskv_set_leaf_cache", "atlaskv_leaf_cache_stats")
MAX_LAYERS = 32
MAX_LEVELS = 4
# Size of the library's static device scratch (ATLASKV_STATIC_SCRATCH_BYTES).
ATLASKV_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024


class AtlaskvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), message))
        self.status = status


class atlaskv_tree_desc(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("fanout", ctypes.c_int32 * 3),
        ("root_keys", ctypes.c_void_p),
        ("mid_keys", ctypes.c_void_p),
        ("leaf_keys", ctypes.c_void_p),
        ("leaf_values", ctypes.c_void_p),
        ("leaf_location", ctypes.c_int32),
        ("root_child", ctypes.c_void_p),
        ("mid_child", ctypes.c_void_p),
        ("mid_location", ctypes.c_int32),
    ]


class atlaskv_csr_tree_desc(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("n_levels", ctypes.c_int32),
        ("rows", ctypes.c_int64 * 4),
        ("keys", ctypes.c_void_p * 4),
        ("child_off", ctypes.c_void_p * 3),
        ("child_id", ctypes.c_void_p * 3),
        ("leaf_values", ctypes.c_void_p),
    ]


class atlaskv_level_params(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32 * 4), ("scale", ctypes.c_float)]


class atlaskv_params(ctypes.Structure):
    _fields_ = [("K_root", ctypes.c_int32), ("K_mid", ctypes.c_int32), ("K_leaf", ctypes.c_int32),
                ("scale", ctypes.c_float)]


class atlaskv_io(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("N", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32),
        ("q_kg", ctypes.c_void_p), ("q_seq", ctypes.c_void_p), ("k_seq", ctypes.c_void_p), ("v_seq", ctypes.c_void_p),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("kept_root", ctypes.c_void_p), ("kept_mid", ctypes.c_void_p), ("kept_leaf", ctypes.c_void_p),
    ]


_lib = None
_lock = threading.Lock()


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load the in-tree library (raises OSError if it is missing)."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise OSError("libatlaskv.so not built at %s (run python -m hierarchical_kv_pruning_b200.build)" % p)
            lib = ctypes.CDLL(p)
            V, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            lib.atlaskv_create_tree.argtypes = [ctypes.POINTER(atlaskv_tree_desc), V, ctypes.POINTER(V)]
            lib.atlaskv_workspace_size.argtypes = [V, ctypes.POINTER(atlaskv_params), I32, I32, I32, I32,
                                                   ctypes.POINTER(SZ)]
            lib.atlaskv_attend.argtypes = [V, ctypes.POINTER(atlaskv_params), ctypes.POINTER(atlaskv_io), V, SZ, V]
            lib.atlaskv_attend_static.argtypes = [V, ctypes.POINTER(atlaskv_params), ctypes.POINTER(atlaskv_io), V]
            lib.atlaskv_workspace_size_layers.argtypes = [I32, ctypes.POINTER(V), ctypes.POINTER(atlaskv_params),
                                                          ctypes.POINTER(atlaskv_io), ctypes.POINTER(SZ)]
            lib.atlaskv_attend_layers.argtypes = [I32, ctypes.POINTER(V), ctypes.POINTER(atlaskv_params),
                                                  ctypes.POINTER(atlaskv_io), V, SZ, V]
            lib.atlaskv_create_tree_csr.argtypes = [ctypes.POINTER(atlaskv_csr_tree_desc), V, ctypes.POINTER(V)]
            lib.atlaskv_workspace_size_csr.argtypes = [V, ctypes.POINTER(atlaskv_level_params), I32, I32, I32, I32,
                                                       ctypes.POINTER(SZ)]
            lib.atlaskv_attend_csr.argtypes = [V, ctypes.POINTER(atlaskv_level_params), ctypes.POINTER(atlaskv_io),
                                               ctypes.POINTER(V), V, SZ, V]
            lib.atlaskv_sync_status.argtypes = [V, V]
            lib.atlaskv_set_profiling.argtypes = [V, I32]
            lib.atlaskv_set_descent.argtypes = [V, I32]
            lib.atlaskv_set_leaf_cache.argtypes = [V, ctypes.c_int64, V]
            lib.atlaskv_leaf_cache_stats.argtypes = [V, ctypes.POINTER(ctypes.c_uint64), I32]
            lib.atlaskv_stage_times.argtypes = [V, ctypes.POINTER(ctypes.c_float), I32]
            lib.atlaskv_refine_stats.argtypes = [V, ctypes.POINTER(ctypes.c_uint64), I32]
            lib.atlaskv_probe_wait_timeout.argtypes = [V, V]
            lib.atlaskv_destroy.argtypes = [V]
            lib.atlaskv_last_error.argtypes = []
            lib.atlaskv_last_error.restype = ctypes.c_char_p
            for name in EXPORTED:
                if name != "atlaskv_last_error":
                    getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _check(status: int):
    if status != ATLASKV_OK:
        raise AtlaskvError(status, atlaskv_last_error())


# ---- one-to-one wrappers of the C entry points ------------------------------

def atlaskv_last_error() -> str:
    return load_library().atlaskv_last_error().decode()


def atlaskv_create_tree(desc: atlaskv_tree_desc, stream: int = 0) -> int:
    handle = ctypes.c_void_p()
    _check(load_library().atlaskv_create_tree(ctypes.byref(desc), ctypes.c_void_p(stream), ctypes.byref(handle)))
    return handle.value


def atlaskv_workspace_size(tree: int, params: atlaskv_params, B: int, N: int, H: int, T: int) -> int:
    out = ctypes.c_size_t()
    _check(load_library().atlaskv_workspace_size(ctypes.c_void_p(tree), ctypes.byref(params), B, N, H, T,
                                                 ctypes.byref(out)))
    return out.value


def atlaskv_attend(tree: int, params: atlaskv_params, io: atlaskv_io, workspace: int, workspace_bytes: int,
                   stream: int = 0) -> None:
    _check(load_library().atlaskv_attend(ctypes.c_void_p(tree), ctypes.byref(params), ctypes.byref(io),
                                         ctypes.c_void_p(workspace), workspace_bytes, ctypes.c_void_p(stream)))


def atlaskv_attend_static(tree: int, params: atlaskv_params, io: atlaskv_io, stream: int = 0) -> None:
    """atlaskv_attend without a caller workspace: the library's static device
    scratch (ATLASKV_STATIC_SCRATCH_BYTES) is used instead.  For callers that
    cannot allocate device memory; calls that overlap on the GPU race."""
    _check(load_library().atlaskv_attend_static(ctypes.c_void_p(tree), ctypes.byref(params), ctypes.byref(io),
                                                ctypes.c_void_p(stream)))


def atlaskv_workspace_size_layers(trees, params: atlaskv_params, ios) -> int:
    n = len(trees)
    th = (ctypes.c_void_p * n)(*trees)
    io_arr = (atlaskv_io * n)(*ios)
    out = ctypes.c_size_t()
    _check(load_library().atlaskv_workspace_size_layers(n, th, ctypes.byref(params), io_arr, ctypes.byref(out)))
    return out.value


def atlaskv_attend_layers(trees, params: atlaskv_params, ios, workspace: int, workspace_bytes: int,
                          stream: int = 0) -> None:
    n = len(trees)
    th = (ctypes.c_void_p * n)(*trees)
    io_arr = (atlaskv_io * n)(*ios)
    _check(load_library().atlaskv_attend_layers(n, th, ctypes.byref(params), io_arr, ctypes.c_void_p(workspace),
                                                workspace_bytes, ctypes.c_void_p(stream)))


def atlaskv_create_tree_csr(desc: atlaskv_csr_tree_desc, stream: int = 0) -> int:
    handle = ctypes.c_void_p()
    _check(load_library().atlaskv_create_tree_csr(ctypes.byref(desc), ctypes.c_void_p(stream), ctypes.byref(handle)))
    return handle.value


def atlaskv_workspace_size_csr(tree: int, params: atlaskv_level_params, B: int, N: int, H: int, T: int) -> int:
    out = ctypes.c_size_t()
    _check(load_library().atlaskv_workspace_size_csr(ctypes.c_void_p(tree), ctypes.byref(params), B, N, H, T,
                                                     ctypes.byref(out)))
    return out.value


def atlaskv_attend_csr(tree: int, params: atlaskv_level_params, io: atlaskv_io, kept, workspace: int,
                       workspace_bytes: int, stream: int = 0) -> None:
    """kept: a list of n_levels device pointers (or None entries), or None."""
    arr = None if kept is None else (ctypes.c_void_p * len(kept))(*kept)
    _check(load_library().atlaskv_attend_csr(ctypes.c_void_p(tree), ctypes.byref(params), ctypes.byref(io), arr,
                                             ctypes.c_void_p(workspace), workspace_bytes, ctypes.c_void_p(stream)))


def atlaskv_sync_status(tree: int, stream: int = 0) -> None:
    _check(load_library().atlaskv_sync_status(ctypes.c_void_p(tree), ctypes.c_void_p(stream)))


def atlaskv_set_profiling(tree: int, enable: int) -> None:
    """enable: bit mask of ATLASKV_PROFILE_TIMES and ATLASKV_PROFILE_COUNTERS (0: off)."""
    _check(load_library().atlaskv_set_profiling(ctypes.c_void_p(tree), int(enable)))


def atlaskv_set_descent(tree: int, mode: int) -> None:
    """mode: ATLASKV_DESCENT_AUTO, ATLASKV_DESCENT_FUSED or ATLASKV_DESCENT_PARENT_MAJOR."""
    _check(load_library().atlaskv_set_descent(ctypes.c_void_p(tree), int(mode)))


def atlaskv_set_leaf_cache(tree: int, blocks: int, stream: int = 0) -> None:
    """HBM cache of `blocks` staged leaf-key blocks across calls (0: none)."""
    _check(load_library().atlaskv_set_leaf_cache(ctypes.c_void_p(tree), int(blocks), ctypes.c_void_p(stream)))


def atlaskv_leaf_cache_stats(tree: int):
    """Cumulative cache counters: dict(hits, fills, bypasses)."""
    out = (ctypes.c_uint64 * 3)()
    _check(load_library().atlaskv_leaf_cache_stats(ctypes.c_void_p(tree), out, 3))
    return {"hits": int(out[0]), "fills": int(out[1]), "bypasses": int(out[2])}


def atlaskv_stage_times(tree: int):
    """Stage times (ms) of the last timed call, in the order of STAGE_NAMES."""
    buf = (ctypes.c_float * 5)()
    _check(load_library().atlaskv_stage_times(ctypes.c_void_p(tree), buf, 5))
    return [float(x) for x in buf]


def atlaskv_refine_stats(tree: int):
    """Descent counters of the last profiled call: per level [selections,
    selections needing exact refinement, ambiguous candidates, exact scores]."""
    buf = (ctypes.c_uint64 * 16)()
    _check(load_library().atlaskv_refine_stats(ctypes.c_void_p(tree), buf, 16))
    v = [int(x) for x in buf]
    names = ("root", "mid", "leaf", "level3")
    return {names[i]: dict(zip(("selections", "refined", "ambiguous", "exact_scores"), v[4 * i:4 * i + 4]))
            for i in range(4) if i < 3 or v[4 * i] > 0}


def atlaskv_probe_wait_timeout(tree: int, stream: int = 0) -> None:
    _check(load_library().atlaskv_probe_wait_timeout(ctypes.c_void_p(tree), ctypes.c_void_p(stream)))


def atlaskv_destroy(tree: int) -> None:
    _check(load_library().atlaskv_destroy(ctypes.c_void_p(tree)))


# ---- torch-facing convenience ------------------------------------------------

def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return ATLASKV_F32
    if t == torch.bfloat16:
        return ATLASKV_BF16
    raise AtlaskvError(ATLASKV_EINVAL, "dtype %s not supported (float32 or bfloat16)" % t)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise AtlaskvError(ATLASKV_EINVAL, "tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


class HikvpTree:
    """A key tree registered with the library.  Holds references to the
    tensors it borrows; call ``close()`` (or use ``with``) to release."""

    def __init__(self, root_keys, mid_keys, leaf_keys, leaf_values, fanout, root_child=None, mid_child=None,
                 stream=None):
        self._keep = (root_keys, mid_keys, leaf_keys, leaf_values, root_child, mid_child)
        self.dtype = root_keys.dtype
        self.fanout = tuple(int(f) for f in fanout)
        self.n_kv_heads, _, self.head_dim = root_keys.shape
        on_host = not leaf_keys.is_cuda
        mids_on_host = not mid_keys.is_cuda
        if on_host and not (leaf_keys.is_pinned() and leaf_values.is_pinned()):
            raise AtlaskvError(ATLASKV_EINVAL, "host-resident leaves must be pinned tensors")
        if mids_on_host and not mid_keys.is_pinned():
            raise AtlaskvError(ATLASKV_EINVAL, "host-resident mid keys must be a pinned tensor")
        d = atlaskv_tree_desc()
        d.dtype = _dtype_code(self.dtype)
        d.n_kv_heads = self.n_kv_heads
        d.head_dim = self.head_dim
        d.fanout[:] = self.fanout
        d.root_keys, d.mid_keys = _ptr(root_keys), _ptr(mid_keys)
        d.leaf_keys, d.leaf_values = _ptr(leaf_keys), _ptr(leaf_values)
        d.leaf_location = ATLASKV_LEAVES_HOST_PINNED if on_host else ATLASKV_LEAVES_DEVICE
        d.root_child, d.mid_child = _ptr(root_child), _ptr(mid_child)
        d.mid_location = ATLASKV_LEAVES_HOST_PINNED if mids_on_host else ATLASKV_LEAVES_DEVICE
        self.desc = d
        self.handle = atlaskv_create_tree(d, _stream(stream))
        self.leaves_on_host = on_host
        self.mids_on_host = mids_on_host

    @classmethod
    def from_workload(cls, w, stream=None):
        return cls(w.root_keys, w.mid_keys, w.leaf_keys, w.leaf_values, w.shape.fanout, w.root_child, w.mid_child,
                   stream)

    def close(self):
        if getattr(self, "handle", None):
            atlaskv_destroy(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def params(self, K, scale: float = 0.0) -> atlaskv_params:
        return atlaskv_params(int(K[0]), int(K[1]), int(K[2]), float(scale))

    def workspace_size(self, K, B, N, H, T, scale: float = 0.0) -> int:
        return atlaskv_workspace_size(self.handle, self.params(K, scale), B, N, H, T)

    def attend(self, q_kg, q_seq, k_seq, v_seq, K, scale: float = 0.0, out=None, lse=None, kept=None,
               workspace=None, want_kept: bool = True, want_lse: bool = True, stream=None):
        """Enqueue the whole path.  Returns dict(out, lse, kept_root, kept_mid,
        kept_leaf) of device tensors (lse / kept_* None when not requested)."""
        B, N, H, D = q_kg.shape
        T = k_seq.shape[1]
        dev = q_kg.device
        p = self.params(K, scale)
        if out is None:
            out = torch.empty_like(q_kg)
        if want_lse and lse is None:
            lse = torch.empty((B, N, H), dtype=torch.float32, device=dev)
        if want_kept and kept is None:
            kept = tuple(torch.empty((B, H, int(k)), dtype=torch.int32, device=dev) for k in K)
        if kept is None:
            kept = (None, None, None)
        if workspace is None:
            nbytes = atlaskv_workspace_size(self.handle, p, B, N, H, T)
            workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        io = atlaskv_io(B, N, H, T, _ptr(q_kg), _ptr(q_seq), _ptr(k_seq), _ptr(v_seq), _ptr(out), _ptr(lse),
                        _ptr(kept[0]), _ptr(kept[1]), _ptr(kept[2]))
        atlaskv_attend(self.handle, p, io, workspace.data_ptr(), workspace.numel(), _stream(stream))
        return {"out": out, "lse": lse, "kept_root": kept[0], "kept_mid": kept[1], "kept_leaf": kept[2],
                "workspace": workspace}

    def sync_status(self, stream=None):
        atlaskv_sync_status(self.handle, _stream(stream))

    def probe_wait_timeout(self, stream=None):
        atlaskv_probe_wait_timeout(self.handle, _stream(stream))

    def set_profiling(self, times: bool = True, counters: bool = True):
        atlaskv_set_profiling(self.handle, (ATLASKV_PROFILE_TIMES if times else 0) |
                              (ATLASKV_PROFILE_COUNTERS if counters else 0))

    def set_descent(self, mode: int):
        """ATLASKV_DESCENT_AUTO, ATLASKV_DESCENT_FUSED or ATLASKV_DESCENT_PARENT_MAJOR (same results)."""
        atlaskv_set_descent(self.handle, mode)

    def set_leaf_cache(self, blocks: int, stream=None):
        """HBM cache of staged leaf blocks across calls (host-resident leaves; 0 removes it)."""
        atlaskv_set_leaf_cache(self.handle, blocks, _stream(stream))

    def leaf_cache_stats(self):
        return atlaskv_leaf_cache_stats(self.handle)

    def stage_times(self):
        return atlaskv_stage_times(self.handle)

    def refine_stats(self):
        return atlaskv_refine_stats(self.handle)


def attend_layers(trees, inputs, K, scale: float = 0.0, workspace=None, stream=None):
    """Several layers' calls in one batch (atlaskv_attend_layers).  trees: a
    HikvpTree per layer; inputs: per layer (q_kg, q_seq, k_seq, v_seq).
    Returns per layer dict(out, lse, kept_root, kept_mid, kept_leaf)."""
    outs, ios = [], []
    for tree, (q_kg, q_seq, k_seq, v_seq) in zip(trees, inputs):
        B, N, H, D = q_kg.shape
        T = k_seq.shape[1]
        dev = q_kg.device
        r = {"out": torch.empty_like(q_kg), "lse": torch.empty((B, N, H), dtype=torch.float32, device=dev)}
        for name, k in zip(("kept_root", "kept_mid", "kept_leaf"), K):
            r[name] = torch.empty((B, H, int(k)), dtype=torch.int32, device=dev)
        ios.append(atlaskv_io(B, N, H, T, _ptr(q_kg), _ptr(q_seq), _ptr(k_seq), _ptr(v_seq), _ptr(r["out"]),
                              _ptr(r["lse"]), _ptr(r["kept_root"]), _ptr(r["kept_mid"]), _ptr(r["kept_leaf"])))
        outs.append(r)
    p = trees[0].params(K, scale)
    handles = [t.handle for t in trees]
    if workspace is None:
        nbytes = atlaskv_workspace_size_layers(handles, p, ios)
        workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=inputs[0][0].device)
    atlaskv_attend_layers(handles, p, ios, workspace.data_ptr(), workspace.numel(), _stream(stream))
    for r in outs:
        r["workspace"] = workspace
    return outs


class CsrHikvpTree:
    """A CSR tree (any depth, variable numbers of children) registered with
    the library: keys[l] [H_kv][rows_l][D] per level, child_off[l]
    [H_kv][rows_l + 1], child_id[l] [H_kv][rows_{l+1}] or None, leaf values of
    the last level.  Holds references to the tensors it borrows."""

    def __init__(self, keys, leaf_values, child_off, child_id=None, stream=None):
        n = len(keys)
        child_id = child_id if child_id is not None else [None] * (n - 1)
        self._keep = (keys, leaf_values, child_off, child_id)
        self.n_levels = n
        self.dtype = keys[0].dtype
        self.n_kv_heads, _, self.head_dim = keys[0].shape
        d = atlaskv_csr_tree_desc()
        d.dtype = _dtype_code(self.dtype)
        d.n_kv_heads = self.n_kv_heads
        d.head_dim = self.head_dim
        d.n_levels = n
        for l, k in enumerate(keys):
            d.rows[l] = k.shape[1]
            d.keys[l] = _ptr(k)
        for l in range(n - 1):
            d.child_off[l] = _ptr(child_off[l])
            d.child_id[l] = _ptr(child_id[l])
        d.leaf_values = _ptr(leaf_values)
        self.desc = d
        self.handle = atlaskv_create_tree_csr(d, _stream(stream))

    @classmethod
    def from_workload(cls, w, stream=None):
        return cls(w.keys, w.leaf_values, w.child_off, w.child_id, stream)

    def close(self):
        if getattr(self, "handle", None):
            atlaskv_destroy(self.handle)
            self.handle = None

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def params(self, K, scale: float = 0.0) -> atlaskv_level_params:
        p = atlaskv_level_params()
        for l, k in enumerate(K):
            p.K[l] = int(k)
        p.scale = float(scale)
        return p

    def attend(self, q_kg, q_seq, k_seq, v_seq, K, scale: float = 0.0, workspace=None, stream=None):
        """Returns dict(out, lse, kept: a list of [B][H][K_l] per level)."""
        B, N, H, D = q_kg.shape
        T = k_seq.shape[1]
        dev = q_kg.device
        p = self.params(K, scale)
        out = torch.empty_like(q_kg)
        lse = torch.empty((B, N, H), dtype=torch.float32, device=dev)
        kept = [torch.empty((B, H, int(k)), dtype=torch.int32, device=dev) for k in K]
        if workspace is None:
            nbytes = atlaskv_workspace_size_csr(self.handle, p, B, N, H, T)
            workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        io = atlaskv_io(B, N, H, T, _ptr(q_kg), _ptr(q_seq), _ptr(k_seq), _ptr(v_seq), _ptr(out), _ptr(lse),
                        None, None, None)
        atlaskv_attend_csr(self.handle, p, io, [k.data_ptr() for k in kept], workspace.data_ptr(), workspace.numel(),
                           _stream(stream))
        return {"out": out, "lse": lse, "kept": kept, "workspace": workspace}

    def sync_status(self, stream=None):
        atlaskv_sync_status(self.handle, _stream(stream))

    def set_profiling(self, times: bool = True, counters: bool = True):
        atlaskv_set_profiling(self.handle, (ATLASKV_PROFILE_TIMES if times else 0) |
                              (ATLASKV_PROFILE_COUNTERS if counters else 0))

    def set_descent(self, mode: int):
        """ATLASKV_DESCENT_AUTO, ATLASKV_DESCENT_FUSED or ATLASKV_DESCENT_PARENT_MAJOR (same results)."""
        atlaskv_set_descent(self.handle, mode)

    def refine_stats(self):
        return atlaskv_refine_stats(self.handle)
