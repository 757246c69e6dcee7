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

# Every symbol include/atlaskv.h declares.
EXPORTED = ("atlaskv_create_tree", "atlaskv_workspace_size", "atlaskv_attend", "atlaskv_sync_status",
            "atlaskv_set_profiling", "atlaskv_stage_times", "atlaskv_refine_stats", "atlaskv_attend_static",
            "atlaskv_probe_wait_timeout", "atlaskv_destroy", "atlaskv_last_error")
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
    ]


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
            lib.atlaskv_sync_status.argtypes = [V, V]
            lib.atlaskv_set_profiling.argtypes = [V, I32]
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


def atlaskv_sync_status(tree: int, stream: int = 0) -> None:
    _check(load_library().atlaskv_sync_status(ctypes.c_void_p(tree), ctypes.c_void_p(stream)))


def atlaskv_set_profiling(tree: int, enable: bool) -> None:
    _check(load_library().atlaskv_set_profiling(ctypes.c_void_p(tree), int(bool(enable))))


def atlaskv_stage_times(tree: int):
    buf = (ctypes.c_float * 3)()
    _check(load_library().atlaskv_stage_times(ctypes.c_void_p(tree), buf, 3))
    return [float(x) for x in buf]


def atlaskv_refine_stats(tree: int):
    """Descent counters of the last profiled call: per level [selections,
    selections needing exact refinement, ambiguous candidates, exact scores]."""
    buf = (ctypes.c_uint64 * 12)()
    _check(load_library().atlaskv_refine_stats(ctypes.c_void_p(tree), buf, 12))
    v = [int(x) for x in buf]
    return {lvl: dict(zip(("selections", "refined", "ambiguous", "exact_scores"), v[4 * i:4 * i + 4]))
            for i, lvl in enumerate(("root", "mid", "leaf"))}


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
        if on_host and not (leaf_keys.is_pinned() and leaf_values.is_pinned()):
            raise AtlaskvError(ATLASKV_EINVAL, "host-resident leaves must be pinned tensors")
        d = atlaskv_tree_desc()
        d.dtype = _dtype_code(self.dtype)
        d.n_kv_heads = self.n_kv_heads
        d.head_dim = self.head_dim
        d.fanout[:] = self.fanout
        d.root_keys, d.mid_keys = _ptr(root_keys), _ptr(mid_keys)
        d.leaf_keys, d.leaf_values = _ptr(leaf_keys), _ptr(leaf_values)
        d.leaf_location = ATLASKV_LEAVES_HOST_PINNED if on_host else ATLASKV_LEAVES_DEVICE
        d.root_child, d.mid_child = _ptr(root_child), _ptr(mid_child)
        self.desc = d
        self.handle = atlaskv_create_tree(d, _stream(stream))
        self.leaves_on_host = on_host

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

    def set_profiling(self, enable: bool):
        atlaskv_set_profiling(self.handle, enable)

    def stage_times(self):
        return atlaskv_stage_times(self.handle)

    def refine_stats(self):
        return atlaskv_refine_stats(self.handle)
