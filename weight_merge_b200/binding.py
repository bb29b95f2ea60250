"""ctypes binding of ``libadafuse.so``: same names as the C ABI, marshalling only.

The functions take raw integers for device pointers and streams (for example
``tensor.data_ptr()`` and ``torch.cuda.current_stream().cuda_stream``); the
``Switcher`` helper below builds the model descriptor from torch tensors.
There is no fallback path: if the compiled library is missing or cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))

ADAFUSE_OK = 0
ADAFUSE_ERR_INVALID_ARG = -1
ADAFUSE_ERR_UNSUPPORTED_SHAPE = -2
ADAFUSE_ERR_CUDA = -3
ADAFUSE_ERR_DEVICE_FAULT = -4
ADAFUSE_ERR_UNSUPPORTED_DEVICE = -5
ADAFUSE_ERR_OUT_OF_MEMORY = -6
ADAFUSE_STATUS_BAD_EXPERT = 0x1
ADAFUSE_STATUS_BAD_GATE = 0x2
ADAFUSE_STATUS_TIMEOUT = 0x4
ADAFUSE_KERNEL_AUTO = 0
ADAFUSE_KERNEL_MMA_SYNC = 1
ADAFUSE_KERNEL_TCGEN05 = 2
ADAFUSE_KERNEL_TCGEN05_PAIR = 3
ADAFUSE_KERNEL_TCGEN05_FOLD = 4
ADAFUSE_SCHEDULE_STATIC = 0
ADAFUSE_SCHEDULE_DYNAMIC = 1
ADAFUSE_SCHEDULE_AUTO = 2
ADAFUSE_MAPS_NONE = 0
ADAFUSE_MAPS_PLAIN = 1
ADAFUSE_MAPS_BLOCKED = 2
ADAFUSE_MAX_TOP_K = 4
ADAFUSE_MAX_BATCH_TOKENS = 4096


class AdafuseError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {adafuse_strerror(code)} ({code})"
        if code == ADAFUSE_ERR_CUDA:
            msg += f": {adafuse_last_error()}"
        super().__init__(msg)


class Route(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_int32 * 2), ("gate", ctypes.c_float * 2)]


class Route4(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_int32 * 4), ("gate", ctypes.c_float * 4)]


class Target(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("out", ctypes.c_int64), ("in_", ctypes.c_int64),
                ("W", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p)]


class Desc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("n_targets", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("targets", ctypes.POINTER(Target))]


_lib = None


def library_path() -> str:
    return os.path.join(_PKG, "libadafuse.so")


def lib() -> ctypes.CDLL:
    """Load the compiled library (raises if it is missing: no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m weight_merge_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(path)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "adafuse_create": ([ctypes.POINTER(P), ctypes.POINTER(Desc), ctypes.c_int], ctypes.c_int),
        "adafuse_destroy": ([P], ctypes.c_int),
        "adafuse_pregate": ([P, P, i64, i64, P, P, P], ctypes.c_int),
        "adafuse_switch": ([P, P, P, P], ctypes.c_int),
        "adafuse_switch_batch_layers": ([P, i32, i32, P, P, P], ctypes.c_int),
        "adafuse_get_device_status": ([P, P, ctypes.POINTER(i32)], ctypes.c_int),
        "adafuse_set_switch_kernel": ([P, ctypes.c_int], ctypes.c_int),
        "adafuse_set_tile_schedule": ([P, ctypes.c_int], ctypes.c_int),
        "adafuse_set_max_ctas": ([P, i32], ctypes.c_int),
        "adafuse_get_topk_switch_kernel": ([P], ctypes.c_int),
        "adafuse_set_base": ([P, ctypes.POINTER(P)], ctypes.c_int),
        "adafuse_rebase": ([P, P, P], ctypes.c_int),
        "adafuse_rebase_layers": ([P, i32, i32, P, P], ctypes.c_int),
        "adafuse_get_switch_kernel": ([P], ctypes.c_int),
        "adafuse_get_tensor_map_layout": ([P], ctypes.c_int),
        "adafuse_pregate_topk": ([P, P, i64, i64, P, i32, P, P], ctypes.c_int),
        "adafuse_pregate_batch": ([P, P, i64, i64, P, P, P], ctypes.c_int),
        "adafuse_pregate_batch_topk": ([P, P, i64, i64, P, i32, P, P], ctypes.c_int),
        "adafuse_switch_topk": ([P, P, P, P], ctypes.c_int),
        "adafuse_switch_topk_layers": ([P, i32, i32, P, P, P], ctypes.c_int),
        "adafuse_rebase_topk": ([P, P, P], ctypes.c_int),
        "adafuse_debug_stall_next_switch": ([P], ctypes.c_int),
        "adafuse_debug_stall_next_switch_at": ([P, i32], ctypes.c_int),
        "adafuse_refresh_adapters": ([P, P], ctypes.c_int),
        "adafuse_segment_table": ([ctypes.POINTER(Desc), P, i64, ctypes.POINTER(i64)], ctypes.c_int),
        "adafuse_tile_size": ([], ctypes.c_int),
        "adafuse_strerror": ([ctypes.c_int], ctypes.c_char_p),
        "adafuse_last_error": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _check(code: int, where: str) -> int:
    if code != ADAFUSE_OK:
        raise AdafuseError(code, where)
    return code


# ---- the C entry points, one to one --------------------------------------

def adafuse_strerror(code: int) -> str:
    return lib().adafuse_strerror(int(code)).decode()


def adafuse_last_error() -> str:
    return lib().adafuse_last_error().decode()


def adafuse_tile_size() -> int:
    return lib().adafuse_tile_size()


def adafuse_create(desc: Desc, device: int) -> int:
    """Returns the context handle (an integer)."""
    h = ctypes.c_void_p()
    _check(lib().adafuse_create(ctypes.byref(h), ctypes.byref(desc), int(device)), "adafuse_create")
    return h.value


def adafuse_destroy(ctx: Optional[int]) -> None:
    _check(lib().adafuse_destroy(ctx), "adafuse_destroy")


def adafuse_pregate(ctx: int, h: int, T: int, d: int, Wr: int, route: int, stream: int = 0) -> None:
    _check(lib().adafuse_pregate(ctx, h, int(T), int(d), Wr, route, stream or None), "adafuse_pregate")


def adafuse_switch(ctx: int, prev: Optional[int], cur: Optional[int], stream: int = 0) -> None:
    _check(lib().adafuse_switch(ctx, prev or None, cur or None, stream or None), "adafuse_switch")


def adafuse_switch_batch_layers(ctx: int, layer_begin: int, n_layers: int, prev: Optional[int],
                                cur: Optional[int], stream: int = 0) -> None:
    _check(lib().adafuse_switch_batch_layers(ctx, int(layer_begin), int(n_layers), prev or None,
                                             cur or None, stream or None),
           "adafuse_switch_batch_layers")


def adafuse_set_base(ctx: int, W0: Sequence[int]) -> None:
    arr = (ctypes.c_void_p * len(W0))(*W0)
    _check(lib().adafuse_set_base(ctx, arr), "adafuse_set_base")


def adafuse_rebase(ctx: int, cur: Optional[int], stream: int = 0) -> None:
    _check(lib().adafuse_rebase(ctx, cur or None, stream or None), "adafuse_rebase")


def adafuse_rebase_layers(ctx: int, layer_begin: int, n_layers: int, cur: Optional[int],
                          stream: int = 0) -> None:
    _check(lib().adafuse_rebase_layers(ctx, int(layer_begin), int(n_layers), cur or None,
                                       stream or None), "adafuse_rebase_layers")


def adafuse_pregate_topk(ctx: int, h: int, T: int, d: int, Wr: int, k: int, route: int,
                         stream: int = 0) -> None:
    _check(lib().adafuse_pregate_topk(ctx, h, int(T), int(d), Wr, int(k), route, stream or None),
           "adafuse_pregate_topk")


def adafuse_pregate_batch(ctx: int, h: int, T: int, d: int, Wr: int, route: int,
                          stream: int = 0) -> None:
    _check(lib().adafuse_pregate_batch(ctx, h, int(T), int(d), Wr, route, stream or None),
           "adafuse_pregate_batch")


def adafuse_pregate_batch_topk(ctx: int, h: int, T: int, d: int, Wr: int, k: int, route: int,
                               stream: int = 0) -> None:
    _check(lib().adafuse_pregate_batch_topk(ctx, h, int(T), int(d), Wr, int(k), route,
                                            stream or None), "adafuse_pregate_batch_topk")


def adafuse_switch_topk(ctx: int, prev: Optional[int], cur: Optional[int], stream: int = 0) -> None:
    _check(lib().adafuse_switch_topk(ctx, prev or None, cur or None, stream or None),
           "adafuse_switch_topk")


def adafuse_switch_topk_layers(ctx: int, layer_begin: int, n_layers: int, prev: Optional[int],
                               cur: Optional[int], stream: int = 0) -> None:
    _check(lib().adafuse_switch_topk_layers(ctx, int(layer_begin), int(n_layers), prev or None,
                                            cur or None, stream or None),
           "adafuse_switch_topk_layers")


def adafuse_rebase_topk(ctx: int, cur: Optional[int], stream: int = 0) -> None:
    _check(lib().adafuse_rebase_topk(ctx, cur or None, stream or None), "adafuse_rebase_topk")


def adafuse_refresh_adapters(ctx: int, stream: int = 0) -> None:
    _check(lib().adafuse_refresh_adapters(ctx, stream or None), "adafuse_refresh_adapters")


def adafuse_debug_stall_next_switch(ctx: int) -> None:
    _check(lib().adafuse_debug_stall_next_switch(ctx), "adafuse_debug_stall_next_switch")


def adafuse_debug_stall_next_switch_at(ctx: int, tile: int) -> None:
    _check(lib().adafuse_debug_stall_next_switch_at(ctx, int(tile)),
           "adafuse_debug_stall_next_switch_at")


def adafuse_set_switch_kernel(ctx: int, kernel: int) -> None:
    _check(lib().adafuse_set_switch_kernel(ctx, int(kernel)), "adafuse_set_switch_kernel")


def adafuse_set_tile_schedule(ctx: int, schedule: int) -> None:
    _check(lib().adafuse_set_tile_schedule(ctx, int(schedule)), "adafuse_set_tile_schedule")


def adafuse_set_max_ctas(ctx: int, max_ctas: int) -> None:
    _check(lib().adafuse_set_max_ctas(ctx, int(max_ctas)), "adafuse_set_max_ctas")


def adafuse_get_topk_switch_kernel(ctx: int) -> int:
    k = lib().adafuse_get_topk_switch_kernel(ctx)
    if k < 0:
        _check(k, "adafuse_get_topk_switch_kernel")
    return k


def adafuse_get_switch_kernel(ctx: int) -> int:
    k = lib().adafuse_get_switch_kernel(ctx)
    if k < 0:
        raise AdafuseError(k, "adafuse_get_switch_kernel")
    return k


def adafuse_get_tensor_map_layout(ctx: int) -> int:
    k = lib().adafuse_get_tensor_map_layout(ctx)
    if k < 0:
        raise AdafuseError(k, "adafuse_get_tensor_map_layout")
    return k


def adafuse_get_device_status(ctx: int, stream: int = 0, raise_on_fault: bool = False) -> int:
    v = ctypes.c_int32(0)
    code = lib().adafuse_get_device_status(ctx, stream or None, ctypes.byref(v))
    if code not in (ADAFUSE_OK, ADAFUSE_ERR_DEVICE_FAULT) or (raise_on_fault and code != ADAFUSE_OK):
        raise AdafuseError(code, "adafuse_get_device_status")
    return v.value


def adafuse_segment_table(desc: Desc):
    """Host-only: the (layer, target, row0, col0) tiles the context would use."""
    import numpy as np
    n = ctypes.c_int64(0)
    _check(lib().adafuse_segment_table(ctypes.byref(desc), None, 0, ctypes.byref(n)),
           "adafuse_segment_table")
    out = np.empty((n.value, 4), dtype=np.int32)
    _check(lib().adafuse_segment_table(ctypes.byref(desc), out.ctypes.data_as(ctypes.c_void_p),
                                       n.value, ctypes.byref(n)), "adafuse_segment_table")
    return out


# ---- descriptor helper ----------------------------------------------------

def make_desc(n_layers: int, n_targets: int, n_experts: int, rank: int, alpha: float,
              targets: Sequence[tuple]) -> Desc:
    """targets: (name, out, in, W_ptr, A_ptr, B_ptr) per (layer, target), layer-major.
    The returned Desc keeps its target array alive."""
    arr = (Target * len(targets))()
    names = []
    for i, (name, out, inn, W, A, B) in enumerate(targets):
        nb = name.encode() if isinstance(name, str) else name
        names.append(nb)
        arr[i] = Target(nb, int(out), int(inn), W, A, B)
    d = Desc(int(n_layers), int(n_targets), int(n_experts), int(rank), float(alpha),
             ctypes.cast(arr, ctypes.POINTER(Target)))
    d._keep = (arr, names)
    return d


class Switcher:
    """Owns one context built from torch tensors (W, A, B lists, layer-major).

    switcher.pregate(h, Wr, routes)          -> adafuse_pregate
    switcher.switch(prev, cur)               -> adafuse_switch
    switcher.switch_layers(l0, n, prev, cur) -> adafuse_switch_batch_layers
    prev / cur are single-route views of an int32 [T, 4]-shaped route buffer
    (or None); see ``route_ptr``.
    """

    def __init__(self, W, A, B, n_layers: int, n_targets: int, n_experts: int, rank: int,
                 alpha: float, device: int = 0, names: Optional[Sequence[str]] = None):
        ts = []
        for i, (w, a, b) in enumerate(zip(W, A, B)):
            name = names[i % n_targets] if names else f"t{i % n_targets}"
            ts.append((name, w.shape[0], w.shape[1], w.data_ptr(), a.data_ptr(), b.data_ptr()))
        self._tensors = (list(W), list(A), list(B))
        self.desc = make_desc(n_layers, n_targets, n_experts, rank, alpha, ts)
        self.n_layers = n_layers
        self.ctx = adafuse_create(self.desc, device)

    @staticmethod
    def route_ptr(routes, t: Optional[int]) -> Optional[int]:
        """Device address of route t of a [T, 4] int32 route buffer (None -> None)."""
        if t is None or routes is None:
            return None
        return routes.data_ptr() + 16 * int(t)

    def pregate(self, h, Wr, routes, stream: int = 0) -> None:
        T, d = h.shape
        adafuse_pregate(self.ctx, h.data_ptr(), T, d, Wr.data_ptr(), routes.data_ptr(), stream)

    def switch(self, prev: Optional[int], cur: Optional[int], stream: int = 0) -> None:
        adafuse_switch(self.ctx, prev, cur, stream)

    def switch_layers(self, layer_begin: int, n_layers: int, prev: Optional[int],
                      cur: Optional[int], stream: int = 0) -> None:
        adafuse_switch_batch_layers(self.ctx, layer_begin, n_layers, prev, cur, stream)

    def set_base(self, W0) -> None:
        """W0: list of tensors (pristine copies of W, same order); kept alive here."""
        self._base = list(W0)
        adafuse_set_base(self.ctx, [w.data_ptr() for w in self._base])

    def rebase(self, cur: Optional[int], stream: int = 0) -> None:
        adafuse_rebase(self.ctx, cur, stream)

    def rebase_layers(self, layer_begin: int, n_layers: int, cur: Optional[int],
                      stream: int = 0) -> None:
        adafuse_rebase_layers(self.ctx, layer_begin, n_layers, cur, stream)

    @staticmethod
    def route4_ptr(routes, t: Optional[int]) -> Optional[int]:
        """Device address of route t of a [T, 8] int32 top-k route buffer."""
        if t is None or routes is None:
            return None
        return routes.data_ptr() + 32 * int(t)

    def pregate_topk(self, h, Wr, k: int, routes, stream: int = 0) -> None:
        T, d = h.shape
        adafuse_pregate_topk(self.ctx, h.data_ptr(), T, d, Wr.data_ptr(), k, routes.data_ptr(),
                             stream)

    def pregate_batch(self, h, Wr, route, stream: int = 0) -> None:
        """One top-2 route for the whole batch h [T, d] into ``route`` (one
        16-byte record, e.g. a row of an int32 [n, 4] buffer)."""
        T, d = h.shape
        adafuse_pregate_batch(self.ctx, h.data_ptr(), T, d, Wr.data_ptr(), route.data_ptr(), stream)

    def pregate_batch_topk(self, h, Wr, k: int, route, stream: int = 0) -> None:
        T, d = h.shape
        adafuse_pregate_batch_topk(self.ctx, h.data_ptr(), T, d, Wr.data_ptr(), k,
                                   route.data_ptr(), stream)

    def switch_topk(self, prev: Optional[int], cur: Optional[int], stream: int = 0) -> None:
        adafuse_switch_topk(self.ctx, prev, cur, stream)

    def switch_topk_layers(self, layer_begin: int, n_layers: int, prev: Optional[int],
                           cur: Optional[int], stream: int = 0) -> None:
        adafuse_switch_topk_layers(self.ctx, layer_begin, n_layers, prev, cur, stream)

    def rebase_topk(self, cur: Optional[int], stream: int = 0) -> None:
        adafuse_rebase_topk(self.ctx, cur, stream)

    def set_kernel(self, kernel: int) -> None:
        adafuse_set_switch_kernel(self.ctx, kernel)

    def set_schedule(self, schedule: int) -> None:
        adafuse_set_tile_schedule(self.ctx, schedule)

    def set_max_ctas(self, max_ctas: int) -> None:
        adafuse_set_max_ctas(self.ctx, max_ctas)

    @property
    def kernel(self) -> int:
        return adafuse_get_switch_kernel(self.ctx)

    @property
    def map_layout(self) -> int:
        return adafuse_get_tensor_map_layout(self.ctx)

    @property
    def topk_kernel(self) -> int:
        return adafuse_get_topk_switch_kernel(self.ctx)

    def status(self, stream: int = 0) -> int:
        return adafuse_get_device_status(self.ctx, stream)

    def close(self) -> None:
        if self.ctx:
            adafuse_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
