"""Thin Python binding of the C ABI in ``include/tri.h`` (ctypes).

Argument marshalling only: every step of the pass runs in the CUDA library
``lib/libtri_b200.so``. Importing this module loads that library and fails
loudly if it is missing; there is no fallback of any kind.

The module-level functions carry the C names (``tri_create``, ``tri_prune`` ...)
and take raw handles; :class:`TriContext` wraps them for torch tensors.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libtri_b200.so")

TRI_OK, TRI_EINVAL, TRI_ENOMEM, TRI_ECUDA, TRI_ESTATE, TRI_EDEVICE, TRI_EUNSUPPORTED = range(7)
TRI_ROPE_HALF, TRI_ROPE_INTERLEAVED = 0, 1
TRI_OFFSETS_MEAN, TRI_OFFSETS_MAX = 0, 1
TRI_ENGINE_AUTO, TRI_ENGINE_CUDA_CORES, TRI_ENGINE_TENSOR = 0, 1, 2
TRI_DEV_NONE, TRI_DEV_LEN_GT_CAP, TRI_DEV_BAD_PAGE, TRI_DEV_TIMEOUT, TRI_DEV_INTERNAL, TRI_DEV_T_NOT_AFTER_POS = range(6)


class tri_kv(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_void_p),
        ("V", ctypes.c_void_p),
        ("pos", ctypes.c_void_p),
        ("lens", ctypes.c_void_p),
        ("lens_out", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("cap", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("max_pages", ctypes.c_int32),
        ("n_pages", ctypes.c_int32),
        ("layer_begin", ctypes.c_int32),
        ("n_layers", ctypes.c_int32),
    ]


class TriError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_str(status)}" + (f" [{detail}]" if detail else ""))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"the CUDA library {LIB_PATH} is missing; build it with "
            "`python -m rope_aware_key_tri_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    L.tri_create.argtypes = [ctypes.POINTER(P), ctypes.c_int]
    L.tri_destroy.argtypes = [P]
    L.tri_calibrate_load.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, D,
                                     ctypes.c_int, P, P, P, P, ctypes.c_int]
    L.tri_prune.argtypes = [P, ctypes.POINTER(tri_kv), P, I32, P]
    L.tri_prune_noalloc.argtypes = [P, ctypes.POINTER(tri_kv), P, I32, P]
    L.tri_score.argtypes = [P, ctypes.POINTER(tri_kv), P, P, P, P]
    L.tri_calibrate_estimate.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, P, P, P, P]
    L.tri_append.argtypes = [P, ctypes.POINTER(tri_kv), P, P, P, P]
    L.tri_append_advance.argtypes = [P, ctypes.POINTER(tri_kv), P, P, P, P]
    L.tri_get_error.argtypes = [P, P, ctypes.POINTER(I32), ctypes.POINTER(I64)]
    L.tri_get_failed_units.argtypes = [P, P, P, I32, ctypes.POINTER(I32)]
    L.tri_decode_attention.argtypes = [P, ctypes.POINTER(tri_kv), P, P, P]
    L.tri_set_test_fault.argtypes = [P, I64, I32]
    L.tri_set_tuning.argtypes = [P, ctypes.c_int, ctypes.c_int]
    L.tri_set_offset_combine.argtypes = [P, ctypes.c_int]
    L.tri_set_score_engine.argtypes = [P, ctypes.c_int]
    L.tri_last_error.argtypes = [P]
    L.tri_last_error.restype = ctypes.c_char_p
    L.tri_status_str.argtypes = [ctypes.c_int]
    L.tri_status_str.restype = ctypes.c_char_p
    for fn in ("tri_create", "tri_destroy", "tri_calibrate_load", "tri_prune", "tri_prune_noalloc", "tri_score",
               "tri_calibrate_estimate", "tri_append", "tri_append_advance", "tri_get_error", "tri_set_tuning",
               "tri_set_offset_combine",
               "tri_get_failed_units", "tri_set_test_fault", "tri_decode_attention", "tri_set_score_engine",
               "tri_version"):
        getattr(L, fn).restype = ctypes.c_int
    return L


_lib = _load()


def library():
    return _lib


def status_str(st: int) -> str:
    return _lib.tri_status_str(int(st)).decode()


# ---- raw C names -----------------------------------------------------------------------

def tri_version() -> int:
    return _lib.tri_version()


def tri_status_str(st: int) -> str:
    return status_str(st)


def tri_create(device: int = 0) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    st = _lib.tri_create(ctypes.byref(h), int(device))
    if st != TRI_OK:
        raise TriError(st, "tri_create")
    return h


def tri_destroy(ctx) -> int:
    return _lib.tri_destroy(ctx)


def tri_calibrate_load(ctx, n_layers, n_kv_heads, group, head_dim, rope_base, layout,
                       q_mean, q_norm_mean, R, offsets) -> int:
    qm = np.ascontiguousarray(q_mean, dtype=np.float32)
    qn = np.ascontiguousarray(q_norm_mean, dtype=np.float32)
    rr = np.ascontiguousarray(R, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int64)
    return _lib.tri_calibrate_load(ctx, int(n_layers), int(n_kv_heads), int(group), int(head_dim),
                                   float(rope_base), int(layout), qm.ctypes.data, qn.ctypes.data,
                                   rr.ctypes.data, off.ctypes.data, int(off.shape[0]))


def tri_prune(ctx, kv: tri_kv, t_ptr: int, budget: int, stream: int) -> int:
    return _lib.tri_prune(ctx, ctypes.byref(kv), t_ptr, int(budget), stream)


def tri_prune_noalloc(ctx, kv: tri_kv, t_ptr: int, budget: int, stream: int) -> int:
    return _lib.tri_prune_noalloc(ctx, ctypes.byref(kv), t_ptr, int(budget), stream)


def tri_score(ctx, kv: tri_kv, t_ptr: int, raw_ptr: int, zmax_ptr: int, stream: int) -> int:
    return _lib.tri_score(ctx, ctypes.byref(kv), t_ptr, raw_ptr, zmax_ptr, stream)


def tri_calibrate_estimate(ctx, q_ptr: int, n_layers: int, T: int, n_q_heads: int, head_dim: int, layout: int,
                           q_mean_ptr: int, q_norm_mean_ptr: int, R_ptr: int, stream: int) -> int:
    return _lib.tri_calibrate_estimate(ctx, q_ptr, int(n_layers), int(T), int(n_q_heads), int(head_dim),
                                       int(layout), q_mean_ptr, q_norm_mean_ptr, R_ptr, stream)


def tri_decode_attention(ctx, kv: tri_kv, q_ptr: int, out_ptr: int, stream: int) -> int:
    return _lib.tri_decode_attention(ctx, ctypes.byref(kv), q_ptr, out_ptr, stream)


def tri_append(ctx, kv: tri_kv, k_new_ptr: int, v_new_ptr: int, pos_new_ptr: int, stream: int) -> int:
    return _lib.tri_append(ctx, ctypes.byref(kv), k_new_ptr, v_new_ptr, pos_new_ptr, stream)


def tri_append_advance(ctx, kv: tri_kv, k_new_ptr: int, v_new_ptr: int, pos_ptr: int, stream: int) -> int:
    return _lib.tri_append_advance(ctx, ctypes.byref(kv), k_new_ptr, v_new_ptr, pos_ptr, stream)


def tri_get_error(ctx, stream: int):
    code = ctypes.c_int32()
    unit = ctypes.c_int64()
    st = _lib.tri_get_error(ctx, stream, ctypes.byref(code), ctypes.byref(unit))
    return st, code.value, unit.value


def tri_get_failed_units(ctx, stream: int, capacity: int = 4096):
    """(status, total count, list of unit indices) of units left uncompacted by unit-level failures."""
    buf = (ctypes.c_int32 * max(1, capacity))()
    n = ctypes.c_int32()
    st = _lib.tri_get_failed_units(ctx, stream, buf, int(capacity), ctypes.byref(n))
    return st, n.value, [buf[i] for i in range(min(n.value, capacity))]


def tri_set_test_fault(ctx, unit: int = -1, wait_tries: int = 0) -> int:
    return _lib.tri_set_test_fault(ctx, int(unit), int(wait_tries))


def tri_last_error(ctx) -> str:
    r = _lib.tri_last_error(ctx)
    return r.decode() if r else ""


def tri_set_tuning(ctx, cluster_size: int = 0, buffers_per_warp: int = 0) -> int:
    return _lib.tri_set_tuning(ctx, int(cluster_size), int(buffers_per_warp))


def tri_set_offset_combine(ctx, combine: int) -> int:
    return _lib.tri_set_offset_combine(ctx, int(combine))


def tri_set_score_engine(ctx, engine: int) -> int:
    return _lib.tri_set_score_engine(ctx, int(engine))


# ---- torch-facing wrapper ----------------------------------------------------------------

def _ptr(x: Optional[torch.Tensor]) -> Optional[int]:
    return None if x is None else x.data_ptr()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check_t(t, lens):
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous() or t.shape != lens.shape:
        raise ValueError(f"t must be a contiguous CUDA int32 tensor shaped like lens {tuple(lens.shape)}")


def make_kv(K, V, pos, lens, lens_out=None, block_table=None, n_pages=None, layer_begin=0) -> tri_kv:
    """Describe a cache held in torch tensors.

    Dense: K, V bf16 [L][batch][Hkv][cap][d], pos int32 [L][batch][Hkv][cap].
    Paged: K, V bf16 [L][pages][Hkv][page_size][d], pos int32 [L][pages][Hkv][page_size],
           block_table int32 [batch][max_pages].
    """
    for name, x, dt in (("K", K, torch.bfloat16), ("V", V, torch.bfloat16), ("pos", pos, torch.int32),
                        ("lens", lens, torch.int32), ("lens_out", lens_out, torch.int32),
                        ("block_table", block_table, torch.int32)):
        if x is None:
            continue
        if x.dtype != dt or not x.is_cuda or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor of {dt}")
    # the C ABI sees plain pointers: check here that every buffer holds what the call describes
    batch = int(lens.shape[0])
    if K.dim() != 5 or (V is not None and V.shape != K.shape):
        raise ValueError("K (and V) must be 5-D: [L][batch][Hkv][cap][d] dense or [L][pages][Hkv][page][d] paged")
    if pos is not None and tuple(pos.shape) != tuple(K.shape[:4]):
        raise ValueError(f"pos must be {tuple(K.shape[:4])}, got {tuple(pos.shape)}")
    if block_table is None and int(K.shape[1]) != batch:
        raise ValueError(f"dense cache holds {int(K.shape[1])} sequences, lens describes {batch}")
    if block_table is not None and (block_table.dim() != 2 or int(block_table.shape[0]) != batch):
        raise ValueError(f"block_table must be [batch={batch}][max_pages]")
    kv = tri_kv()
    kv.K, kv.V, kv.pos = _ptr(K), _ptr(V), _ptr(pos)
    kv.lens, kv.lens_out, kv.block_table = _ptr(lens), _ptr(lens_out), _ptr(block_table)
    kv.batch = int(lens.shape[0])
    kv.layer_begin = int(layer_begin)
    kv.n_layers = int(K.shape[0])
    if block_table is None:
        kv.cap = int(K.shape[3])
    else:
        kv.page_size = int(K.shape[3])
        kv.max_pages = int(block_table.shape[1])
        kv.n_pages = int(K.shape[1]) if n_pages is None else int(n_pages)
    return kv


class TriContext:
    """One library context on one CUDA device."""

    def __init__(self, device: int = 0):
        self.device = int(device)
        self.handle = tri_create(self.device)

    def close(self):
        if self.handle is not None:
            tri_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def calibrate_load(self, n_layers, n_kv_heads, group, head_dim, rope_base, layout,
                       q_mean, q_norm_mean, R, offsets):
        st = tri_calibrate_load(self.handle, n_layers, n_kv_heads, group, head_dim, rope_base, layout,
                                q_mean, q_norm_mean, R, offsets)
        if st != TRI_OK:
            raise TriError(st, "tri_calibrate_load")

    def set_offset_combine(self, combine):
        """"mean" (the default) or "max" over the future offsets (or the TRI_OFFSETS_* value)."""
        code = {"mean": TRI_OFFSETS_MEAN, "max": TRI_OFFSETS_MAX}.get(combine, combine)
        st = tri_set_offset_combine(self.handle, code)
        if st != TRI_OK:
            raise TriError(st, "tri_set_offset_combine")

    def set_score_engine(self, engine):
        """"auto" (the default), "cuda_cores" or "tensor" (or the TRI_ENGINE_* value)."""
        code = {"auto": TRI_ENGINE_AUTO, "cuda_cores": TRI_ENGINE_CUDA_CORES, "tensor": TRI_ENGINE_TENSOR}.get(
            engine, engine)
        st = tri_set_score_engine(self.handle, code)
        if st != TRI_OK:
            raise TriError(st, "tri_set_score_engine")

    def set_tuning(self, cluster_size=0, buffers_per_warp=0):
        st = tri_set_tuning(self.handle, cluster_size, buffers_per_warp)
        if st != TRI_OK:
            raise TriError(st, "tri_set_tuning")

    def prune(self, K, V, pos, lens, t, budget, lens_out="inplace", block_table=None,
              layer_begin=0, stream=None, check=True):
        if isinstance(lens_out, str):
            lens_out = lens
        kv = make_kv(K, V, pos, lens, lens_out, block_table, layer_begin=layer_begin)
        _check_t(t, lens)
        st = tri_prune(self.handle, kv, t.data_ptr(), budget, _stream_handle(stream))
        if check and st != TRI_OK:
            raise TriError(st, "tri_prune", tri_last_error(self.handle))
        return st

    def prune_noalloc(self, K, V, pos, lens, t, budget, lens_out="inplace", block_table=None,
                      layer_begin=0, stream=None, check=True):
        """tri_prune_noalloc: the same prune with fixed, library-held scratch (no allocation)."""
        if isinstance(lens_out, str):
            lens_out = lens
        kv = make_kv(K, V, pos, lens, lens_out, block_table, layer_begin=layer_begin)
        _check_t(t, lens)
        st = tri_prune_noalloc(self.handle, kv, t.data_ptr(), budget, _stream_handle(stream))
        if check and st != TRI_OK:
            raise TriError(st, "tri_prune_noalloc", tri_last_error(self.handle))
        return st

    def score(self, K, lens, t, raw=None, zmax=None, block_table=None, layer_begin=0,
              stream=None, check=True):
        kv = make_kv(K, None, None, lens, None, block_table, layer_begin=layer_begin)
        _check_t(t, lens)
        st = tri_score(self.handle, kv, t.data_ptr(), _ptr(raw), _ptr(zmax), _stream_handle(stream))
        if check and st != TRI_OK:
            raise TriError(st, "tri_score", tri_last_error(self.handle))
        return st

    def append(self, K, V, pos, lens, block_table, K_new, V_new, pos_new, lens_out="inplace", n_pages=None,
               layer_begin=0, stream=None, check=True, advance=False):
        """Append one token per sequence to a paged cache (see make_kv for the layouts):
        K_new, V_new bf16 [n_layers][batch][n_kv_heads][head_dim], pos_new int32 [batch].
        advance=True: tri_append_advance (pos_new then holds the next positions)."""
        if isinstance(lens_out, str):
            lens_out = lens
        kv = make_kv(K, V, pos, lens, lens_out, block_table, n_pages=n_pages, layer_begin=layer_begin)
        for name, x, dt in (("K_new", K_new, torch.bfloat16), ("V_new", V_new, torch.bfloat16),
                            ("pos_new", pos_new, torch.int32)):
            if x.dtype != dt or not x.is_cuda or not x.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA tensor of {dt}")
        fn = tri_append_advance if advance else tri_append
        st = fn(self.handle, kv, K_new.data_ptr(), V_new.data_ptr(), pos_new.data_ptr(), _stream_handle(stream))
        if check and st != TRI_OK:
            raise TriError(st, fn.__name__, tri_last_error(self.handle))
        return st

    def decode_attention(self, K, V, lens, q, out=None, block_table=None, n_pages=None, layer_begin=0,
                         stream=None, check=True):
        """Attention of the post-RoPE queries q (bf16 [n_layers][batch][Hq][d]) over the cached
        rows [0, lens[s]) of K/V (layouts as in make_kv). Returns out (fp32, like q), or the
        status when check is False."""
        kv = make_kv(K, V, None, lens, None, block_table, n_pages=n_pages, layer_begin=layer_begin)
        if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous():
            raise ValueError("q must be a contiguous CUDA tensor of torch.bfloat16")
        if q.dim() != 4 or tuple(q.shape[:2]) != (int(K.shape[0]), int(lens.shape[0])) or q.shape[3] != K.shape[4]:
            raise ValueError(f"q must be [n_layers][batch][Hq][d] for this cache, got {tuple(q.shape)}")
        if out is not None and (out.dtype != torch.float32 or tuple(out.shape) != tuple(q.shape)
                                or not out.is_contiguous()):
            raise ValueError("out must be a contiguous float32 tensor shaped like q")
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        st = tri_decode_attention(self.handle, kv, q.data_ptr(), out.data_ptr(), _stream_handle(stream))
        if not check:
            return st
        if st != TRI_OK:
            raise TriError(st, "tri_decode_attention", tri_last_error(self.handle))
        return out

    def calibrate_estimate(self, Q, layout, out=None, stream=None, check=True):
        """Calibration statistics from pre-RoPE queries Q (bf16 [n_layers][T][n_q_heads][head_dim],
        on this context's device). Returns fp32 device tensors (q_mean [L][Hq][d],
        q_norm_mean [L][Hq][d/2], R [L][Hq][d/2]), or the status when check is False."""
        if Q.dtype != torch.bfloat16 or Q.dim() != 4 or not Q.is_contiguous():
            raise TriError(TRI_EINVAL, "tri_calibrate_estimate", "Q must be a contiguous bf16 [L][T][Hq][d] tensor")
        nl, T, Hq, d = Q.shape
        if out is None:
            out = (torch.empty((nl, Hq, d), dtype=torch.float32, device=Q.device),
                   torch.empty((nl, Hq, d // 2), dtype=torch.float32, device=Q.device),
                   torch.empty((nl, Hq, d // 2), dtype=torch.float32, device=Q.device))
        qm, qn, R = out
        st = tri_calibrate_estimate(self.handle, Q.data_ptr(), nl, T, Hq, d, int(layout), qm.data_ptr(),
                                    qn.data_ptr(), R.data_ptr(), _stream_handle(stream))
        if not check:
            return st
        if st != TRI_OK:
            raise TriError(st, "tri_calibrate_estimate", tri_last_error(self.handle))
        return qm, qn, R

    def get_error(self, stream=None):
        return tri_get_error(self.handle, _stream_handle(stream))

    def failed_units(self, stream=None, capacity=4096):
        """(total count, unit indices) of units left uncompacted by unit-level failures."""
        st, n, units = tri_get_failed_units(self.handle, _stream_handle(stream), capacity)
        if st != TRI_OK:
            raise TriError(st, "tri_get_failed_units")
        return n, units

    def set_test_fault(self, unit=-1, wait_tries=0):
        """Test hook: withhold the first key copy of `unit` on later calls (-1: off)."""
        st = tri_set_test_fault(self.handle, unit, wait_tries)
        if st != TRI_OK:
            raise TriError(st, "tri_set_test_fault")
