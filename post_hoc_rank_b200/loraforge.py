"""ctypes binding of libloraforge.so: the C ABI of include/loraforge.h, same names.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch tensors used as device allocations; their data
pointers are passed through.  There is no fallback: if the shared library is
missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libloraforge.so")

LF_OK = 0
STATUS_NAMES = {0: "LF_OK", 1: "LF_ERR_INVALID_ARG", 2: "LF_ERR_SHAPE", 3: "LF_ERR_BAD_INDEX",
                4: "LF_ERR_WORKSPACE", 5: "LF_ERR_NUMERIC", 6: "LF_ERR_TIMEOUT", 7: "LF_ERR_CUDA",
                8: "LF_ERR_ALIGNMENT"}

# lf_module: int32 d_out, d_in, r, group; int64 B_off, A_off  (32 bytes, natural alignment)
MODULE_DTYPE = np.dtype([("d_out", "<i4"), ("d_in", "<i4"), ("r", "<i4"), ("group", "<i4"),
                         ("B_off", "<i8"), ("A_off", "<i8")], align=True)
assert MODULE_DTYPE.itemsize == 32


# lf_jd_problem: int32 d_out, d_in, rank, first, count; int64 U_off, Vt_off, sigma_off (48 bytes)
JD_PROBLEM_DTYPE = np.dtype([("d_out", "<i4"), ("d_in", "<i4"), ("rank", "<i4"), ("first", "<i4"),
                             ("count", "<i4"), ("U_off", "<i8"), ("Vt_off", "<i8"), ("sigma_off", "<i8")],
                            align=True)
assert JD_PROBLEM_DTYPE.itemsize == 48


class lf_policy(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("ratio_num", ctypes.c_int32),
                ("ratio_den", ctypes.c_int32), ("floor", ctypes.c_int32)]


def policy_U(num: int, den: int, floor: int = 1) -> lf_policy:
    return lf_policy(0, num, den, floor)


def policy_S(num: int, den: int, floor: int = 1, absolute: bool = False) -> lf_policy:
    """LoRAForge-S (normalised energies), or with absolute=True the variant that ranks
    candidates by sigma^2 (kind 2)."""
    return lf_policy(2 if absolute else 1, num, den, floor)


def policy_E(num: int, den: int, floor: int = 1) -> lf_policy:
    """Energy fraction (kind 3): the smallest rank >= floor keeping num/den of each
    module's spectral energy."""
    return lf_policy(3, num, den, floor)


class lf_phase_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("total_ms", ctypes.c_double), ("launches", ctypes.c_int64)]


class lf_slice(ctypes.Structure):
    """One output slice of lf_lora_shrink_expand_slices (mirrors the C struct)."""
    _fields_ = [("d_out", ctypes.c_int32), ("max_rank", ctypes.c_int32), ("y_offset", ctypes.c_int64),
                ("ranks", ctypes.c_void_p), ("off_A", ctypes.c_void_p), ("off_Bt", ctypes.c_void_p),
                ("A_pool", ctypes.c_void_p), ("Bt_pool", ctypes.c_void_p),
                ("pool_elems_A", ctypes.c_int64), ("pool_elems_Bt", ctypes.c_int64)]


class lf_projection(ctypes.Structure):
    """One projection of lf_lora_shrink_expand_projections (mirrors the C struct)."""
    _fields_ = [("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("d_in", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("y_ld", ctypes.c_int64), ("slice", lf_slice)]


MAX_PROJECTIONS = 8


class LFError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """Load libloraforge.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libloraforge.so not built (expected at {LIB_PATH}); "
                          "run python -m post_hoc_rank_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        L.lf_rank_stride.argtypes = [_P, _I32]; L.lf_rank_stride.restype = _I32
        L.lf_tsqr_workspace_size.argtypes = [_P, _I32]; L.lf_tsqr_workspace_size.restype = _SZ
        L.lf_tsqr_batched.argtypes = [_P, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.lf_tsqr_batched.restype = ctypes.c_int
        L.lf_select_workspace_size.argtypes = [_P, _I32]; L.lf_select_workspace_size.restype = _SZ
        L.lf_select_ranks.argtypes = [_P, _I32, lf_policy, _P, _P, _P, _P, _P, _SZ, _P]
        L.lf_select_ranks.restype = ctypes.c_int
        L.lf_export_workspace_size.argtypes = [_P, _I32]; L.lf_export_workspace_size.restype = _SZ
        L.lf_export_pool_bound.argtypes = [_P, _I32, lf_policy, _P, _P]; L.lf_export_pool_bound.restype = None
        L.lf_truncate_export.argtypes = [_P, _I32, lf_policy, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                         _P, _P, _P, _P, _I64, _I64, _P, _SZ, _P]
        L.lf_truncate_export.restype = ctypes.c_int
        L.lf_apply_workspace_size.argtypes = [_I32, _I32]; L.lf_apply_workspace_size.restype = _SZ
        L.lf_lora_shrink_expand.argtypes = [_I32, _I32, _I32, _P, _P, _P, _I32, _P, _P, _P, _P, _P,
                                            _I64, _I64, ctypes.c_float, _P, _P, _SZ, _P]
        L.lf_lora_shrink_expand.restype = ctypes.c_int
        L.lf_apply_slices_workspace_size.argtypes = [_I32, _I32, _I32]
        L.lf_apply_slices_workspace_size.restype = _SZ
        L.lf_lora_shrink_expand_slices.argtypes = [_I32, _I32, _P, _P, _I64, _P, _I32, _P, _I32,
                                                   ctypes.c_float, _P, _P, _P, _SZ, _P]
        L.lf_lora_shrink_expand_slices.restype = ctypes.c_int
        L.lf_lora_sigma_sandwich.argtypes = [_I32, _I32, _I32, _P, _P, _P, _I32, _I32, _P, _P, _P, _I32,
                                             ctypes.c_float, _P, _SZ, _P]
        L.lf_lora_sigma_sandwich.restype = ctypes.c_int
        L.lf_route_tokens.argtypes = [_I32, _P, _I32, _P, _SZ, _P]; L.lf_route_tokens.restype = ctypes.c_int
        L.lf_lora_shrink_expand_slices_routed.argtypes = [_I32, _I32, _P, _P, _I64, _P, _I32, _P, _I32,
                                                          ctypes.c_float, _P, _P, _SZ, _P]
        L.lf_lora_shrink_expand_slices_routed.restype = ctypes.c_int
        L.lf_lora_shrink_expand_projections.argtypes = [_I32, _P, _I32, _P, _I32, ctypes.c_float, _P, _P, _SZ, _P]
        L.lf_lora_shrink_expand_projections.restype = ctypes.c_int
        L.lf_jd_workspace_size.argtypes = [_P, _I32, _P, _I32, _P, _I32]; L.lf_jd_workspace_size.restype = _SZ
        L.lf_jd_full.argtypes = [_P, _I32, _P, _I32, _P, _I32, _P, _P, _P, _I32, _P, _P, _P, _P, _SZ, _P]
        L.lf_jd_full.restype = ctypes.c_int
        L.lf_lora_shrink_expand_noalloc.argtypes = [_I32, _I32, _I32, _P, _P, _P, _I32, _P, _P, _P, _P, _P,
                                                    _I64, _I64, ctypes.c_float, _P, _P]
        L.lf_lora_shrink_expand_noalloc.restype = ctypes.c_int
        L.lf_check_bounded_wait.argtypes = [_I32, _P]; L.lf_check_bounded_wait.restype = ctypes.c_int
        L.lf_pool_workspace_size.argtypes = [_I32, _I32, _P, _P, _I32]; L.lf_pool_workspace_size.restype = _SZ
        L.lf_pool_subspace.argtypes = [_I32, _I32, _P, _P, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.lf_pool_subspace.restype = ctypes.c_int
        L.lf_status_string.argtypes = [ctypes.c_int]; L.lf_status_string.restype = ctypes.c_char_p
        L.lf_get_device_status.argtypes = [_P]; L.lf_get_device_status.restype = ctypes.c_int
        L.lf_profile_enable.argtypes = [ctypes.c_int]; L.lf_profile_enable.restype = None
        L.lf_profile_reset.argtypes = []; L.lf_profile_reset.restype = None
        L.lf_profile_read.argtypes = [_P, _I32]; L.lf_profile_read.restype = _I32
        L.lf_launch_count.argtypes = []; L.lf_launch_count.restype = _I64
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return ["lf_rank_stride", "lf_tsqr_workspace_size", "lf_tsqr_batched", "lf_select_workspace_size",
            "lf_select_ranks", "lf_export_workspace_size", "lf_export_pool_bound", "lf_truncate_export",
            "lf_apply_workspace_size", "lf_lora_shrink_expand", "lf_status_string", "lf_get_device_status",
            "lf_profile_enable", "lf_profile_reset", "lf_profile_read", "lf_launch_count",
            "lf_lora_shrink_expand_noalloc", "lf_apply_slices_workspace_size", "lf_lora_shrink_expand_slices",
            "lf_lora_sigma_sandwich", "lf_jd_workspace_size", "lf_jd_full", "lf_route_tokens",
            "lf_lora_shrink_expand_slices_routed", "lf_check_bounded_wait", "lf_pool_workspace_size",
            "lf_pool_subspace", "lf_lora_shrink_expand_projections"]

# Limits of lf_lora_shrink_expand_noalloc (its scratch is a fixed array in the library).
NOALLOC_MAX_TOKENS = 16384
NOALLOC_MAX_ADAPTERS = 4096


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _mods_ptr(mods: np.ndarray):
    assert mods.dtype == MODULE_DTYPE and mods.flags["C_CONTIGUOUS"]
    return mods.ctypes.data, int(mods.shape[0])


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str) -> int:
    if st != LF_OK:
        raise LFError(st, where)
    return st


def lf_rank_stride(mods: np.ndarray) -> int:
    p, n = _mods_ptr(mods)
    return lib().lf_rank_stride(p, n)


def lf_tsqr_workspace_size(mods: np.ndarray) -> int:
    p, n = _mods_ptr(mods)
    return lib().lf_tsqr_workspace_size(p, n)


def lf_tsqr_batched(mods, B_base, A_base, R_B, R_A, sigma, U, V, ws, stream=None, check=True) -> int:
    p, n = _mods_ptr(mods)
    st = lib().lf_tsqr_batched(p, n, _ptr(B_base), _ptr(A_base), _ptr(R_B), _ptr(R_A), _ptr(sigma),
                               _ptr(U), _ptr(V), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_tsqr_batched") if check else st


def lf_select_workspace_size(mods: np.ndarray) -> int:
    p, n = _mods_ptr(mods)
    return lib().lf_select_workspace_size(p, n)


def lf_select_ranks(mods, pol: lf_policy, sigma, ranks, off_A, off_Bt, ws, stream=None, check=True) -> int:
    p, n = _mods_ptr(mods)
    st = lib().lf_select_ranks(p, n, pol, _ptr(sigma), _ptr(ranks), _ptr(off_A), _ptr(off_Bt), _ptr(ws),
                               ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_select_ranks") if check else st


def lf_export_workspace_size(mods: np.ndarray) -> int:
    p, n = _mods_ptr(mods)
    return lib().lf_export_workspace_size(p, n)


def lf_export_pool_bound(mods: np.ndarray, pol: lf_policy) -> tuple[int, int]:
    p, n = _mods_ptr(mods)
    a, b = ctypes.c_int64(0), ctypes.c_int64(0)
    lib().lf_export_pool_bound(p, n, pol, ctypes.addressof(a), ctypes.addressof(b))
    return a.value, b.value


def lf_truncate_export(mods, pol, B_base, A_base, R_B, R_A, sigma, U, V, ranks, off_A, off_Bt,
                       A_pool, Bt_pool, A_pool_bf16, Bt_pool_bf16, ws, stream=None, check=True) -> int:
    p, n = _mods_ptr(mods)
    st = lib().lf_truncate_export(p, n, pol, _ptr(B_base), _ptr(A_base), _ptr(R_B), _ptr(R_A), _ptr(sigma),
                                  _ptr(U), _ptr(V), _ptr(ranks), _ptr(off_A), _ptr(off_Bt), _ptr(A_pool),
                                  _ptr(Bt_pool), _ptr(A_pool_bf16), _ptr(Bt_pool_bf16), A_pool.numel(),
                                  Bt_pool.numel(), _ptr(ws), ws.numel() if ws is not None else 0,
                                  _stream(stream))
    return _check(st, "lf_truncate_export") if check else st


def lf_apply_workspace_size(T: int, n_adapters: int) -> int:
    return lib().lf_apply_workspace_size(T, n_adapters)


def lf_lora_shrink_expand(x, y, ids, n_adapters, ranks, off_A, off_Bt, A_pool, Bt_pool, scale, ws,
                          seg_out=None, stream=None, check=True) -> int:
    T, d_in = x.shape
    d_out = y.shape[1]
    st = lib().lf_lora_shrink_expand(T, d_in, d_out, _ptr(x), _ptr(y), _ptr(ids), n_adapters, _ptr(ranks),
                                     _ptr(off_A), _ptr(off_Bt), _ptr(A_pool), _ptr(Bt_pool), A_pool.numel(),
                                     Bt_pool.numel(), float(scale),
                                     _ptr(seg_out), _ptr(ws), ws.numel() if ws is not None else 0,
                                     _stream(stream))
    return _check(st, "lf_lora_shrink_expand") if check else st


def lf_apply_slices_workspace_size(T: int, n_adapters: int, n_slices: int) -> int:
    return lib().lf_apply_slices_workspace_size(T, n_adapters, n_slices)


def make_slice(d_out, y_offset, ranks, off_A, off_Bt, A_pool, Bt_pool, max_rank=0) -> lf_slice:
    """lf_slice from device tensors (ranks int32, offsets int64, pools bf16); max_rank: 0, or
    an upper bound of the slice's ranks the caller knows."""
    return lf_slice(int(d_out), int(max_rank), int(y_offset), _ptr(ranks), _ptr(off_A), _ptr(off_Bt), _ptr(A_pool),
                    _ptr(Bt_pool), A_pool.numel(), Bt_pool.numel())


def lf_lora_shrink_expand_slices(x, y, ids, n_adapters, slices, scale, ws, adapter_scale=None, seg_out=None,
                                 stream=None, check=True) -> int:
    """slices: list of lf_slice (make_slice); y: T x y_ld bf16 holding every slice."""
    T, d_in = x.shape
    arr = (lf_slice * len(slices))(*slices)
    st = lib().lf_lora_shrink_expand_slices(T, d_in, _ptr(x), _ptr(y), y.shape[1], _ptr(ids), n_adapters, arr,
                                            len(slices), float(scale), _ptr(adapter_scale), _ptr(seg_out), _ptr(ws),
                                            ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_lora_shrink_expand_slices") if check else st


def lf_route_tokens(ids, n_adapters, ws, stream=None, check=True) -> int:
    """Routing of a token batch into `ws`, for routed calls on the same batch."""
    st = lib().lf_route_tokens(int(ids.numel()), _ptr(ids), n_adapters, _ptr(ws), ws.numel() if ws is not None else 0,
                               _stream(stream))
    return _check(st, "lf_route_tokens") if check else st


def lf_lora_shrink_expand_slices_routed(x, y, ids, n_adapters, slices, scale, ws, adapter_scale=None, stream=None,
                                        check=True) -> int:
    """lf_lora_shrink_expand_slices on a workspace that already holds this batch's routing."""
    T, d_in = x.shape
    arr = (lf_slice * len(slices))(*slices)
    st = lib().lf_lora_shrink_expand_slices_routed(T, d_in, _ptr(x), _ptr(y), y.shape[1], _ptr(ids), n_adapters, arr,
                                                   len(slices), float(scale), _ptr(adapter_scale), _ptr(ws),
                                                   ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_lora_shrink_expand_slices_routed") if check else st


def make_projection(x, y, sl: lf_slice) -> lf_projection:
    """lf_projection from device tensors: x T x d_in bf16, y T x y_ld bf16, and the slice
    (make_slice) saying where in y and with which factors."""
    return lf_projection(_ptr(x), _ptr(y), int(x.shape[1]), 0, int(y.shape[1]), sl)


def lf_lora_shrink_expand_projections(T, ids, n_adapters, projections, scale, ws=None, adapter_scale=None,
                                      stream=None, check=True) -> int:
    """Up to MAX_PROJECTIONS projections (make_projection) of one token batch in one call."""
    arr = (lf_projection * len(projections))(*projections)
    st = lib().lf_lora_shrink_expand_projections(int(T), _ptr(ids), n_adapters, arr, len(projections), float(scale),
                                                 _ptr(adapter_scale), _ptr(ws), ws.numel() if ws is not None else 0,
                                                 _stream(stream))
    return _check(st, "lf_lora_shrink_expand_projections") if check else st


def lf_lora_sigma_sandwich(x, y, ids, n_adapters, Vt, Ut, sigma, diagonal, scale, ws, stream=None,
                           check=True) -> int:
    """Sigma-sandwich serving: y += scale * U (Sigma_a (V^T x)); Vt rank x d_in, Ut rank x d_out
    (bf16), sigma n_adapters x rank (diagonal) or n_adapters x rank x rank (fp32)."""
    T, d_in = x.shape
    d_out = y.shape[1]
    st = lib().lf_lora_sigma_sandwich(T, d_in, d_out, _ptr(x), _ptr(y), _ptr(ids), n_adapters, Vt.shape[0],
                                      _ptr(Vt), _ptr(Ut), _ptr(sigma), 1 if diagonal else 0, float(scale), _ptr(ws),
                                      ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_lora_sigma_sandwich") if check else st


def _jd_tables(mods, members, probs):
    pm, nm = _mods_ptr(mods)
    assert members.dtype == np.int32 and members.flags["C_CONTIGUOUS"]
    assert probs.dtype == JD_PROBLEM_DTYPE and probs.flags["C_CONTIGUOUS"]
    return pm, nm, members.ctypes.data, int(members.shape[0]), probs.ctypes.data, int(probs.shape[0])


def lf_jd_workspace_size(mods: np.ndarray, members: np.ndarray, probs: np.ndarray) -> int:
    return lib().lf_jd_workspace_size(*_jd_tables(mods, members, probs))


def lf_pool_workspace_size(side, ranks, offs, d) -> int:
    rk = np.ascontiguousarray(ranks, dtype=np.int32)
    of = np.ascontiguousarray(offs, dtype=np.int64)
    return lib().lf_pool_workspace_size(int(side), len(rk), rk.ctypes.data, of.ctypes.data, int(d))


def lf_pool_subspace(side, ranks, offs, d, base, num, den, k, sigma, basis, coef, resid, ws, stream=None,
                     check=True) -> int:
    """Pool-wide subspace of stacked factors (side 0: rows A_i; side 1: columns of B_i)."""
    rk = np.ascontiguousarray(ranks, dtype=np.int32)
    of = np.ascontiguousarray(offs, dtype=np.int64)
    st = lib().lf_pool_subspace(int(side), len(rk), rk.ctypes.data, of.ctypes.data, int(d), _ptr(base), int(num),
                                int(den), _ptr(k), _ptr(sigma), _ptr(basis), _ptr(coef), _ptr(resid), _ptr(ws),
                                ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_pool_subspace") if check else st


def lf_jd_full(mods, members, probs, B_base, A_base, weights, iters, U_base, Vt_base, sigma, ws, stream=None,
               check=True) -> int:
    """JD-Full eigenvalue iteration: U_base / Vt_base hold the starting bases on entry and the
    bases after `iters` steps on return; sigma (nullable) receives Sigma_i = U^T B_i A_i V."""
    st = lib().lf_jd_full(*_jd_tables(mods, members, probs), _ptr(B_base), _ptr(A_base), _ptr(weights),
                          int(iters), _ptr(U_base), _ptr(Vt_base), _ptr(sigma), _ptr(ws),
                          ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "lf_jd_full") if check else st


def lf_lora_shrink_expand_noalloc(x, y, ids, n_adapters, ranks, off_A, off_Bt, A_pool, Bt_pool, scale,
                                  seg_out=None, stream=None, check=True) -> int:
    """lf_lora_shrink_expand without a workspace argument, for callers that cannot
    allocate device memory; the library keeps the routing scratch itself."""
    T, d_in = x.shape
    d_out = y.shape[1]
    st = lib().lf_lora_shrink_expand_noalloc(T, d_in, d_out, _ptr(x), _ptr(y), _ptr(ids), n_adapters,
                                             _ptr(ranks), _ptr(off_A), _ptr(off_Bt), _ptr(A_pool), _ptr(Bt_pool),
                                             A_pool.numel(), Bt_pool.numel(), float(scale), _ptr(seg_out),
                                             _stream(stream))
    return _check(st, "lf_lora_shrink_expand_noalloc") if check else st


def lf_status_string(st: int) -> str:
    return lib().lf_status_string(st).decode()


def lf_get_device_status(stream=None) -> int:
    return lib().lf_get_device_status(_stream(stream))


def lf_profile_enable(on: bool) -> None:
    lib().lf_profile_enable(1 if on else 0)


def lf_profile_reset() -> None:
    lib().lf_profile_reset()


def lf_profile_read() -> dict[str, tuple[float, int]]:
    """{phase: (total device ms, launches)} accumulated since the last reset."""
    buf = (lf_phase_time * 64)()
    n = lib().lf_profile_read(ctypes.addressof(buf), 64)
    return {buf[i].name.decode(): (buf[i].total_ms, buf[i].launches) for i in range(min(n, 64))}


def lf_launch_count() -> int:
    return lib().lf_launch_count()
