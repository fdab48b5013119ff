"""Python binding of the B200 multi-tenant mixed-precision delta library (include/dc.h).

Argument marshalling only: every step of the serving path runs in the CUDA library
``libdc.so`` built in this directory.  PyTorch is used by callers for device memory and streams;
functions here take tensors (device pointers are read with ``data_ptr()``) or numpy arrays
(host buffers) and return the C status as a raised ``DcError`` when it is not DC_OK.

If the library has not been built, every entry point raises ``DcLibraryMissing``: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdc.so")
SYNTH_LIB_PATH = os.path.join(_HERE, "libdc_synth.so")

DC_OK, DC_ERR_INVALID_ARG, DC_ERR_SHAPE, DC_ERR_BITS, DC_ERR_ALIGN = 0, 1, 2, 3, 4
DC_ERR_WORKSPACE, DC_ERR_TENANT, DC_ERR_CUDA, DC_ERR_UNSUPPORTED = 5, 6, 7, 8
DC_DTYPE_F32, DC_DTYPE_BF16, DC_DTYPE_FP8 = 0, 1, 2
DC_BASE, DC_DELTA, DC_REUSE_ROUTING, DC_DECODE_ONLY = 1, 2, 4, 8
DC_MAX_BANDS = 4
DC_GROUP = 128


class DcError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"dc status {status}: {message}")
        self.status = status


class DcLibraryMissing(RuntimeError):
    pass


class dc_factor_desc(C.Structure):
    _fields_ = [("d_out", C.c_int32), ("d_in", C.c_int32), ("n_bands", C.c_int32),
                ("bits", C.c_int32 * DC_MAX_BANDS), ("rank", C.c_int32 * DC_MAX_BANDS)]


class dc_delta_handle(C.Structure):
    _fields_ = [("dev_base", C.c_uint64), ("bytes", C.c_uint64), ("desc", dc_factor_desc),
                ("rank_total", C.c_int32), ("reserved", C.c_int32)]


class dc_pager_desc(C.Structure):
    _fields_ = [("n_tenants", C.c_int32), ("n_slots", C.c_int32), ("slot_bytes", C.c_uint64),
                ("n_tables", C.c_int32), ("reserved", C.c_int32)]


class dc_pager_stats(C.Structure):
    _fields_ = [("hits", C.c_int64), ("misses", C.c_int64), ("evictions", C.c_int64), ("bytes_loaded", C.c_int64),
                ("batches", C.c_int64)]


class dc_linear(C.Structure):
    _fields_ = [("W_base", C.c_void_p), ("w_dtype", C.c_int32), ("d_out", C.c_int32), ("d_in", C.c_int32),
                ("n_tenants", C.c_int32), ("max_rank", C.c_int32), ("tenants_dev", C.c_void_p)]


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise DcLibraryMissing(f"{LIB_PATH} is not built; run `python -m tenant_mixed_precision_b200.build`")
    lib = C.CDLL(LIB_PATH)
    P, I32, SZ, VP = C.POINTER, C.c_int32, C.c_size_t, C.c_void_p
    sig = {
        "dc_last_error": (C.c_char_p, []),
        "dc_version": (C.c_char_p, []),
        "dc_packed_size": (SZ, [P(dc_factor_desc)]),
        "dc_quantize_rtn": (I32, [P(dc_factor_desc), VP, VP, VP, VP, VP, VP]),
        "dc_pack_upload": (I32, [P(dc_factor_desc), VP, VP, VP, VP, VP, VP, SZ, VP, P(dc_delta_handle)]),
        "dc_quantize_pack_device": (I32, [P(dc_factor_desc), VP, VP, VP, VP, SZ, VP, SZ, VP, P(dc_delta_handle)]),
        "dc_quantize_scratch_size": (SZ, [P(dc_factor_desc)]),
        "dc_tenant_table_upload": (I32, [P(dc_delta_handle), I32, VP, SZ, VP]),
        "dc_workspace_size": (SZ, [I32, I32, I32, I32, I32]),
        "dc_build_segments": (I32, [VP, I32, I32, VP, SZ, VP]),
        "dc_read_segments": (I32, [VP, I32, VP, VP, VP, VP, VP]),
        "dc_delta_linear_segmented": (I32, [P(dc_linear), VP, VP, VP, I32, I32, I32, I32, VP, SZ, VP]),
        "dc_delta_linear_segmented_static": (I32, [P(dc_linear), VP, VP, VP, I32, I32, I32, I32, VP, P(I32)]),
        "dc_layer_forward": (I32, [P(dc_linear), VP, VP, VP, P(VP), VP, I32, I32, I32, I32, VP, SZ, VP]),
        "dc_unpack_codes_debug": (I32, [P(dc_delta_handle), I32, VP, VP]),
        "dc_read_device_status": (I32, [VP, VP, P(I32)]),
        "dc_profile_begin": (I32, [I32]),
        "dc_profile_end": (I32, [P(C.c_float), P(I32), I32]),
        "dc_quantize_fp8_rows": (I32, [VP, I32, I32, VP, VP]),
        "dc_quantize_fp8_rows_device": (I32, [VP, I32, I32, I32, VP, VP, VP]),
        "dc_prinmix_scores": (I32, [VP, VP, I32, I32, VP, I32, VP, I32, VP]),
        "dc_prinmix_allocate": (I32, [VP, I32, VP, I32, I32, I32, C.c_double, I32, VP, P(C.c_double)]),
        "dc_prinmix_rtc": (I32, [VP, VP, VP, VP, I32, I32, I32, VP, I32, VP]),
        "dc_prinmix_compress": (I32, [VP, VP, VP, I32, I32, I32, VP, I32, C.c_double, VP, I32, I32, I32,
                                      VP, VP, VP, VP, VP, P(C.c_double)]),
        "dc_svd_workspace_size": (SZ, [I32, I32, I32, I32]),
        "dc_svd_device": (I32, [VP, VP, I32, I32, I32, I32, I32, I32, C.c_uint64, VP, VP, VP, VP, SZ, VP, P(I32)]),
        "dc_pager_scratch_size": (SZ, [P(dc_pager_desc)]),
        "dc_pager_create": (I32, [P(dc_pager_desc), VP, SZ, P(VP), VP, SZ, P(VP)]),
        "dc_pager_set_tenant": (I32, [VP, I32, VP, C.c_uint64, P(C.c_int64)]),
        "dc_pager_prepare": (I32, [VP, P(I32), I32, VP, VP]),
        "dc_pager_commit": (I32, [VP, VP]),
        "dc_pager_get_stats": (I32, [VP, P(dc_pager_stats)]),
        "dc_pager_slot_of": (I32, [VP, I32]),
        "dc_pager_destroy": (I32, [VP]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def lib():
    return _load()


def exported_symbols() -> list[str]:
    """Names of the C entry points this binding declares (all must be exported by libdc.so)."""
    return ["dc_last_error", "dc_version", "dc_packed_size", "dc_quantize_rtn", "dc_pack_upload",
            "dc_quantize_pack_device", "dc_quantize_scratch_size", "dc_tenant_table_upload",
            "dc_workspace_size", "dc_build_segments", "dc_read_segments", "dc_delta_linear_segmented",
            "dc_delta_linear_segmented_static",
            "dc_layer_forward", "dc_unpack_codes_debug", "dc_read_device_status", "dc_profile_begin",
            "dc_profile_end", "dc_quantize_fp8_rows", "dc_quantize_fp8_rows_device", "dc_prinmix_scores", "dc_prinmix_allocate", "dc_prinmix_rtc", "dc_prinmix_compress",
            "dc_svd_workspace_size", "dc_svd_device", "dc_pager_scratch_size", "dc_pager_create", "dc_pager_set_tenant", "dc_pager_prepare",
            "dc_pager_commit", "dc_pager_get_stats", "dc_pager_slot_of", "dc_pager_destroy"]


def _check(st: int):
    if st != DC_OK:
        raise DcError(st, _load().dc_last_error().decode())


def _stream(stream) -> int | None:
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:
            pass
        return None
    return getattr(stream, "cuda_stream", stream)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return DC_DTYPE_F32
    if t.dtype == torch.bfloat16:
        return DC_DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------------------------------
# descriptors
# ------------------------------------------------------------------------------------------
def make_desc(d_out: int, d_in: int, plan) -> dc_factor_desc:
    """plan: [(bits, rank), ...] in descending singular-value order (at most 4 bands)."""
    plan = list(plan)
    if len(plan) > DC_MAX_BANDS:
        raise ValueError("at most 4 bands")
    d = dc_factor_desc()
    d.d_out, d.d_in, d.n_bands = d_out, d_in, len(plan)
    for i, (b, r) in enumerate(plan):
        d.bits[i], d.rank[i] = int(b), int(r)
    return d


def desc_rank(desc: dc_factor_desc) -> int:
    return sum(desc.rank[i] for i in range(desc.n_bands) if desc.bits[i])


# ------------------------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ------------------------------------------------------------------------------------------
def dc_version() -> str:
    return _load().dc_version().decode()


def dc_last_error() -> str:
    return _load().dc_last_error().decode()


def dc_packed_size(desc: dc_factor_desc) -> int:
    n = _load().dc_packed_size(C.byref(desc))
    if n == 0:
        raise DcError(DC_ERR_INVALID_ARG, dc_last_error())
    return n


def dc_quantize_rtn(desc: dc_factor_desc, U: np.ndarray, Vt: np.ndarray):
    """Host RTN.  U: float32 [d_out, r] (any order), Vt: float32 [r, d_in].
    Returns (codes_u uint8 [r, d_out], codes_v uint8 [r, d_in], sz_u uint16 [r, d_out/128, 2],
    sz_v uint16 [r, d_in/128, 2])."""
    r = desc_rank(desc)
    Uc = np.ascontiguousarray(np.asarray(U, dtype=np.float32).T)  # [r, d_out] = column-major U
    Vc = np.ascontiguousarray(np.asarray(Vt, dtype=np.float32))
    cu = np.zeros((r, desc.d_out), np.uint8)
    cv = np.zeros((r, desc.d_in), np.uint8)
    su = np.zeros((r, desc.d_out // DC_GROUP, 2), np.uint16)
    sv = np.zeros((r, desc.d_in // DC_GROUP, 2), np.uint16)
    _check(_load().dc_quantize_rtn(C.byref(desc), _ptr(Uc), _ptr(Vc), _ptr(cu), _ptr(cv), _ptr(su), _ptr(sv)))
    return cu, cv, su, sv


def dc_pack_upload(desc: dc_factor_desc, codes_u, codes_v, sz_u, sz_v, S, dev_dst, stream=None) -> dc_delta_handle:
    h = dc_delta_handle()
    arrs = [np.ascontiguousarray(a) for a in (codes_u, codes_v, sz_u, sz_v)]
    S = np.ascontiguousarray(np.asarray(S, dtype=np.float32))
    nbytes = dev_dst.numel() * dev_dst.element_size()
    _check(_load().dc_pack_upload(C.byref(desc), *[_ptr(a) for a in arrs], _ptr(S), _ptr(dev_dst), nbytes,
                                  _stream(stream), C.byref(h)))
    return h


def dc_quantize_scratch_size(desc: dc_factor_desc) -> int:
    return _load().dc_quantize_scratch_size(C.byref(desc))


def dc_quantize_pack_device(desc: dc_factor_desc, U_dev, Vt_dev, S_dev, dev_dst, scratch, stream=None,
                            dst_offset: int = 0, dst_bytes: int | None = None) -> dc_delta_handle:
    """U_dev: float32 device [r, d_out] contiguous (= column-major U), Vt_dev: [r, d_in], S_dev: [r]."""
    h = dc_delta_handle()
    nbytes = dst_bytes if dst_bytes is not None else dev_dst.numel() * dev_dst.element_size() - dst_offset
    _check(_load().dc_quantize_pack_device(C.byref(desc), _ptr(U_dev), _ptr(Vt_dev), _ptr(S_dev),
                                           _ptr(dev_dst) + dst_offset, nbytes, _ptr(scratch),
                                           scratch.numel() * scratch.element_size(), _stream(stream), C.byref(h)))
    return h


def dc_tenant_table_upload(handles, dev_dst, stream=None):
    n = len(handles)
    arr = (dc_delta_handle * max(n, 1))(*handles)
    _check(_load().dc_tenant_table_upload(arr, n, _ptr(dev_dst), dev_dst.numel() * dev_dst.element_size(),
                                          _stream(stream)))
    return arr  # keep alive until the stream reaches the copy


def empty_handle() -> dc_delta_handle:
    return dc_delta_handle()


def dc_workspace_size(T: int, max_rank: int, max_d_in: int, n_linears: int, max_tenants: int) -> int:
    return _load().dc_workspace_size(T, max_rank, max_d_in, n_linears, max_tenants)


def dc_build_segments(tenant_ids, T: int, n_tenants: int, ws, stream=None):
    _check(_load().dc_build_segments(_ptr(tenant_ids), T, n_tenants, _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream(stream)))


def dc_read_segments(ws, T: int, perm, inv_perm, segments, n_segments, stream=None):
    _check(_load().dc_read_segments(_ptr(ws), T, _ptr(perm), _ptr(inv_perm), _ptr(segments), _ptr(n_segments),
                                    _stream(stream)))


def make_linear(W_base, d_out: int, d_in: int, n_tenants: int, max_rank: int, tenants_dev,
                w_dtype: int | None = None) -> dc_linear:
    lin = dc_linear()
    lin.W_base = _ptr(W_base)
    if w_dtype is not None:
        lin.w_dtype = w_dtype
    elif W_base is None or isinstance(W_base, int):
        lin.w_dtype = DC_DTYPE_BF16
    elif str(getattr(W_base, "dtype", "")) in ("torch.uint8", "uint8"):
        lin.w_dtype = DC_DTYPE_FP8  # an fp8 weight blob (dc_quantize_fp8_rows_device / fp8_weight_blob)
    else:
        lin.w_dtype = _dtype_code(W_base)
    lin.d_out, lin.d_in, lin.n_tenants, lin.max_rank = d_out, d_in, n_tenants, max_rank
    lin.tenants_dev = _ptr(tenants_dev)
    return lin


def dc_delta_linear_segmented(lin: dc_linear, x, y, tenant_ids, T: int, flags: int, ws, stream=None):
    _check(_load().dc_delta_linear_segmented(C.byref(lin), _ptr(x), _ptr(y), _ptr(tenant_ids), T, _dtype_code(x),
                                             _dtype_code(y), flags, _ptr(ws), ws.numel() * ws.element_size(),
                                             _stream(stream)))


STATIC_WORKSPACE_BYTES = 16 << 20  # DC_STATIC_WORKSPACE_BYTES


def dc_delta_linear_segmented_static(lin: dc_linear, x, y, tenant_ids, T: int, flags: int, stream=None,
                                     read_status: bool = False):
    """dc_delta_linear_segmented on the library's static workspace (no workspace argument).

    Returns the device status word of the call when read_status is set (the call then waits for
    the stream), else None."""
    v = C.c_int32(0)
    _check(_load().dc_delta_linear_segmented_static(C.byref(lin), _ptr(x), _ptr(y), _ptr(tenant_ids), T,
                                                    _dtype_code(x), _dtype_code(y), flags, _stream(stream),
                                                    C.byref(v) if read_status else None))
    return v.value if read_status else None


def dc_layer_forward(lins, x_h, x_o, x_f, ys, tenant_ids, T: int, flags: int, ws, stream=None):
    arr = (dc_linear * 7)(*lins)
    yp = (C.c_void_p * 7)(*[_ptr(y) for y in ys])
    _check(_load().dc_layer_forward(arr, _ptr(x_h), _ptr(x_o), _ptr(x_f), yp, _ptr(tenant_ids), T,
                                    _dtype_code(x_h), _dtype_code(ys[0]), flags, _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)))


def dc_unpack_codes_debug(handle: dc_delta_handle, which: int, out_dev, stream=None):
    _check(_load().dc_unpack_codes_debug(C.byref(handle), which, _ptr(out_dev), _stream(stream)))


def dc_read_device_status(ws, stream=None) -> int:
    v = C.c_int32(0)
    _check(_load().dc_read_device_status(_ptr(ws), _stream(stream), C.byref(v)))
    return v.value


KERNEL_KINDS = ("routing", "prep", "rank_reduction", "delta_output", "backbone_output")


def dc_profile_begin(capacity: int):
    _check(_load().dc_profile_begin(capacity))


def dc_profile_end(capacity: int):
    """Returns a list of (kind name, milliseconds) per recorded launch."""
    ms = (C.c_float * capacity)()
    kinds = (C.c_int32 * capacity)()
    n = _load().dc_profile_end(ms, kinds, capacity)
    if n < 0:
        raise DcError(DC_ERR_CUDA, "profiling failed: " + dc_last_error())
    return [(KERNEL_KINDS[kinds[i]], float(ms[i])) for i in range(min(n, capacity))]


# ------------------------------------------------------------------------------------------
# fp8 backbone weights (host quantiser)
# ------------------------------------------------------------------------------------------
def dc_quantize_fp8_rows(W) -> tuple[np.ndarray, np.ndarray]:
    """W: float32 [rows, cols] -> (E4M3 codes uint8 [rows, cols], fp32 row scales [rows])."""
    W = np.ascontiguousarray(np.asarray(W, dtype=np.float32))
    codes = np.zeros(W.shape, np.uint8)
    scales = np.zeros(W.shape[0], np.float32)
    _check(_load().dc_quantize_fp8_rows(_ptr(W), W.shape[0], W.shape[1], _ptr(codes), _ptr(scales)))
    return codes, scales


def dc_quantize_fp8_rows_device(W, stream=None):
    """W: device tensor [rows, cols] (fp32 or bf16) -> the DC_DTYPE_FP8 W_base blob as a device
    uint8 tensor (codes row-major, then the fp32 row scales), quantised on the device."""
    import torch
    rows, cols = W.shape
    W = W.contiguous()
    blob = torch.empty(rows * cols + 4 * rows, dtype=torch.uint8, device=W.device)
    _check(_load().dc_quantize_fp8_rows_device(_ptr(W), _dtype_code(W), rows, cols, _ptr(blob),
                                               blob.data_ptr() + rows * cols, _stream(stream)))
    if isinstance(stream, torch.cuda.Stream):  # both buffers are in use on that stream
        W.record_stream(stream)
        blob.record_stream(stream)
    return blob


def fp8_weight_blob(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """The W_base buffer of a DC_DTYPE_FP8 linear: codes row-major, then the fp32 row scales."""
    return np.concatenate([np.ascontiguousarray(codes, np.uint8).reshape(-1),
                           np.ascontiguousarray(scales, np.float32).view(np.uint8)])


# ------------------------------------------------------------------------------------------
# PrinMix allocation variants (host)
# ------------------------------------------------------------------------------------------
PRINMIX_WIDTHS = (0, 2, 3, 8)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def dc_prinmix_scores(Vt, S, X, widths=PRINMIX_WIDTHS) -> np.ndarray:
    Vt, S, X = _f32(Vt), _f32(S), _f32(X)
    w = np.ascontiguousarray(widths, dtype=np.int32)
    out = np.zeros((Vt.shape[0], len(w)), np.float64)
    _check(_load().dc_prinmix_scores(_ptr(Vt), _ptr(S), Vt.shape[0], Vt.shape[1], _ptr(X), X.shape[0], _ptr(w), len(w),
                                     _ptr(out)))
    return out


def dc_prinmix_allocate(scores, widths, d_out: int, d_in: int, ratio: float, max_kinds: int):
    sc = np.ascontiguousarray(scores, dtype=np.float64)
    w = np.ascontiguousarray(widths, dtype=np.int32)
    out = np.zeros(sc.shape[0], np.int32)
    obj = C.c_double(0.0)
    _check(_load().dc_prinmix_allocate(_ptr(sc), sc.shape[0], _ptr(w), len(w), d_out, d_in, ratio, max_kinds, _ptr(out),
                                       C.byref(obj)))
    return out, obj.value


def dc_prinmix_rtc(U, S, Vt, Vt_hat, X) -> np.ndarray:
    """U: [d_out, k] (columns u_i) -> U~ [d_out, k]."""
    Uc = _f32(np.asarray(U, dtype=np.float32).T)  # rows u_i
    S, Vt, Vh, X = _f32(S), _f32(Vt), _f32(Vt_hat), _f32(X)
    k, d_out, d_in = Uc.shape[0], Uc.shape[1], Vt.shape[1]
    out = np.zeros((k, d_out), np.float32)
    _check(_load().dc_prinmix_rtc(_ptr(Uc), _ptr(S), _ptr(Vt), _ptr(Vh), k, d_out, d_in, _ptr(X), X.shape[0], _ptr(out)))
    return out.T


def dc_prinmix_compress(U, S, Vt, X, ratio: float, max_kinds: int, widths=PRINMIX_WIDTHS, rtc: bool = True):
    """U: [d_out, r] (columns u_i), S [r], Vt [r, d_in]; returns (desc, perm, U_out [d_out, k],
    S_out [k], Vt_out [k, d_in], objective)."""
    Uc = _f32(np.asarray(U, dtype=np.float32).T)
    S, Vt, X = _f32(S), _f32(Vt), _f32(X)
    r, d_out, d_in = Uc.shape[0], Uc.shape[1], Vt.shape[1]
    w = np.ascontiguousarray(widths, dtype=np.int32)
    desc = dc_factor_desc()
    perm = np.zeros(r, np.int32)
    Uo = np.zeros((r, d_out), np.float32)
    So = np.zeros(r, np.float32)
    Vo = np.zeros((r, d_in), np.float32)
    obj = C.c_double(0.0)
    _check(_load().dc_prinmix_compress(_ptr(Uc), _ptr(S), _ptr(Vt), r, d_out, d_in, _ptr(X), X.shape[0], ratio, _ptr(w),
                                       len(w), max_kinds, 1 if rtc else 0, C.addressof(desc), _ptr(perm), _ptr(Uo),
                                       _ptr(So), _ptr(Vo), C.byref(obj)))
    k = desc_rank(desc)
    return desc, perm, Uo[:k].T, So[:k], Vo[:k], obj.value


# ------------------------------------------------------------------------------------------
# device compressor (SVD step)
# ------------------------------------------------------------------------------------------
def dc_svd_workspace_size(d_out: int, d_in: int, r: int, oversample: int) -> int:
    return _load().dc_svd_workspace_size(d_out, d_in, r, oversample)


def dc_svd_device(W_ft, W_base, r: int, oversample: int, power_iters: int, seed: int, U_out, S_out, Vt_out, ws,
                  stream=None) -> int:
    """Top-r SVD of W_ft - W_base on the device into U_out [r, d_out], S_out [r], Vt_out [r, d_in]
    (float32 device tensors).  Returns the number of Jacobi sweeps run."""
    d_out, d_in = W_ft.shape
    sw = C.c_int32(0)
    _check(_load().dc_svd_device(_ptr(W_ft), _ptr(W_base), _dtype_code(W_ft), d_out, d_in, r, oversample, power_iters,
                                 seed, _ptr(U_out), _ptr(S_out), _ptr(Vt_out), _ptr(ws), ws.numel() * ws.element_size(),
                                 _stream(stream), C.byref(sw)))
    return sw.value


# ------------------------------------------------------------------------------------------
# tenant paging
# ------------------------------------------------------------------------------------------
class Pager:
    """dc_pager_* over caller-owned device memory: `arena` (n_slots * slot_bytes bytes), the device
    tenant tables `tables` (one per linear) and a patch scratch allocated here as a torch tensor."""

    def __init__(self, n_tenants: int, n_slots: int, slot_bytes: int, arena, tables):
        import torch
        self.desc = dc_pager_desc(n_tenants, n_slots, slot_bytes, len(tables), 0)
        nsc = _load().dc_pager_scratch_size(C.byref(self.desc))
        self.scratch = torch.empty(max(nsc, 16), dtype=torch.uint8, device=arena.device)
        self._tables = (C.c_void_p * len(tables))(*[_ptr(t) for t in tables])
        self._arena = arena
        h = C.c_void_p()
        _check(_load().dc_pager_create(C.byref(self.desc), _ptr(arena), arena.numel() * arena.element_size(),
                                       self._tables, _ptr(self.scratch), nsc, C.byref(h)))
        self.h = h
        self._images = {}

    def set_tenant(self, tenant: int, image_host, blob_offsets):
        """image_host: pinned host uint8 tensor (kept alive here); blob_offsets: per table, -1 = none."""
        offs = (C.c_int64 * len(blob_offsets))(*[int(o) for o in blob_offsets])
        _check(_load().dc_pager_set_tenant(self.h, tenant, _ptr(image_host), image_host.numel(), offs))
        self._images[tenant] = image_host

    def prepare(self, tenant_ids_host: np.ndarray, copy_stream, compute_stream):
        ids = np.ascontiguousarray(tenant_ids_host, dtype=np.int32)
        _check(_load().dc_pager_prepare(self.h, ids.ctypes.data_as(C.POINTER(C.c_int32)), len(ids),
                                        _stream(copy_stream), _stream(compute_stream)))

    def commit(self, compute_stream):
        _check(_load().dc_pager_commit(self.h, _stream(compute_stream)))

    def stats(self) -> dict:
        st = dc_pager_stats()
        _check(_load().dc_pager_get_stats(self.h, C.byref(st)))
        return {f: getattr(st, f) for f, _ in dc_pager_stats._fields_}

    def slot_of(self, tenant: int) -> int:
        return _load().dc_pager_slot_of(self.h, tenant)

    def close(self):
        if self.h:
            _load().dc_pager_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------------------------------
# device input generator (test/benchmark inputs; twin of synth.py's counter-based stream)
# ------------------------------------------------------------------------------------------
_synth_lib = None


def _synth_loader():
    global _synth_lib
    if _synth_lib is None:
        if not os.path.exists(SYNTH_LIB_PATH):
            raise DcLibraryMissing(f"{SYNTH_LIB_PATH} is not built")
        l = C.CDLL(SYNTH_LIB_PATH)
        for n in ("dcs_normal_f32", "dcs_normal_bf16"):
            f = getattr(l, n)
            f.restype = C.c_int
            f.argtypes = [C.c_uint64, C.c_uint64, C.c_uint64, C.c_uint64, C.c_float, C.c_void_p, C.c_void_p]
        _synth_lib = l
    return _synth_lib


def synth_normal_device(out, seed: int, stream_id: int, start: int, c: float, stream=None):
    """Fill a float32 or bf16 device tensor with the counter-based stream (see synth.py)."""
    import torch
    l = _synth_loader()
    f = l.dcs_normal_f32 if out.dtype == torch.float32 else l.dcs_normal_bf16
    rc = f(seed, stream_id, start, out.numel(), C.c_float(c), _ptr(out), _stream(stream))
    if rc != 0:
        raise RuntimeError(f"synth kernel launch failed: {rc}")
