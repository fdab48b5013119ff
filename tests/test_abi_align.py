"""Every device entry point refuses a misaligned device pointer with DC_ERR_ALIGN before it touches
the device (the C ABI's convention: device pointers 16-byte aligned, packed blobs, arenas and the SVD
workspace 256-byte aligned).

The calls go straight through ctypes with made-up addresses, so this runs only where no GPU is
visible: the checks must come before any CUDA call, and no kernel may see these addresses.
"""
import ctypes as C

import numpy as np
import pytest

import tenant_mixed_precision_b200 as dc

torch = pytest.importorskip("torch")
if torch.cuda.is_available():  # pragma: no cover - the made-up addresses must never reach a device
    pytest.skip("host-side argument checks only (no GPU visible)", allow_module_level=True)

A = 0x7f0000000000      # an aligned made-up device address
MIS = A + 4             # misaligned by 4 bytes
BIG = 1 << 40           # a size no check refuses


def _lin(W=A, tab=A):
    return dc.make_linear(W, 512, 384, 2, 64, tab, w_dtype=dc.DC_DTYPE_BF16)


def _status(f, *args):
    lib = dc.lib()
    return getattr(lib, f)(*args)


def test_build_segments():
    assert _status("dc_build_segments", A, 4, 2, MIS, BIG, None) == dc.DC_ERR_ALIGN


@pytest.mark.parametrize("which", ["x", "y", "ws", "W"])
def test_delta_linear_segmented(which):
    lin = _lin(W=MIS if which == "W" else A)
    x = MIS if which == "x" else A
    y = MIS if which == "y" else A
    ws = MIS if which == "ws" else A
    st = _status("dc_delta_linear_segmented", C.byref(lin), x, y, A, 4, dc.DC_DTYPE_BF16, dc.DC_DTYPE_F32,
                 dc.DC_BASE | dc.DC_DELTA, ws, BIG, None)
    assert st == dc.DC_ERR_ALIGN


@pytest.mark.parametrize("which", ["x", "y", "W"])
def test_delta_linear_segmented_static(which):
    lin = _lin(W=MIS if which == "W" else A)
    st = _status("dc_delta_linear_segmented_static", C.byref(lin), MIS if which == "x" else A,
                 MIS if which == "y" else A, A, 4, dc.DC_DTYPE_BF16, dc.DC_DTYPE_F32, dc.DC_BASE, None, None)
    assert st == dc.DC_ERR_ALIGN


def test_layer_forward():
    lins = (dc.dc_linear * 7)(*[dc.make_linear(A, 512, 512 if p != 6 else 1024, 2, 64, A,
                                               w_dtype=dc.DC_DTYPE_BF16) for p in range(7)])
    ys = (C.c_void_p * 7)(*[A] * 7)
    st = _status("dc_layer_forward", lins, MIS, A, A, ys, A, 4, dc.DC_DTYPE_BF16, dc.DC_DTYPE_F32, dc.DC_BASE, A,
                 BIG, None)
    assert st == dc.DC_ERR_ALIGN


def test_pack_upload_and_device_quantiser():
    desc = dc.make_desc(256, 256, [(2, 16)])
    cu = np.zeros((16, 256), np.uint8)
    su = np.zeros((16, 2, 2), np.uint16)
    S = np.ones(16, np.float32)
    h = dc.dc_delta_handle()
    st = _status("dc_pack_upload", C.byref(desc), cu.ctypes.data, cu.ctypes.data, su.ctypes.data, su.ctypes.data,
                 S.ctypes.data, A + 16, BIG, None, C.byref(h))
    assert st == dc.DC_ERR_ALIGN  # blobs need 256 bytes
    st = _status("dc_quantize_pack_device", C.byref(desc), A, A, A, A + 16, BIG, A, BIG, None, C.byref(h))
    assert st == dc.DC_ERR_ALIGN
    st = _status("dc_quantize_pack_device", C.byref(desc), MIS, A, A, A, BIG, A, BIG, None, C.byref(h))
    assert st == dc.DC_ERR_ALIGN


def test_tenant_table_and_checks():
    hs = (dc.dc_delta_handle * 1)()
    assert _status("dc_tenant_table_upload", hs, 1, MIS, BIG, None) == dc.DC_ERR_ALIGN
    assert _status("dc_read_segments", A, 4, MIS, A, A, A, None) == dc.DC_ERR_ALIGN
    assert _status("dc_read_segments", MIS, 4, A, A, A, A, None) == dc.DC_ERR_ALIGN
    v = C.c_int32(0)
    assert _status("dc_read_device_status", MIS, None, C.byref(v)) == dc.DC_ERR_ALIGN
    h = dc.dc_delta_handle()
    h.dev_base = A
    h.desc = dc.make_desc(256, 256, [(2, 16)])
    assert _status("dc_unpack_codes_debug", C.byref(h), 0, MIS, None) == dc.DC_ERR_ALIGN


def test_pager_and_svd():
    d = dc.dc_pager_desc(4, 2, 1 << 20, 1, 0)
    tabs = (C.c_void_p * 1)(A)
    out = C.c_void_p()
    st = _status("dc_pager_create", C.byref(d), A + 16, BIG, tabs, A, BIG, C.byref(out))
    assert st == dc.DC_ERR_ALIGN
    st = _status("dc_pager_create", C.byref(d), A, BIG, tabs, MIS, BIG, C.byref(out))
    assert st == dc.DC_ERR_ALIGN
    sw = C.c_int32(0)
    st = _status("dc_svd_device", A, A, dc.DC_DTYPE_F32, 512, 512, 8, 8, 1, 0, A, A, A, A + 16, BIG, None, C.byref(sw))
    assert st == dc.DC_ERR_ALIGN
    st = _status("dc_svd_device", MIS, A, dc.DC_DTYPE_F32, 512, 512, 8, 8, 1, 0, A, A, A, A, BIG, None, C.byref(sw))
    assert st == dc.DC_ERR_ALIGN


def test_fp8_quantiser_and_backbone_checks():
    assert _status("dc_quantize_fp8_rows_device", MIS, dc.DC_DTYPE_F32, 4, 128, A, A, None) == dc.DC_ERR_ALIGN
    assert _status("dc_quantize_fp8_rows_device", A, dc.DC_DTYPE_F32, 4, 128, A, MIS, None) == dc.DC_ERR_ALIGN
    assert _status("dc_quantize_fp8_rows_device", A, dc.DC_DTYPE_F32, 4, 120, A, A, None) == dc.DC_ERR_SHAPE
    assert _status("dc_quantize_fp8_rows_device", A, dc.DC_DTYPE_FP8, 4, 128, A, A, None) == dc.DC_ERR_INVALID_ARG
    # an fp8 backbone is all or nothing within one call (one tensor-core kernel serves every linear)
    lins = (dc.dc_linear * 7)(*[dc.make_linear(A, 512, 512 if p != 6 else 1024, 2, 64, A,
                                               w_dtype=dc.DC_DTYPE_FP8 if p != 4 else dc.DC_DTYPE_BF16)
                                for p in range(7)])
    ys = (C.c_void_p * 7)(*[A] * 7)
    st = _status("dc_layer_forward", lins, A, A, A, ys, A, 4, dc.DC_DTYPE_BF16, dc.DC_DTYPE_F32, dc.DC_BASE, A,
                 BIG, None)
    assert st == dc.DC_ERR_UNSUPPORTED
