"""Host-side checks of the library that need no GPU: the shared library loads and exports every
entry point include/dc.h declares; the host quantiser reproduces the oracle's codes bit for bit;
descriptor validation returns the documented status codes; plan arithmetic matches the oracle's
rank table.  (No kernel is launched here.)"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from tenant_mixed_precision_b200 import build
    build.build()


def _header_functions():
    text = open(os.path.join(ROOT, "include", "dc.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dc_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _header_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(dc.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/dc.h but not exported"
    assert set(names) == set(dc.exported_symbols())


def test_version_and_error_text():
    assert "sm_100a" in dc.dc_version()
    with pytest.raises(dc.DcError) as e:
        dc.dc_packed_size(dc.make_desc(100, 128, [(2, 4)]))
    assert e.value.status == dc.DC_ERR_INVALID_ARG
    assert "multiples of 128" in dc.dc_last_error()


@pytest.mark.parametrize("desc_args,status", [
    ((128, 100, [(2, 4)]), dc.DC_ERR_SHAPE),
    ((256, 128, [(4, 4)]), dc.DC_ERR_BITS),
    ((256, 128, [(2, 100), (3, 40)]), dc.DC_ERR_SHAPE),
    ((256, 128, [(2, -1)]), dc.DC_ERR_SHAPE),
])
def test_descriptor_errors(desc_args, status):
    d = dc.make_desc(*desc_args)
    U = np.zeros((d.d_out, 8), np.float32)
    Vt = np.zeros((8, d.d_in), np.float32)
    st = dc.lib().dc_quantize_rtn(ctypes.byref(d), U.ctypes.data, Vt.ctypes.data, U.ctypes.data, U.ctypes.data,
                                  U.ctypes.data, U.ctypes.data)
    assert st == status


@pytest.mark.parametrize("d_out,d_in,plan", [
    (512, 512, [(8, 2), (3, 8), (2, 32)]),
    (384, 640, [(8, 3), (3, 35), (2, 150)]),
    (256, 1152, [(3, 100), (2, 130)]),
    (128, 256, [(8, 100)]),
])
def test_host_quantizer_bit_exact_with_oracle(d_out, d_in, plan):
    rng = np.random.default_rng(d_out + d_in)
    r = sum(x for _, x in plan)
    U = (rng.standard_normal((d_out, r)) * rng.uniform(0.001, 1.0, size=r)).astype(np.float32)
    Vt = (rng.standard_normal((r, d_in)) * 0.03).astype(np.float32)
    Vt[0, :128] = 0.0           # an all-zero group
    Vt[1, :128] = np.abs(Vt[1, :128])  # a group with lo forced to 0
    S = np.linspace(1, 0.1, r).astype(np.float32)
    desc = dc.make_desc(d_out, d_in, plan)
    cu, cv, su, sv = dc.dc_quantize_rtn(desc, U, Vt)
    a = oracle.compress_factors(U, S, Vt, plan)
    assert np.array_equal(cu, a.u_codes) and np.array_equal(cv, a.v_codes)
    for got, ref in ((su[..., 0], a.u_scales), (sv[..., 0], a.v_scales), (su[..., 1], a.u_zeros),
                     (sv[..., 1], a.v_zeros)):
        assert np.array_equal(got.view(np.float16).astype(np.float64), ref)


def test_host_quantizer_ties_and_fp16_rounding():
    # values exactly on k + 0.5 grid points and scales that need correct fp16 rounding
    d_out = d_in = 128
    Vt = np.zeros((1, d_in), np.float32)
    Vt[0, :10] = [-0.5, 0.0, 0.25, 1.0, 0.3, -0.2, 0.6, 0.74, 0.75, -0.25]
    U = np.zeros((d_out, 1), np.float32)
    U[:4, 0] = [0.1, 0.2, 0.7, 0.35]
    desc = dc.make_desc(d_out, d_in, [(2, 1)])
    cu, cv, su, sv = dc.dc_quantize_rtn(desc, U, Vt)
    assert list(cv[0, :10]) == [0, 1, 1, 3, 2, 1, 2, 2, 3, 1]
    assert float(sv[0, 0, 0:1].view(np.float16)[0]) == 0.5
    d3 = dc.make_desc(d_out, d_in, [(3, 1)])
    cu3, _, su3, _ = dc.dc_quantize_rtn(d3, U, Vt)
    assert list(cu3[0, :4]) == [1, 2, 7, 4]
    assert float(su3[0, 0, 0:1].view(np.float16)[0]) == 0.0999755859375


def test_host_quantizer_rejects_non_finite():
    desc = dc.make_desc(128, 128, [(2, 1)])
    U = np.zeros((128, 1), np.float32)
    Vt = np.zeros((1, 128), np.float32)
    Vt[0, 3] = np.nan
    with pytest.raises(dc.DcError) as e:
        dc.dc_quantize_rtn(desc, U, Vt)
    assert e.value.status == dc.DC_ERR_INVALID_ARG


def test_packed_size_counts_codes_and_meta():
    for (d_out, d_in), ratio in (((4096, 4096), 1 / 16), ((11008, 4096), 1 / 16), ((4096, 11008), 1 / 32)):
        plan = plans.budget_plan(d_out, d_in, ratio, plans.MIXED_1_16 if ratio == 1 / 16 else plans.MIXED_1_32)
        n = dc.dc_packed_size(dc.make_desc(d_out, d_in, plan))
        r = sum(x for _, x in plan)
        codes = sum(b * x for b, x in plan) * (d_out + d_in) // 8
        meta = r * (d_out + d_in) // 128 * 4 + 4 * r
        assert codes + meta <= n <= codes + meta + 64 * 1024  # alignment and partial-tile meta only


def test_plans_match_oracle_rank_table():
    for d_out, d_in in synth.llama_proj_shapes(4096, 11008) + synth.llama_proj_shapes(5120, 13824):
        for ratio, widths in ((1 / 16, plans.MIXED_1_16), (1 / 32, plans.MIXED_1_32), (1 / 16, plans.ALL_3BIT)):
            assert plans.budget_plan(d_out, d_in, ratio, widths) == oracle.allocate_ranks(d_out, d_in, ratio, widths)


def test_workspace_size_rules():
    assert dc.dc_workspace_size(64, 1470, 11008, 7, 50) > dc.dc_workspace_size(8, 1470, 11008, 7, 50) > 0
    assert dc.dc_workspace_size(64, 1470, 11008, 3, 50) == 0  # n_linears must be 1 or 7


def test_workspace_holds_the_prefill_planes_from_64_tokens():
    """From T = 64 on the workspace also holds the prefill path's fp16 t plane [n_lin][T][tcols]
    (tcols: the ranks rounded up to 64, plus 64 per further band) and the fp16 scaled activations
    [n_in][T][max_d_in]; below 64 tokens it holds neither."""
    max_rank, max_d_in, n_lin, n_in = 1470, 11008, 7, 3
    tcols = (max_rank + 63) // 64 * 64 + 64 * (dc.DC_MAX_BANDS - 1)
    planes = n_lin * 64 * tcols * 2 + n_in * 64 * max_d_in * 2
    ws = {T: dc.dc_workspace_size(T, max_rank, max_d_in, n_lin, 50) for T in (62, 63, 64)}
    per_token = ws[63] - ws[62]
    assert per_token < planes // 8
    assert ws[64] - ws[63] >= planes
    assert ws[64] - ws[63] <= planes + 2 * per_token + 256 * 32  # token-sized regions and alignment


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(dc, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(dc, "_lib", None)
    with pytest.raises(dc.DcLibraryMissing):
        dc.dc_version()
    importlib.reload(dc)
