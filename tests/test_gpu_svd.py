"""Device compressor, SVD step (dc_svd_device) against the fp64 oracle and the Eckart-Young bound.

Pages: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", "Delta-CoMe的技术原理" (SVD of
the delta); "Delta-CoMe: Training-Free Delta-Compression ...", "Approach".  The device path is a
randomized top-r SVD, so parity is on what an SVD fixes, not on bits (signs and rounding differ):

* the truncation error |Delta - U diag(S) V^T|_F is within 5 % of the Eckart-Young optimum
  sqrt(sum_{i>r} sigma_i^2), sigma from the oracle's SVD or from the constructed spectrum;
* well-separated leading singular values and their rank-k reconstruction match the oracle's;
* U and V have orthonormal columns and the sign rule (largest |v_i| entry positive) holds;
* the whole device pipeline (SVD, device quantiser, serving kernels) matches the oracle evaluated on
  the same device factors, within the serving tolerances.
Shapes: the 512x512 single-linear case, a 512x1024 non-square case, and the 4096x4096 7B shape
with a full-rank long-tail spectrum (sigma_i = 1.28 i^-0.8) truncated at the 1/16 plan's rank 1002.
"""
import math

import numpy as np
import pytest

import oracle
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth

from dc_testlib import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


def _run_svd(w_ft, w_base, r, seed=7, power_iters=2):
    d_out, d_in = w_ft.shape
    over = 16 + r // 10
    U = torch.empty((r, d_out), dtype=torch.float32, device="cuda")
    S = torch.empty(r, dtype=torch.float32, device="cuda")
    Vt = torch.empty((r, d_in), dtype=torch.float32, device="cuda")
    ws = torch.empty(dc.dc_svd_workspace_size(d_out, d_in, r, over), dtype=torch.uint8, device="cuda")
    sweeps = dc.dc_svd_device(w_ft, w_base, r, over, power_iters, seed, U, S, Vt, ws)
    return U.cpu().numpy().astype(np.float64), S.cpu().numpy().astype(np.float64), Vt.cpu().numpy().astype(np.float64), sweeps


def _check_factors(U, S, Vt, D, tail, what):
    r = S.shape[0]
    err = np.linalg.norm(D - (U.T * S) @ Vt)
    assert err <= 1.05 * tail, f"{what}: truncation error {err:.4e} vs Eckart-Young {tail:.4e}"
    assert np.all(np.diff(S) <= 0) and S[-1] > 0, f"{what}: singular values not descending"
    assert np.abs(U @ U.T - np.eye(r)).max() < 1e-3, f"{what}: U columns not orthonormal"
    assert np.abs(Vt @ Vt.T - np.eye(r)).max() < 1e-3, f"{what}: V columns not orthonormal"
    j = np.argmax(np.abs(Vt), axis=1)
    assert np.all(Vt[np.arange(r), j] > 0), f"{what}: sign rule"
    return err


def test_single_linear_case_against_oracle_svd():
    case = synth.single_linear_case(seed=0)
    D = oracle.delta_weights(case.w_base, case.w_ft[0])
    U0, s0, V0 = oracle.svd_factors(D)
    r = 42
    wf = torch.from_numpy(case.w_ft[0].astype(np.float32)).cuda()
    wb = torch.from_numpy(case.w_base.astype(np.float32)).cuda()
    U, S, Vt, sweeps = _run_svd(wf, wb, r)
    _check_factors(U, S, Vt, D, oracle.eckart_young_tail(s0, r), "512x512")
    # the leading 8 singular values stand clear of the noise floor: values and rank-8 part agree
    k = 8
    assert np.max(np.abs(S[:k] - s0[:k]) / s0[:k]) < 1e-2
    R = (U[:k].T * S[:k]) @ Vt[:k]
    R0 = (U0[:, :k] * s0[:k]) @ V0[:k]
    assert np.linalg.norm(R - R0) / np.linalg.norm(R0) < 2e-2
    assert sweeps > 0


def test_non_square_bf16_inputs():
    rng = np.random.default_rng(3)
    d_out, d_in, r = 512, 1024, 64
    s = 0.5 * np.arange(1, d_out + 1) ** -1.0
    Q1, _ = np.linalg.qr(rng.standard_normal((d_out, d_out)))
    Q2, _ = np.linalg.qr(rng.standard_normal((d_in, d_out)))
    D = (Q1 * s) @ Q2.T
    wb32 = (0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32)
    wbb, wbv = synth.bf16_round(wb32)
    wfb, wfv = synth.bf16_round((wbv + D).astype(np.float32))
    Dq = wfv.astype(np.float64) - wbv.astype(np.float64)  # the delta the bf16 inputs hold
    sq = np.linalg.svd(Dq, compute_uv=False)
    wf = torch.from_numpy(wfb.view(np.int16)).cuda().view(torch.bfloat16)
    wb = torch.from_numpy(wbb.view(np.int16)).cuda().view(torch.bfloat16)
    U, S, Vt, _ = _run_svd(wf, wb, r)
    _check_factors(U, S, Vt, Dq, oracle.eckart_young_tail(sq, r), "512x1024 bf16")
    assert np.max(np.abs(S[:10] - sq[:10]) / sq[:10]) < 1e-3


def test_7b_shape_long_tail_full_rank():
    # Delta = Q1 diag(s) Q2^T with every singular value present, made on the device (torch QR of a
    # seeded Gaussian, test input only); the bound uses the constructed spectrum
    d, r = 4096, sum(x for _, x in plans.budget_plan(4096, 4096, 1 / 16, plans.MIXED_1_16))
    g = torch.Generator(device="cuda").manual_seed(11)
    Q1, _ = torch.linalg.qr(torch.randn((d, d), device="cuda", dtype=torch.float64, generator=g))
    Q2, _ = torch.linalg.qr(torch.randn((d, d), device="cuda", dtype=torch.float64, generator=g))
    s = 1.28 * torch.arange(1, d + 1, device="cuda", dtype=torch.float64) ** -0.8
    D = (Q1 * s) @ Q2.T
    wb = (0.02 * torch.randn((d, d), device="cuda", generator=g, dtype=torch.float64)).float()
    wf = (wb.double() + D).float()
    Dq = (wf.double() - wb.double())
    del Q1, Q2
    U, S, Vt, _ = _run_svd(wf, wb, r)
    sv = s.cpu().numpy()
    tail = math.sqrt(float(np.sum(sv[r:] ** 2)))
    Dn = Dq.cpu().numpy()
    # fp32 inputs shift the spectrum by ~1e-7 relative: the constructed tail stands for the optimum
    _check_factors(U, S, Vt, Dn, tail, "4096x4096")
    assert np.max(np.abs(S[:10] - sv[:10]) / sv[:10]) < 1e-3


def test_device_pipeline_matches_oracle_on_device_factors():
    case = synth.single_linear_case(seed=0)
    d_out, d_in = case.w_base.shape
    plan = [(8, 2), (3, 8), (2, 32)]
    r = sum(x for _, x in plan)
    wb = torch.from_numpy(case.w_base.astype(np.float32)).cuda()
    handles, bufs, arts = [], [], {}
    for t in range(2):
        wf = torch.from_numpy(case.w_ft[t].astype(np.float32)).cuda()
        over = 16 + r // 10
        U = torch.empty((r, d_out), dtype=torch.float32, device="cuda")
        S = torch.empty(r, dtype=torch.float32, device="cuda")
        Vt = torch.empty((r, d_in), dtype=torch.float32, device="cuda")
        ws = torch.empty(dc.dc_svd_workspace_size(d_out, d_in, r, over), dtype=torch.uint8, device="cuda")
        dc.dc_svd_device(wf, wb, r, over, 2, 100 + t, U, S, Vt, ws)
        desc = dc.make_desc(d_out, d_in, plan)
        buf = torch.empty(dc.dc_packed_size(desc), dtype=torch.uint8, device="cuda")
        scratch = torch.zeros(dc.dc_quantize_scratch_size(desc), dtype=torch.uint8, device="cuda")
        handles.append(dc.dc_quantize_pack_device(desc, U, Vt, S, buf, scratch))
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(scratch) == 0
        bufs.append(buf)
        Uh = U.cpu().numpy().T.astype(np.float32)
        arts[t] = oracle.compress_factors(Uh, S.cpu().numpy(), Vt.cpu().numpy(), plan)
    import ctypes
    table = torch.empty(2 * ctypes.sizeof(dc.dc_delta_handle), dtype=torch.uint8, device="cuda")
    keep = dc.dc_tenant_table_upload(handles, table)
    ids = case.tenant_ids.astype(np.int32)
    T = len(ids)
    x = torch.from_numpy(case.x.astype(np.float32)).cuda()
    lin = dc.make_linear(wb, d_out, d_in, 2, r, table)
    ws = torch.zeros(dc.dc_workspace_size(T, r, max(d_in, d_out), 1, 2), dtype=torch.uint8, device="cuda")
    for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
        y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
        dc.dc_delta_linear_segmented(lin, x, y, torch.from_numpy(ids).cuda(), T, flags, ws)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(ws) == 0
        xv = case.x.astype(np.float32).astype(np.float64)
        want = oracle.delta_only(arts, xv, ids)
        if flags & dc.DC_BASE:
            want = want + xv @ case.w_base.astype(np.float32).astype(np.float64).T
        assert_close(y.cpu().numpy(), want, f"device pipeline flags={flags}")
    # and its activation error is that of the oracle's own fp64 compression of the same delta
    D = oracle.delta_weights(case.w_base, case.w_ft[0])
    e_dev = oracle.activation_error(D, arts[0], case.x.astype(np.float64))
    e_ref = oracle.activation_error(D, oracle.compress_delta(D, plan), case.x.astype(np.float64))
    assert e_dev <= 1.1 * e_ref + 1e-3, (e_dev, e_ref)
    del keep
