"""Allocation-free entry point (static device workspace) against the workspace-taking one.

dc_delta_linear_segmented_static serves one linear from a workspace compiled into the library.
It must give the same outputs as dc_delta_linear_segmented with a caller workspace, on two calls
in a row (the second call finds the static workspace as the first one left it), and reject
requests whose workspace would not fit before launching anything.  This file is collected last
so that it also runs after every other GPU test in the same process.
"""
from __future__ import annotations

import numpy as np
import pytest

import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import synth

from dc_testlib import TenantDeltas, assert_close, gaussian_factors, oracle_y

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def case():
    import torch

    rng = np.random.default_rng(2024)
    d_out = d_in = 4096
    plan = [(8, 2), (3, 32), (2, 968)]
    n_ten = 6
    factors = [gaussian_factors(rng, d_out, d_in, 1002) for _ in range(n_ten)]
    td = TenantDeltas(torch, d_out, d_in, factors, [plan] * n_ten)
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    T = 64
    ids = rng.integers(0, n_ten, size=T).astype(np.int32)
    ids[[3, 40]] = -1
    xb, xv = synth.bf16_round(rng.standard_normal((T, d_in)).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    return dict(td=td, W=W, x=x, ids=ids, ids_dev=torch.from_numpy(ids).cuda(), T=T, wv=wv, xv=xv,
                lin=td.linear(W))


def _with_workspace(torch, c, flags):
    y = torch.empty((c["T"], c["td"].d_out), dtype=torch.float32, device="cuda")
    ws = torch.zeros(dc.dc_workspace_size(c["T"], c["td"].max_rank, c["td"].d_in, 1, len(c["td"].handles)),
                     dtype=torch.uint8, device="cuda")
    dc.dc_delta_linear_segmented(c["lin"], c["x"], y, c["ids_dev"], c["T"], flags, ws)
    torch.cuda.synchronize()
    assert dc.dc_read_device_status(ws) == 0
    return y.cpu().numpy()


@pytest.mark.parametrize("flags", [dc.DC_BASE | dc.DC_DELTA, dc.DC_DELTA])
def test_static_matches_workspace_entry_point_twice(case, flags):
    import torch

    c = case
    ref = _with_workspace(torch, c, flags)
    for call in range(2):
        y = torch.full((c["T"], c["td"].d_out), float("nan"), dtype=torch.float32, device="cuda")
        status = dc.dc_delta_linear_segmented_static(c["lin"], c["x"], y, c["ids_dev"], c["T"], flags,
                                                     read_status=True)
        assert status == 0, f"call {call}: device status {status}"
        got = y.cpu().numpy()
        assert np.isfinite(got).all()
        assert_close(got, ref, f"static call {call} vs workspace entry point")
    want = oracle_y(c["wv"].astype(np.float64), c["td"], c["xv"].astype(np.float64), c["ids"], flags)
    assert_close(got, want, "static call vs oracle")


def test_static_reports_bad_tenant_then_recovers(case):
    import torch

    c = case
    bad = c["ids"].copy()
    bad[5] = 1000
    y = torch.empty((c["T"], c["td"].d_out), dtype=torch.float32, device="cuda")
    status = dc.dc_delta_linear_segmented_static(c["lin"], c["x"], y, torch.from_numpy(bad).cuda(), c["T"],
                                                 dc.DC_DELTA, read_status=True)
    assert status == dc.DC_ERR_TENANT
    status = dc.dc_delta_linear_segmented_static(c["lin"], c["x"], y, c["ids_dev"], c["T"], dc.DC_DELTA,
                                                 read_status=True)
    assert status == 0


def test_static_rejects_oversize_and_reused_routing(case):
    import torch

    c = case
    big_T = 4096
    need = dc.dc_workspace_size(big_T, c["td"].max_rank, c["td"].d_in, 1, len(c["td"].handles))
    assert need > dc.STATIC_WORKSPACE_BYTES
    y = torch.empty((c["T"], c["td"].d_out), dtype=torch.float32, device="cuda")
    with pytest.raises(dc.DcError) as e:  # rejected on the host, nothing is launched
        dc.dc_delta_linear_segmented_static(c["lin"], c["x"], y, c["ids_dev"], big_T, dc.DC_DELTA)
    assert e.value.status == dc.DC_ERR_WORKSPACE
    with pytest.raises(dc.DcError) as e:
        dc.dc_delta_linear_segmented_static(c["lin"], c["x"], y, c["ids_dev"], c["T"],
                                            dc.DC_DELTA | dc.DC_REUSE_ROUTING)
    assert e.value.status == dc.DC_ERR_INVALID_ARG
