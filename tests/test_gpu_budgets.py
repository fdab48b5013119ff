"""GPU parity for the stress-sweep workload: 7B-shaped linears with the 1/16 mixed budget, the
1/32 mixed budget (8-bit rank 1, 3-bit rank 16, 2-bit fill) and the single-precision all-3-bit
allocation of the 1/16 size, Zipf(1.1) tenant popularity and batches of 1, 16 and 256 tokens.
At 256 tokens the most popular tenants have segments of 64+ tokens, so the batch mixes the decode
kernels and the tensor-core prefill kernels.  Checked against the fp64 oracle on the fp32
output, for the full output and for the delta alone.
"""
import numpy as np
import pytest

import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth

from dc_testlib import TenantDeltas, assert_close, gaussian_factors, oracle_y

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

BUDGETS = {
    "1/16": (1 / 16, plans.MIXED_1_16),
    "1/32": (1 / 32, plans.MIXED_1_32),
    "all-3-bit": (1 / 16, plans.ALL_3BIT),
}
N_TENANTS = 10


@pytest.fixture(scope="module", params=sorted(BUDGETS))
def budget_case(request):
    ratio, widths = BUDGETS[request.param]
    d_out, d_in = 4096, 4096
    plan = plans.budget_plan(d_out, d_in, ratio, widths)
    r = sum(x for _, x in plan)
    rng = np.random.default_rng(5)
    factors = [gaussian_factors(rng, d_out, d_in, r) for _ in range(N_TENANTS)]
    td = TenantDeltas(torch, d_out, d_in, factors, [plan] * N_TENANTS, device_quantizer=True)
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    return request.param, plan, td, W, wv


@pytest.mark.parametrize("T", [1, 16, 256])
def test_budget_zipf_batch(budget_case, T):
    name, plan, td, W, wv = budget_case
    rng = np.random.default_rng(50 + T)
    ids = synth.zipf_tenants(rng, T, N_TENANTS)
    xb, xv = synth.bf16_round(rng.standard_normal((T, td.d_in)).astype(np.float32))
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    lin = td.linear(W)
    ws = torch.zeros(dc.dc_workspace_size(T, td.max_rank, td.d_in, 1, N_TENANTS), dtype=torch.uint8, device="cuda")
    ids_d = torch.from_numpy(ids).cuda()
    for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
        y = torch.full((T, td.d_out), float("nan"), dtype=torch.float32, device="cuda")
        dc.dc_delta_linear_segmented(lin, x, y, ids_d, T, flags, ws)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(ws) == 0
        want = oracle_y(wv.astype(np.float64), td, xv.astype(np.float64), ids, flags)
        assert_close(y.cpu().numpy(), want, f"{name} T={T} flags={flags}")
