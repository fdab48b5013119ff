"""GPU parity of the prefill delta path: segments of 64 or more tokens in a batch of at least 128
tokens take the tensor-core kernels.  Checked against the fp64 oracle (full output and delta
alone) and against the same batch forced through the decode kernels (DC_DECODE_ONLY), whose
parity is established by test_gpu_parity.py.

The prefill kernels multiply fp16 operands: U_hat and V_hat rounded to fp16 as the method's own
fp16 dequantisation does, and t rounded to fp16.  Each rounding adds about 1.5-2e-4 relative L2
error to the delta, about 3e-4 together (the decode kernels are exact up to fp32), so the delta
alone is held to the parity bound 1e-3 and the full output, where the delta is 1-2 %, to 1e-4.
"""
import numpy as np
import pytest

import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import synth

from dc_testlib import TenantDeltas, assert_close, gaussian_factors, oracle_y, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


def _tol(flags):
    """Bound on the prefill path vs the decode path (fp16 operands, see the module docstring)."""
    return 1e-3 if not (flags & dc.DC_BASE) else 1e-4


def _segments(lengths_tenants):
    ids = []
    for n, t in lengths_tenants:
        ids += [t] * n
    return np.asarray(ids, dtype=np.int32)


# (d_out, d_in, plans per tenant, segments as (length, tenant)); lengths mix the prefill path
# (>= 64 tokens, also > 256 tokens: several token tiles) with short segments and tenant -1
PREFILL_CASES = [
    (512, 384, [[(8, 2), (3, 32), (2, 100)], [(2, 130)], [(8, 3), (3, 35), (2, 150)]],
     [(70, 0), (3, 1), (100, 2), (1, -1), (82, 1), (5, 0)]),
    (384, 640, [[(8, 40), (2, 200)], [(3, 100), (2, 130)]],
     [(300, 0), (64, 1), (63, 1), (20, -1)]),
    (1024, 256, [[(2, 256)], [(8, 1), (3, 16), (2, 111)], [(3, 65)]],
     [(128, 2), (200, 0), (64, 1), (2, 2)]),
]


@pytest.mark.parametrize("case", range(len(PREFILL_CASES)))
@pytest.mark.parametrize("flags", [dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA])
def test_prefill_path_against_oracle_and_decode_path(case, flags):
    d_out, d_in, plans, segs = PREFILL_CASES[case]
    rng = np.random.default_rng(100 + case)
    factors = [gaussian_factors(rng, d_out, d_in, sum(r for _, r in pl)) for pl in plans]
    td = TenantDeltas(torch, d_out, d_in, factors, plans)
    ids = _segments(segs)
    # interleave the runs' order so that tenant-sorted positions differ from batch positions
    T = len(ids)
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    xb, xv = synth.bf16_round(rng.standard_normal((T, d_in)).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    lin = td.linear(W)
    ids_d = torch.from_numpy(ids).cuda()
    ws = torch.zeros(dc.dc_workspace_size(T, td.max_rank, max(d_in, d_out), 1, len(plans)), dtype=torch.uint8,
                     device="cuda")
    outs = {}
    for extra in (0, dc.DC_DECODE_ONLY):
        y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
        dc.dc_delta_linear_segmented(lin, x, y, ids_d, T, flags | extra, ws)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(ws) == 0
        outs[extra] = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(outs[0]).all()
    want = oracle_y(wv.astype(np.float64), td, xv.astype(np.float64), ids, flags)
    assert_close(outs[0], want, "prefill path vs oracle")
    assert rel_l2(outs[0], outs[dc.DC_DECODE_ONLY]) <= _tol(flags), "prefill path vs decode path"


def test_prefill_13b_layer_against_decode_path():
    """One 13B-shaped layer (7 projections), 16 tenants at 1/16, 2048 tokens in segments of
    32-256: the whole output of the prefill path against the decode path."""
    from tenant_mixed_precision_b200 import plans
    from tenant_mixed_precision_b200.stack import DeltaStack
    from tenant_mixed_precision_b200.synth_stack import populate

    T = 2048

    def plan_fn(l, p, d_out, d_in, t):
        return plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)

    st = DeltaStack(5120, 13824, 1, 16, T, plan_fn, out_dtype=torch.float32)
    populate(st, 20244, s0=0.02 * np.sqrt(5120.0))
    ids = synth.prefill_segments(np.random.default_rng(4), T, 16)
    ids_d = torch.from_numpy(ids).cuda()
    res = {}
    for extra in (0, dc.DC_DECODE_ONLY):
        for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
            st.forward(ids_d, T, flags=flags | extra)
            torch.cuda.synchronize()
            assert dc.dc_read_device_status(st.ws) == 0
            res[(extra, flags)] = [y.clone() for y in st.y[0]]
    for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
        for p in range(7):
            a = res[(0, flags)][p].cpu().numpy().astype(np.float64)
            b = res[(dc.DC_DECODE_ONLY, flags)][p].cpu().numpy().astype(np.float64)
            assert np.isfinite(a).all()
            assert rel_l2(a, b) <= _tol(flags), (flags, p, rel_l2(a, b))
