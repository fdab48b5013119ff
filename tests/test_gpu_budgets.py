"""GPU parity for the stress-sweep workload: the three 7B linear shapes (4096x4096, 11008x4096,
4096x11008) under the 1/16 mixed budget, the 1/32 mixed budget (8-bit rank 1, 3-bit rank 16, 2-bit
fill) and the single-precision all-3-bit allocation of the 1/16 size, with Zipf(1.1) tenant
popularity and batches of 1, 16 and 256 tokens.  The all-3-bit plan at 11008 output rows keeps
995 three-bit ranks, so the delta-output kernel runs many 3-bit steps per 128-row group.  At 256
tokens over few tenants the most popular tenants have segments of 64+ tokens, so the batch mixes
the decode kernels and the tensor-core prefill kernels.

A second test serves the bench's own 100-tenant Zipf stack (its seed, its plans, its routing
draw; two layers instead of 32, which changes no launch of a layer) and checks sampled outputs of
layer 1 (the routing reused from layer 0) against the oracle.

Compared with the fp64 oracle on the fp32 output, for the full output and for the delta alone.
"""
import numpy as np
import pytest

import oracle
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth
from tenant_mixed_precision_b200.synth_stack import host_activations, host_factors

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
SHAPES = {"4096x4096": (4096, 4096, 10), "11008x4096": (11008, 4096, 6), "4096x11008": (4096, 11008, 6)}


@pytest.fixture(scope="module", params=[(b, s) for b in sorted(BUDGETS) for s in SHAPES])
def budget_case(request):
    bname, sname = request.param
    ratio, widths = BUDGETS[bname]
    d_out, d_in, n_ten = SHAPES[sname]
    plan = plans.budget_plan(d_out, d_in, ratio, widths)
    r = sum(x for _, x in plan)
    rng = np.random.default_rng(5 + d_out + 3 * d_in)
    factors = [gaussian_factors(rng, d_out, d_in, r) for _ in range(n_ten)]
    td = TenantDeltas(torch, d_out, d_in, factors, [plan] * n_ten, device_quantizer=True)
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    yield f"{bname} {sname}", plan, td, W, wv, n_ten
    del td, W
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [1, 16, 256])
def test_budget_zipf_batch(budget_case, T):
    name, plan, td, W, wv, n_ten = budget_case
    rng = np.random.default_rng(50 + T)
    ids = synth.zipf_tenants(rng, T, n_ten)
    xb, xv = synth.bf16_round(rng.standard_normal((T, td.d_in)).astype(np.float32))
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    lin = td.linear(W)
    ws = torch.zeros(dc.dc_workspace_size(T, td.max_rank, max(td.d_in, td.d_out), 1, n_ten), dtype=torch.uint8,
                     device="cuda")
    ids_d = torch.from_numpy(ids).cuda()
    for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
        y = torch.full((T, td.d_out), float("nan"), dtype=torch.float32, device="cuda")
        dc.dc_delta_linear_segmented(lin, x, y, ids_d, T, flags, ws)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(ws) == 0
        want = oracle_y(wv.astype(np.float64), td, xv.astype(np.float64), ids, flags)
        assert_close(y.cpu().numpy(), want, f"{name} T={T} flags={flags} plan={plan}")


SWEEP_SEED = 20245  # the seed the bench's sweep populates its stack with


@pytest.mark.parametrize("bname,T", [("1/16", 256), ("1/32", 64), ("all-3-bit", 256)])
def test_bench_zipf_stack_sampled(bname, T):
    from tenant_mixed_precision_b200.stack import DeltaStack
    from tenant_mixed_precision_b200.synth_stack import populate

    ratio, widths = BUDGETS[bname]
    n_ten, layers = 100, 2

    def plan_fn(l, p, d_out, d_in, t):
        return plans.budget_plan(d_out, d_in, ratio, widths)

    st = DeltaStack(4096, 11008, layers, n_ten, T, plan_fn, out_dtype=torch.float32)
    populate(st, SWEEP_SEED)
    ids = synth.zipf_tenants(np.random.default_rng(5000 + T), T, n_ten)  # the bench's draw for this T
    ids_d = torch.from_numpy(ids).cuda()
    outs = {}
    for flags in (dc.DC_BASE | dc.DC_DELTA, dc.DC_DELTA):
        st.forward(ids_d, T, flags=flags)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(st.ws) == 0
        outs[flags] = [y.cpu().numpy().astype(np.float64) for y in st.y[1]]
    counts = np.bincount(ids, minlength=n_ten)
    rng = np.random.default_rng(T)
    # tokens of the most popular tenant (its longest segment), of a tenant with a single token, and one more
    top = np.flatnonzero(ids == int(np.argmax(counts)))
    single = [k for k in range(T) if counts[ids[k]] == 1]
    toks = sorted({int(top[0]), int(top[-1]), int(single[0]) if single else int(top[1]), int(rng.integers(0, T))})
    toks = np.array(toks)
    for proj in (0, 4, 6):
        d_out, d_in = st.shapes[proj]
        plan = plan_fn(1, proj, d_out, d_in, 0)
        r = sum(x for _, x in plan)
        rows = np.concatenate([np.arange(128) + 128 * int(rng.integers(0, d_out // 128)) for _ in range(2)])
        _, xv = host_activations(SWEEP_SEED, 1, synth.PROJ_INPUT[proj], T, d_in)
        _, wv = synth.stream_base_weight(SWEEP_SEED, 1, proj, d_out, d_in, rows=rows)
        arts = {}
        for k in toks:
            t = int(ids[k])
            if t not in arts:
                f = host_factors(SWEEP_SEED, 1, proj, t, d_out, d_in, r)
                arts[t] = oracle.compress_factors(f.U, f.S, f.Vt, plan)
        x = xv[toks].astype(np.float64)
        ref = oracle.delta_linear(wv.astype(np.float64), arts, x, ids[toks], rows=rows)
        assert_close(outs[dc.DC_BASE | dc.DC_DELTA][proj][toks][:, rows], ref, f"{bname} T={T} proj {proj}")
        ref_d = oracle.delta_only(arts, x, ids[toks], rows=rows)
        assert_close(outs[dc.DC_DELTA][proj][toks][:, rows], ref_d, f"{bname} T={T} proj {proj} delta")
    del st
    torch.cuda.empty_cache()
