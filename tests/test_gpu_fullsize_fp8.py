"""Full-size parity of the fp8 (E4M3) backbone option: the 50-tenant 7B decode launches exactly as
`bench.py --fp8-backbone` makes them (7 projections per layer call, 64 tokens, 50 resident tenants,
CUDA graph), on a 4-layer stack (every layer call is the same launch; layers differ only in their
seeded inputs).  Sampled outputs are checked against the oracle's fp8 backbone of regenerated
weights plus the delta oracle: the backbone within the fp32 accumulation bound of
tests/test_gpu_fp8.py, the delta on top of it at the serving path's parity bound.
"""
import numpy as np
import pytest

import oracle
from oracle import fp8 as ofp8
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth
from tenant_mixed_precision_b200.synth_stack import host_activations, host_factors

from dc_testlib import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import bench  # noqa: E402  (the workload definition the benchmark times)

LAYERS = 4


@pytest.fixture(scope="module")
def fp8_stack():
    from tenant_mixed_precision_b200.stack import DeltaStack
    from tenant_mixed_precision_b200.synth_stack import populate

    W = bench.WORKLOAD

    def plan_fn(l, p, d_out, d_in, t):
        return plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)

    stack = DeltaStack(W["hidden"], W["ffn"], LAYERS, W["n_tenants"], W["T"], plan_fn, out_dtype=torch.float32)
    populate(stack, W["seed"])
    stack.to_fp8_backbone()
    ids = bench._ids(W["n_tenants"], W["T"], W["ids_seed"])
    ids_dev = torch.from_numpy(ids).cuda()
    s = torch.cuda.Stream()
    out = {}
    for flags in (dc.DC_BASE | dc.DC_DELTA, dc.DC_BASE):
        with torch.cuda.stream(s):
            stack.forward(ids_dev, W["T"], flags=flags)
        s.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            stack.forward(ids_dev, W["T"], flags=flags)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(stack.ws) == 0
        out[flags] = [[t.clone() for t in row] for row in stack.y]
        del g
    yield stack, ids, out


@pytest.mark.parametrize("layer,proj", [(0, 0), (1, 6), (2, 3), (3, 4)])
def test_sampled_outputs_against_fp8_oracle(fp8_stack, layer, proj):
    stack, ids, out = fp8_stack
    W = bench.WORKLOAD
    d_out, d_in = stack.shapes[proj]
    plan = plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)
    r = sum(x for _, x in plan)
    rng = np.random.default_rng(100 + layer * 10 + proj)
    toks = rng.choice(len(ids), size=3, replace=False)
    rows = np.concatenate([np.arange(128) + 128 * int(rng.integers(0, d_out // 128)) for _ in range(2)])
    _, xv = host_activations(W["seed"], layer, synth.PROJ_INPUT[proj], W["T"], d_in)
    _, wv = synth.stream_base_weight(W["seed"], layer, proj, d_out, d_in, rows=rows)
    # the sampled rows quantised by the oracle (per-row scales: a row needs only itself), and all 64
    # tokens' activations (per-token scales)
    wc, ws = ofp8.quantize_rows(np.asarray(wv, np.float32))
    x = np.asarray(xv, np.float32)[toks]
    ref_b = ofp8.backbone(wc, ws, x)
    xc, xs = ofp8.quantize_rows(x)
    bound = 2.0 * (d_in + 2) * 2.0 ** -24 * (np.abs(ofp8.dequantize_rows(xc, xs)) @ np.abs(ofp8.dequantize_rows(wc, ws)).T)
    got_b = out[dc.DC_BASE][layer][proj].cpu().numpy()[toks][:, rows].astype(np.float64)
    err = np.abs(got_b - ref_b)
    assert np.all(err <= bound + 1e-30), f"backbone error {np.max(err / (bound + 1e-30)):.3f} x the bound"
    arts = {}
    for k in toks:
        t = int(ids[k])
        if t not in arts:
            f = host_factors(W["seed"], layer, proj, t, d_out, d_in, r)
            arts[t] = oracle.compress_factors(f.U, f.S, f.Vt, plan)
    ref_d = oracle.delta_only(arts, x.astype(np.float64), ids[toks], rows=rows)
    got = out[dc.DC_BASE | dc.DC_DELTA][layer][proj].cpu().numpy()[toks][:, rows].astype(np.float64)
    assert_close(got, ref_b + ref_d, f"layer {layer} proj {proj}")
    assert_close(got - got_b, ref_d, f"delta on the fp8 backbone, layer {layer} proj {proj}")


def test_fp8_outputs_finite_and_deterministic(fp8_stack):
    stack, ids, out = fp8_stack
    y0 = out[dc.DC_BASE | dc.DC_DELTA][LAYERS - 1]
    assert all(torch.isfinite(t).all() for t in y0)
    ids_dev = torch.from_numpy(ids).cuda()
    stack.forward(ids_dev, len(ids))
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(y0, stack.y[LAYERS - 1]))
