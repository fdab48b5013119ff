"""Full-size parity: the 50-tenant 7B decode workload exactly as bench.py builds and launches it
(32 layers x 7 projections, 64 tokens, CUDA graph), checked on sampled outputs that the oracle
computes from regenerated inputs, plus size-independent properties on every output.
"""
import numpy as np
import pytest

import oracle
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth
from tenant_mixed_precision_b200.synth_stack import host_activations, host_factors

from dc_testlib import assert_close

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

import bench  # noqa: E402  (the workload definition the benchmark times)


@pytest.fixture(scope="module")
def decode_stack():
    from tenant_mixed_precision_b200.stack import DeltaStack
    from tenant_mixed_precision_b200.synth_stack import populate

    W = bench.WORKLOAD

    def plan_fn(l, p, d_out, d_in, t):
        return plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)

    stack = DeltaStack(W["hidden"], W["ffn"], W["layers"], W["n_tenants"], W["T"], plan_fn, out_dtype=torch.float32)
    populate(stack, W["seed"])
    ids = bench._ids(W["n_tenants"], W["T"], W["ids_seed"])
    ids_dev = torch.from_numpy(ids).cuda()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        stack.forward(ids_dev, W["T"])
    s.synchronize()
    with torch.cuda.graph(g, stream=s):
        stack.forward(ids_dev, W["T"])
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert dc.dc_read_device_status(stack.ws) == 0
    # the same graph launched with the delta alone, so the delta is checked without the backbone
    stack.y_full = [[t.clone() for t in row] for row in stack.y]
    with torch.cuda.stream(s):
        stack.forward(ids_dev, W["T"], flags=dc.DC_DELTA)
    s.synchronize()
    stack.y_delta = [[t.clone() for t in row] for row in stack.y]
    yield stack, ids
    del g


@pytest.mark.parametrize("layer,proj", [(0, 0), (0, 6), (15, 3), (31, 4), (31, 6)])
def test_sampled_outputs_against_oracle(decode_stack, layer, proj):
    stack, ids = decode_stack
    W = bench.WORKLOAD
    d_out, d_in = stack.shapes[proj]
    plan = plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)
    r = sum(x for _, x in plan)
    # three sampled tokens (distinct tenants) and 256 sampled output rows spanning two 128-row groups
    rng = np.random.default_rng(layer * 10 + proj)
    toks = rng.choice(len(ids), size=3, replace=False)
    rows = np.concatenate([np.arange(128) + 128 * int(rng.integers(0, d_out // 128)) for _ in range(2)])
    which = synth.PROJ_INPUT[proj]
    _, xv = host_activations(W["seed"], layer, which, W["T"], d_in)
    _, wv = synth.stream_base_weight(W["seed"], layer, proj, d_out, d_in, rows=rows)
    arts = {}
    for k in toks:
        t = int(ids[k])
        if t not in arts:
            f = host_factors(W["seed"], layer, proj, t, d_out, d_in, r)
            arts[t] = oracle.compress_factors(f.U, f.S, f.Vt, plan)
    x = xv[toks].astype(np.float64)
    ref = oracle.delta_linear(wv.astype(np.float64), arts, x, ids[toks], rows=rows)
    got = stack.y_full[layer][proj].cpu().numpy()[toks][:, rows]
    assert_close(got, ref, f"layer {layer} proj {proj}")
    ref_d = oracle.delta_only(arts, x, ids[toks], rows=rows)
    got_d = stack.y_delta[layer][proj].cpu().numpy()[toks][:, rows]
    assert_close(got_d, ref_d, f"delta layer {layer} proj {proj}")


def test_whole_output_properties(decode_stack):
    """Every output is finite, and tokens of the same tenant with equal inputs would agree: here
    we check the size-independent property that the graph replay is deterministic."""
    stack, ids = decode_stack
    y0 = stack.y_full[31]
    assert all(torch.isfinite(t).all() for t in y0)
    ids_dev = torch.from_numpy(ids).cuda()
    stack.forward(ids_dev, len(ids))
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(y0, stack.y[31]))
