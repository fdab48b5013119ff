"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Integer work (codes, routing) must be bit-exact; floating outputs must meet relative L2 error
<= 1e-3 and max abs error <= 1e-2 * max|y| on the fp32 output, for the full output and for the
delta alone (DC_DELTA), since the delta is a small part of y.
"""
import numpy as np
import pytest

import oracle
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import synth

from dc_testlib import Guarded, TenantDeltas, assert_close, gaussian_factors, oracle_y

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


# shapes chosen to cover: partial 16-rank tiles, rank bands not multiples of 32/128, d_in with a
# tail block of 1..3 groups, 3-bit bands of several steps, 8-bit bands of several tiles
LAYOUT_CASES = [
    (512, 512, [(8, 2), (3, 8), (2, 32)]),
    (384, 640, [(8, 3), (3, 35), (2, 150)]),
    (1024, 384, [(2, 300)]),
    (256, 1152, [(3, 100), (2, 130)]),
    (640, 256, [(8, 40), (2, 200)]),
    (128, 128, [(2, 1)]),
    (1536, 896, [(8, 1), (3, 16), (2, 484)]),
]


@pytest.mark.parametrize("d_out,d_in,plan", LAYOUT_CASES)
def test_codes_bit_exact_through_unpack(d_out, d_in, plan):
    rng = np.random.default_rng(d_out * 7 + d_in)
    r = sum(x for _, x in plan)
    f = gaussian_factors(rng, d_out, d_in, r)
    td = TenantDeltas(torch, d_out, d_in, [f], [plan])
    a = td.artefacts[0]
    cu, cv, su, sv = td.codes[0]
    # host quantiser == oracle quantiser, bit for bit (codes, scales, zeros)
    assert np.array_equal(cu, a.u_codes) and np.array_equal(cv, a.v_codes)
    assert np.array_equal(su[..., 0].view(np.float16).astype(np.float64), a.u_scales)
    assert np.array_equal(sv[..., 0].view(np.float16).astype(np.float64), a.v_scales)
    assert np.array_equal(su[..., 1].view(np.float16).astype(np.float64), a.u_zeros)
    assert np.array_equal(sv[..., 1].view(np.float16).astype(np.float64), a.v_zeros)
    # packed layout decoded by the kernels' own extraction helpers == oracle codes
    gu = Guarded(torch, (r, d_out), torch.uint8, fill=255)
    gv = Guarded(torch, (r, d_in), torch.uint8, fill=255)
    dc.dc_unpack_codes_debug(td.handles[0], 0, gu.t)
    dc.dc_unpack_codes_debug(td.handles[0], 1, gv.t)
    gu.check("unpack U")
    gv.check("unpack V")
    assert np.array_equal(gu.t.cpu().numpy(), a.u_codes.astype(np.uint8))
    assert np.array_equal(gv.t.cpu().numpy(), a.v_codes.astype(np.uint8))


@pytest.mark.parametrize("d_out,d_in,plan", LAYOUT_CASES[:5])
def test_device_quantizer_matches_host_bytes(d_out, d_in, plan):
    rng = np.random.default_rng(d_out + 3 * d_in)
    r = sum(x for _, x in plan)
    f = gaussian_factors(rng, d_out, d_in, r)
    host = TenantDeltas(torch, d_out, d_in, [f], [plan])
    dev = TenantDeltas(torch, d_out, d_in, [f], [plan], device_quantizer=True)
    assert torch.equal(host.buffers[0], dev.buffers[0])


@pytest.mark.parametrize("T,n", [(1, 1), (4, 2), (64, 50), (300, 100), (2048, 16), (17, 3)])
def test_routing_bit_exact(T, n):
    rng = np.random.default_rng(T + n)
    ids = rng.integers(-1, n, size=T).astype(np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    g = Guarded(torch, (dc.dc_workspace_size(T, 0, 0, 1, n),), torch.uint8, fill=0)
    ws = g.t
    dc.dc_build_segments(ids_d, T, n, ws)
    perm = torch.empty(T, dtype=torch.int32, device="cuda")
    inv = torch.empty(T, dtype=torch.int32, device="cuda")
    segs = torch.empty(T * 3, dtype=torch.int32, device="cuda")
    ns = torch.empty(1, dtype=torch.int32, device="cuda")
    dc.dc_read_segments(ws, T, perm, inv, segs, ns)
    torch.cuda.synchronize()
    p, i, s = oracle.route_tokens(ids, n)
    assert np.array_equal(perm.cpu().numpy(), p)
    assert np.array_equal(inv.cpu().numpy(), i)
    k = int(ns.item())
    assert k == len(s)
    assert [tuple(v) for v in segs.cpu().numpy().reshape(T, 3)[:k].tolist()] == s
    assert dc.dc_read_device_status(ws) == 0
    g.check("routing workspace")


def test_routing_bad_id_sets_status():
    ids = torch.tensor([0, 5, 1, -3], dtype=torch.int32, device="cuda")
    ws = torch.zeros(dc.dc_workspace_size(4, 0, 0, 1, 2), dtype=torch.uint8, device="cuda")
    dc.dc_build_segments(ids, 4, 2, ws)
    assert dc.dc_read_device_status(ws) == dc.DC_ERR_TENANT
    assert dc.dc_read_device_status(ws) == 0  # read clears


def _run_linear(td, W, x, ids, flags, out_dtype=None):
    T = x.shape[0]
    n_ten = len(td.handles)
    gy = Guarded(torch, (T, td.d_out), out_dtype or torch.float32)
    gw = Guarded(torch, (dc.dc_workspace_size(T, td.max_rank, max(td.d_in, td.d_out), 1, n_ten),), torch.uint8, fill=0)
    y, ws = gy.t, gw.t
    lin = td.linear(W)
    ids_d = torch.from_numpy(np.asarray(ids, np.int32)).cuda()
    dc.dc_delta_linear_segmented(lin, x, y, ids_d, T, flags, ws)
    torch.cuda.synchronize()
    assert dc.dc_read_device_status(ws) == 0
    gy.check("output")
    gw.check("workspace")
    return y


def test_single_linear_fp32_case():
    """The single 512x512 fp32 linear with two tenants (SVD path of the oracle)."""
    case = synth.single_linear_case(seed=0)
    arts, facs = [], []
    for w in case.w_ft:
        U, s, Vt = oracle.svd_factors(oracle.delta_weights(case.w_base, w))
        r = sum(x for _, x in case.plan)
        facs.append(synth.Factors(np.asfortranarray(U[:, :r].astype(np.float32)), s[:r].astype(np.float32),
                                  Vt[:r].astype(np.float32)))
    td = TenantDeltas(torch, 512, 512, facs, [case.plan] * 2)
    W = torch.from_numpy(case.w_base).cuda()
    x = torch.from_numpy(case.x).cuda()
    wf = case.w_base.astype(np.float64)
    xf = case.x.astype(np.float64)
    for flags in (dc.DC_BASE | dc.DC_DELTA, dc.DC_DELTA, dc.DC_BASE):
        y = _run_linear(td, W, x, case.tenant_ids, flags).cpu().numpy()
        assert_close(y, oracle_y(wf, td, xf, case.tenant_ids, flags), f"flags={flags}")
    # and against the oracle's own compression of the delta (same SVD, same rule)
    full = oracle.delta_linear(case.w_base, [oracle.compress_delta(oracle.delta_weights(case.w_base, w), case.plan)
                                             for w in case.w_ft], case.x, case.tenant_ids)
    y = _run_linear(td, W, x, case.tenant_ids, dc.DC_BASE | dc.DC_DELTA).cpu().numpy()
    assert_close(y, full, "svd path")


def _bf16_case(seed, d_out, d_in, plans, n_ten, ids, none_tenants=()):
    rng = np.random.default_rng(seed)
    facs = [None if t in none_tenants else gaussian_factors(rng, d_out, d_in, sum(r for _, r in plans[t]))
            for t in range(n_ten)]
    td = TenantDeltas(torch, d_out, d_in, facs, plans)
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    xb, xv = synth.bf16_round(rng.standard_normal((len(ids), d_in)).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    return td, W, x, wv.astype(np.float64), xv.astype(np.float64)


@pytest.mark.parametrize("pattern", ["one_each", "multi", "with_backbone_only", "long_runs"])
def test_bf16_linear_token_patterns(pattern):
    n_ten = 6
    d_out, d_in = 768, 640
    plans = [[(8, 2), (3, 32), (2, 90 + 7 * t)] for t in range(n_ten)]
    if pattern == "one_each":
        ids = [3, 0, 5, 1, 4, 2]
    elif pattern == "multi":
        ids = [0, 0, 1, 2, 2, 2, 3, 3, 3, 3, 4, 4, 4, 4, 4, 5, 5, 5, 5, 5, 5, 5, 5, 5]
        ids = list(np.random.default_rng(1).permutation(ids))
    elif pattern == "with_backbone_only":
        ids = [-1, 2, -1, 2, 4, 0, -1]
    else:
        ids = [1] * 40 + [3] * 33 + [-1] * 5 + [0] * 9  # T = 87 > one 64-token block
    td, W, x, wf, xf = _bf16_case(11, d_out, d_in, plans, n_ten, ids, none_tenants=(4,) if pattern == "multi" else ())
    for flags in (dc.DC_BASE | dc.DC_DELTA, dc.DC_DELTA):
        y = _run_linear(td, W, x, ids, flags).cpu().numpy()
        assert_close(y, oracle_y(wf, td, xf, ids, flags), f"{pattern} flags={flags}")


def test_bf16_output_matches_rounded_oracle():
    ids = [0, 1, 2, 1]
    plans = [[(8, 2), (3, 32), (2, 60)]] * 3
    td, W, x, wf, xf = _bf16_case(5, 512, 1024, plans, 3, ids)
    y = _run_linear(td, W, x, ids, dc.DC_BASE | dc.DC_DELTA, out_dtype=torch.bfloat16).float().cpu().numpy()
    ref = oracle_y(wf, td, xf, ids, dc.DC_BASE | dc.DC_DELTA)
    _, ref_b = synth.bf16_round(ref.astype(np.float32))
    # only rounding-boundary flips remain: at most one bf16 ulp anywhere, and rarely
    ulp = np.abs(ref_b.astype(np.float64)) * 2.0 ** -7
    diff = np.abs(y - ref_b)
    assert np.all(diff <= ulp + 1e-30)
    assert np.mean(diff > 0) < 0.02


def test_deterministic_and_permutation_invariant():
    ids = [2, 0, 1, 2, 0, 2, 1, -1, 0]
    plans = [[(8, 2), (3, 16), (2, 100)]] * 3
    td, W, x, wf, xf = _bf16_case(8, 384, 512, plans, 3, ids)
    y1 = _run_linear(td, W, x, ids, dc.DC_BASE | dc.DC_DELTA)
    y2 = _run_linear(td, W, x, ids, dc.DC_BASE | dc.DC_DELTA)
    assert torch.equal(y1, y2)
    p = np.random.default_rng(0).permutation(len(ids))
    xp = x[torch.from_numpy(p).cuda()]
    yp = _run_linear(td, W, xp, [ids[k] for k in p], dc.DC_BASE | dc.DC_DELTA)
    assert torch.equal(yp, y1[torch.from_numpy(p).cuda()])


def test_t_zero_is_noop_and_errors_are_reported():
    plans = [[(2, 32)]]
    td, W, x, wf, xf = _bf16_case(2, 256, 256, plans, 1, [0])
    y = torch.full((1, 256), 7.0, device="cuda")
    ws = torch.zeros(dc.dc_workspace_size(1, td.max_rank, 256, 1, 1), dtype=torch.uint8, device="cuda")
    lin = td.linear(W)
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    dc.dc_delta_linear_segmented(lin, x, y, ids, 0, dc.DC_BASE, ws)
    torch.cuda.synchronize()
    assert float(y[0, 0]) == 7.0
    with pytest.raises(dc.DcError) as e:
        dc.dc_delta_linear_segmented(lin, x, y, ids, 1, dc.DC_BASE, ws[:16])
    assert e.value.status == dc.DC_ERR_WORKSPACE
    bad = dc.make_linear(W, 250, 256, 1, td.max_rank, td.table)
    with pytest.raises(dc.DcError) as e:
        dc.dc_delta_linear_segmented(bad, x, y, ids, 1, dc.DC_BASE, ws)
    assert e.value.status == dc.DC_ERR_SHAPE


@pytest.mark.parametrize("T,d_out,d_in", [(257, 384, 640), (513, 640, 256), (1000, 128, 1152)])
def test_backbone_team_schedule_edges(T, d_out, d_in):
    """Batches of several 256-token blocks run the backbone in teams (one CTA per token block):
    a last block of one token (257), an odd number of row tiles, a single row tile whose units
    every team splits (128 rows x 9 chunks over many teams), against the oracle (full output and
    the delta alone) and against the same batch forced onto the decode delta kernels."""
    rng = np.random.default_rng(T)
    n_ten = 3
    plans = [[(8, 2), (3, 16), (2, 40)], [(2, 64)], [(3, 20)]]
    ids = rng.integers(-1, n_ten, size=T).astype(np.int32)
    td, W, x, wf, xf = _bf16_case(T + d_out, d_out, d_in, plans, n_ten, list(ids))
    outs = {}
    for flags in (dc.DC_BASE | dc.DC_DELTA, dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA | dc.DC_DECODE_ONLY):
        outs[flags] = _run_linear(td, W, x, ids, flags).cpu().numpy()
    assert_close(outs[dc.DC_BASE | dc.DC_DELTA], oracle_y(wf, td, xf, ids, dc.DC_BASE | dc.DC_DELTA), f"T={T} full")
    assert_close(outs[dc.DC_DELTA], oracle_y(wf, td, xf, ids, dc.DC_DELTA), f"T={T} delta")
    assert_close(outs[dc.DC_BASE | dc.DC_DELTA | dc.DC_DECODE_ONLY], oracle_y(wf, td, xf, ids, dc.DC_BASE | dc.DC_DELTA),
                 f"T={T} decode kernels")
