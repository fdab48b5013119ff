"""GPU parity of the fp8 (E4M3) backbone option: the device quantiser against the oracle's, bit for
bit, and the served output against oracle/fp8.py's backbone plus the delta oracle.

Bounds.  The quantiser (weights on the device, activations inside the call) rounds like the oracle:
one IEEE fp32 division, then round-to-nearest-even to E4M3 with saturation, so its codes and scales
are compared exactly (values, so that the negative zero code counts as zero).  The backbone product
of E4M3 values is exact in fp32 (4 x 4 significant bits), so the only errors are the fp32
accumulation of d_in products and the two scale multiplications: elementwise at most
2 (d_in + 2) 2^-24 sum_j |w_hat_j x_hat_j| when each addition is within 2 ulp (rounding or
truncation), which is the bound held here.  The delta keeps the parity bound of the serving path.
"""
import numpy as np
import pytest

import oracle
from oracle import fp8 as ofp8
import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import synth

from dc_testlib import Guarded, TenantDeltas, assert_close, gaussian_factors

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


def _values(codes):
    return ofp8.E4M3_TABLE[np.asarray(codes, np.int64)]


def _dev(a, dtype):
    """Device tensor of a float32 array, as fp32 or as its bf16 rounding; returns (tensor, values)."""
    if dtype == "bf16":
        b, v = synth.bf16_round(np.ascontiguousarray(a, np.float32))
        return torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16), v
    a = np.ascontiguousarray(a, np.float32)
    return torch.from_numpy(a).cuda(), a


def _blob_parts(blob, rows, cols):
    h = blob.cpu().numpy()
    return h[:rows * cols].reshape(rows, cols), h[rows * cols:].view(np.float32)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_device_quantiser_matches_oracle(dtype):
    rng = np.random.default_rng(3)
    rows, cols = 9, 1040  # cols a multiple of 16, not of the block's 512-element sweep
    W = (0.05 * rng.standard_normal((rows, cols))).astype(np.float32)
    W[1] = 0.0                                   # zero row: scale 1, every code 0
    W[2] *= 1e-6                                 # tiny row: the scale carries it
    W[3, ::7] *= 1000.0                          # wide range: most codes subnormal or zero
    W[4] = rng.standard_cauchy(cols).astype(np.float32)
    # amax 448 makes the scale exactly 1, so these land on E4M3 ties and edges
    W[5] = 0.0
    W[5, :8] = [448.0, 1.0625, 1.1875, -2.125, 2.0 ** -10, 3 * 2.0 ** -10, -5 * 2.0 ** -10, 240.0 + 8.0]
    W[6] = -W[4]                                 # signs mirrored
    Wd, Wv = _dev(W, dtype)
    blob = dc.dc_quantize_fp8_rows_device(Wd)
    torch.cuda.synchronize()
    codes, scales = _blob_parts(blob, rows, cols)
    rc, rs = ofp8.quantize_rows(Wv)
    assert np.array_equal(scales.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(_values(codes), _values(rc))
    nz = _values(rc) != 0
    assert np.array_equal(codes[nz], rc[nz])  # identical codes wherever the value is not zero
    # the host quantiser of the library agrees as well
    hc, hs = dc.dc_quantize_fp8_rows(Wv)
    assert np.array_equal(hs.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(_values(hc), _values(rc))


def _fp8_weights(rng, d_out, d_in):
    Wf = (0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32)
    Wf[rng.integers(0, d_out)] *= 30.0  # one row of a larger scale
    Wd = torch.from_numpy(Wf).cuda()
    blob = dc.dc_quantize_fp8_rows_device(Wd)
    codes, scales = ofp8.quantize_rows(Wf)
    got_c, got_s = _blob_parts(blob, d_out, d_in)
    assert np.array_equal(_values(got_c), _values(codes)) and np.array_equal(got_s, scales)
    return blob, codes, scales


def _tokens(rng, T, d_in, dtype):
    x = rng.standard_normal((T, d_in)).astype(np.float32)
    x *= (10.0 ** rng.uniform(-2, 2, size=(T, 1))).astype(np.float32)  # per-token scales differ
    if T > 3:
        x[2] = 0.0  # a zero token: scale 1, codes 0
    return _dev(x, dtype)


def _backbone_bound(codes, scales, xv):
    """2 (d_in + 2) 2^-24 sum_j |w_hat_j x_hat_j| per output (see the module docstring)."""
    xc, xs = ofp8.quantize_rows(xv)
    Xa = np.abs(ofp8.dequantize_rows(xc, xs))
    Wa = np.abs(ofp8.dequantize_rows(codes, scales))
    return 2.0 * (codes.shape[1] + 2) * 2.0 ** -24 * (Xa @ Wa.T)


def _run(lin, x, ids, T, d_out, flags, n_ten, max_rank, d_in):
    gy = Guarded(torch, (T, d_out), torch.float32, fill=float("nan"))
    gw = Guarded(torch, (dc.dc_workspace_size(T, max_rank, max(d_in, d_out), 1, n_ten),), torch.uint8, fill=0)
    dc.dc_delta_linear_segmented(lin, x, gy.t, torch.from_numpy(np.asarray(ids, np.int32)).cuda(), T, flags, gw.t)
    torch.cuda.synchronize()
    assert dc.dc_read_device_status(gw.t) == 0
    gy.check("fp8 output")
    gw.check("fp8 workspace")
    return gy.t.cpu().numpy().astype(np.float64)


# (d_out, d_in, ids): ragged token counts (one partial 16-column block; more than one 256-token
# block, down to a last block of one token), several row tiles, d_in of 4, 5 and 9 chunks of 128,
# long runs that take the prefill delta path
LINEAR_CASES = [
    (384, 640, [1, 0, 2, 1, -1, 0, 0, 2, 1] * 4 + [2]),
    (256, 1152, [0] * 150 + [1] * 3 + [-1] * 7 + [2] * 140),
    (640, 256, [2, -1, 0]),
    (384, 512, [0] * 100 + [2] * 90 + [1] * 67),  # 257 tokens: a last token block of one token
]


@pytest.mark.parametrize("case", range(len(LINEAR_CASES)))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fp8_linear_against_oracle(case, dtype):
    d_out, d_in, ids = LINEAR_CASES[case]
    T = len(ids)
    rng = np.random.default_rng(40 + case)
    plans = [[(8, 2), (3, 16), (2, 60)], [(2, 100)], [(8, 4), (3, 20)]]
    td = TenantDeltas(torch, d_out, d_in, [gaussian_factors(rng, d_out, d_in, sum(r for _, r in pl)) for pl in plans],
                      plans)
    blob, codes, scales = _fp8_weights(rng, d_out, d_in)
    x, xv = _tokens(rng, T, d_in, dtype)
    lin = td.linear(blob)
    assert lin.w_dtype == dc.DC_DTYPE_FP8
    ids_eff = np.asarray(ids, np.int32)
    # fp32 activations: the tensor-core prefill delta path takes bf16 only, so keep the delta on
    # the decode kernels (the backbone is the same kernel either way)
    extra = dc.DC_DECODE_ONLY if dtype == "f32" else 0
    base = _run(lin, x, ids, T, d_out, dc.DC_BASE | extra, 3, td.max_rank, d_in)
    ref_b = ofp8.backbone(codes, scales, xv)
    err = np.abs(base - ref_b)
    bound = _backbone_bound(codes, scales, xv)
    assert np.all(err <= bound + 1e-30), f"backbone error {np.max(err / (bound + 1e-30)):.3f} x the bound"
    both = _run(lin, x, ids, T, d_out, dc.DC_BASE | dc.DC_DELTA | extra, 3, td.max_rank, d_in)
    ref_d = oracle.delta_only(td.oracle_artefacts(), np.asarray(xv, np.float64), ids_eff)
    assert_close(both, ref_b + ref_d, "fp8 backbone + delta")
    assert_close(both - base, ref_d, "delta on top of the fp8 backbone")


def test_fp8_layer_forward_against_oracle():
    """Seven projections of a small decoder layer in one call, one fp8 tensor-core launch for all."""
    hid, ffn, T = 256, 384, 300
    shapes = [(hid, hid)] * 4 + [(ffn, hid), (ffn, hid), (hid, ffn)]
    rng = np.random.default_rng(77)
    plans = [[(8, 2), (3, 12), (2, 40)], [(2, 64)], [(3, 30)]]
    ids = np.asarray([0] * 120 + [1] * 3 + [2] * 90 + [-1] * 2 + [1] * 85, np.int32)
    tds, blobs, refw = [], [], []
    for d_out, d_in in shapes:
        tds.append(TenantDeltas(torch, d_out, d_in,
                                [gaussian_factors(rng, d_out, d_in, sum(r for _, r in pl)) for pl in plans], plans))
        b, c, s = _fp8_weights(rng, d_out, d_in)
        blobs.append(b)
        refw.append((c, s))
    xs = [_tokens(rng, T, d, "bf16") for d in (hid, hid, ffn)]
    lins = [td.linear(b) for td, b in zip(tds, blobs)]
    max_rank = max(td.max_rank for td in tds)
    gw = Guarded(torch, (dc.dc_workspace_size(T, max_rank, max(hid, ffn), 7, 3),), torch.uint8, fill=0)
    ys = [Guarded(torch, (T, d_out), torch.float32, fill=float("nan")) for d_out, _ in shapes]
    dc.dc_layer_forward(lins, xs[0][0], xs[1][0], xs[2][0], [g.t for g in ys], torch.from_numpy(ids).cuda(), T,
                        dc.DC_BASE | dc.DC_DELTA, gw.t)
    torch.cuda.synchronize()
    assert dc.dc_read_device_status(gw.t) == 0
    gw.check("layer workspace")
    for p, (td, (c, s)) in enumerate(zip(tds, refw)):
        ys[p].check(f"output {p}")
        xv = xs[1 if p == 3 else (2 if p == 6 else 0)][1]
        ref = ofp8.backbone(c, s, xv) + oracle.delta_only(td.oracle_artefacts(), np.asarray(xv, np.float64), ids)
        assert_close(ys[p].t.cpu().numpy(), ref, f"projection {p}")


def test_fp8_static_entry_matches_workspace_entry():
    d_out, d_in = 512, 512
    ids = [0, 1, -1, 1] * 16
    rng = np.random.default_rng(5)
    plans = [[(2, 64)], [(8, 2), (3, 10)]]
    td = TenantDeltas(torch, d_out, d_in, [gaussian_factors(rng, d_out, d_in, sum(r for _, r in pl)) for pl in plans],
                      plans)
    blob, _, _ = _fp8_weights(rng, d_out, d_in)
    x, _ = _tokens(rng, len(ids), d_in, "bf16")
    lin = td.linear(blob)
    want = _run(lin, x, ids, len(ids), d_out, dc.DC_BASE | dc.DC_DELTA, 2, td.max_rank, d_in)
    y = torch.empty(len(ids), d_out, dtype=torch.float32, device="cuda")
    status = dc.dc_delta_linear_segmented_static(lin, x, y, torch.from_numpy(np.asarray(ids, np.int32)).cuda(),
                                                 len(ids), dc.DC_BASE | dc.DC_DELTA, read_status=True)
    assert status == 0
    assert np.array_equal(y.cpu().numpy().astype(np.float64), want)
