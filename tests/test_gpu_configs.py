"""GPU parity on the remaining workload shapes and edge cases.

* one Llama-2-7B-shaped layer in bf16 (q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008),
  8 tenants at the 1/16 budget, a decode batch of 8 tokens with one token per tenant: every
  output of three projections (q, gate, down: the three shapes) against the oracle;
* the 13B-shaped prefill layer (2048 tokens in segments of 32-256, 16 tenants): sampled outputs
  of q, gate and down against the oracle, with sampled tokens taken both from tenants with 64+
  tokens (the tensor-core prefill path) and from a tenant with fewer (the decode kernels); the
  same layer with the fp8 (E4M3) backbone option against the oracle's fp8 backbone;
* edge cases: a batch of backbone-only tokens, tenants without a delta, one token.
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


def _stack(hidden, ffn, n_ten, T, seed, s0):
    from tenant_mixed_precision_b200.stack import DeltaStack
    from tenant_mixed_precision_b200.synth_stack import populate

    def plan_fn(l, p, d_out, d_in, t):
        return plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)

    st = DeltaStack(hidden, ffn, 1, n_ten, T, plan_fn, out_dtype=torch.float32)
    populate(st, seed, s0=s0)
    return st


def _run(st, ids, flags):
    ids_d = torch.from_numpy(ids).cuda()
    st.forward(ids_d, len(ids), flags=flags)
    torch.cuda.synchronize()
    assert dc.dc_read_device_status(st.ws) == 0
    return [y.cpu().numpy().astype(np.float64) for y in st.y[0]]


def _oracle(seed, s0, proj, d_out, d_in, T, ids, toks, rows, flags):
    plan = plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)
    r = sum(x for _, x in plan)
    _, xv = host_activations(seed, 0, synth.PROJ_INPUT[proj], T, d_in)
    arts = {}
    for k in toks:
        t = int(ids[k])
        if t >= 0 and t not in arts:
            f = host_factors(seed, 0, proj, t, d_out, d_in, r, s0=s0)
            arts[t] = oracle.compress_factors(f.U, f.S, f.Vt, plan)
    x = xv[toks].astype(np.float64)
    if flags & dc.DC_BASE:
        _, wv = synth.stream_base_weight(seed, 0, proj, d_out, d_in, rows=rows)
        return oracle.delta_linear(wv.astype(np.float64), arts, x, ids[toks], rows=rows)
    return oracle.delta_only(arts, x, ids[toks], rows=rows)


def test_one_7b_layer_8_tenants_one_token_each():
    seed, s0, T = 20242, 0.02 * np.sqrt(4096.0), 8
    st = _stack(4096, 11008, 8, T, seed, s0)
    ids = np.arange(8, dtype=np.int32)
    full = _run(st, ids, dc.DC_BASE | dc.DC_DELTA)
    delta = _run(st, ids, dc.DC_DELTA)
    toks = np.arange(T)
    for proj in (0, 4, 6):  # q (4096x4096), gate (11008x4096), down (4096x11008)
        d_out, d_in = st.shapes[proj]
        rows = np.arange(d_out)
        ref = _oracle(seed, s0, proj, d_out, d_in, T, ids, toks, rows, dc.DC_BASE | dc.DC_DELTA)
        assert_close(full[proj], ref, f"7B layer proj {proj}")
        ref_d = _oracle(seed, s0, proj, d_out, d_in, T, ids, toks, rows, dc.DC_DELTA)
        assert_close(delta[proj], ref_d, f"7B layer proj {proj} delta")
    for y in full + delta:
        assert np.isfinite(y).all()


PF_MIN = 64  # a tenant with this many tokens in a batch of 128+ takes the prefill path (include/dc.h)


def test_13b_prefill_layer_sampled_against_oracle():
    seed, s0, T = 20244, 0.02 * np.sqrt(5120.0), 2048
    st = _stack(5120, 13824, 16, T, seed, s0)
    ids = synth.prefill_segments(np.random.default_rng(4), T, 16)
    full = _run(st, ids, dc.DC_BASE | dc.DC_DELTA)
    delta = _run(st, ids, dc.DC_DELTA)
    rng = np.random.default_rng(7)
    # two tokens of tenants with 64+ tokens in the batch (the tensor-core prefill path), one of the
    # tenant with fewer (the decode kernels), and one at random
    counts = np.bincount(ids, minlength=16)
    long_t = [k for k in range(T) if counts[ids[k]] >= PF_MIN]
    short_t = [k for k in range(T) if 0 < counts[ids[k]] < PF_MIN]
    assert long_t and short_t, "the prefill draw should hold both kinds of segment"
    picks = [long_t[0], long_t[-1], short_t[len(short_t) // 2], int(rng.integers(0, T))]
    toks = np.array(sorted(set(int(k) for k in picks)))
    assert counts[ids[toks]].max() >= PF_MIN and counts[ids[toks]].min() < PF_MIN
    for proj in (0, 4, 6):  # q (5120x5120), gate (13824x5120) and down (5120x13824)
        d_out, d_in = st.shapes[proj]
        rows = np.concatenate([np.arange(128) + 128 * int(rng.integers(0, d_out // 128)) for _ in range(2)])
        ref = _oracle(seed, s0, proj, d_out, d_in, T, ids, toks, rows, dc.DC_BASE | dc.DC_DELTA)
        assert_close(full[proj][toks][:, rows], ref, f"13B prefill proj {proj}")
        ref_d = _oracle(seed, s0, proj, d_out, d_in, T, ids, toks, rows, dc.DC_DELTA)
        assert_close(delta[proj][toks][:, rows], ref_d, f"13B prefill proj {proj} delta")


@pytest.mark.parametrize("case", ["all_backbone", "tenants_without_delta", "one_token"])
def test_edge_cases(case):
    rng = np.random.default_rng(11)
    d_out, d_in = 640, 384
    plan = [(8, 2), (3, 20), (2, 90)]
    if case == "tenants_without_delta":
        factors = [gaussian_factors(rng, d_out, d_in, 112), None, gaussian_factors(rng, d_out, d_in, 112), None]
        ids = np.array([1, 0, 3, 2, 1, -1, 0, 3, 3, 1], dtype=np.int32)
    else:
        factors = [gaussian_factors(rng, d_out, d_in, 112) for _ in range(3)]
        ids = np.full(9, -1, dtype=np.int32) if case == "all_backbone" else np.array([2], dtype=np.int32)
    plans_ = [plan if f is not None else None for f in factors]
    td = TenantDeltas(torch, d_out, d_in, factors, plans_)
    T = len(ids)
    wb, wv = synth.bf16_round((0.02 * rng.standard_normal((d_out, d_in))).astype(np.float32))
    xb, xv = synth.bf16_round(rng.standard_normal((T, d_in)).astype(np.float32))
    W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    lin = td.linear(W)
    ws = torch.zeros(dc.dc_workspace_size(T, max(td.max_rank, 1), max(d_in, d_out), 1, len(factors)), dtype=torch.uint8,
                     device="cuda")
    for flags in (dc.DC_DELTA, dc.DC_BASE | dc.DC_DELTA):
        y = torch.full((T, d_out), float("nan"), dtype=torch.float32, device="cuda")
        dc.dc_delta_linear_segmented(lin, x, y, torch.from_numpy(ids).cuda(), T, flags, ws)
        torch.cuda.synchronize()
        assert dc.dc_read_device_status(ws) == 0
        got = y.cpu().numpy().astype(np.float64)
        want = oracle_y(wv.astype(np.float64), td, xv.astype(np.float64), ids, flags)
        if not (flags & dc.DC_BASE) and not np.any(want):
            assert np.array_equal(got, want), case  # no delta anywhere: exactly zero
        else:
            assert_close(got, want, f"{case} flags={flags}")


def test_13b_prefill_layer_fp8_backbone_sampled_against_oracle():
    """The same 13B prefill layer with the fp8 (E4M3) backbone option: sampled outputs against the
    oracle's fp8 backbone of the regenerated weights (within the fp32 accumulation bound of
    tests/test_gpu_fp8.py) plus the delta oracle (at the serving path's parity bound)."""
    from oracle import fp8 as ofp8

    seed, s0, T = 20244, 0.02 * np.sqrt(5120.0), 2048
    st = _stack(5120, 13824, 16, T, seed, s0)
    st.to_fp8_backbone()
    ids = synth.prefill_segments(np.random.default_rng(4), T, 16)
    full = _run(st, ids, dc.DC_BASE | dc.DC_DELTA)
    base = _run(st, ids, dc.DC_BASE)
    rng = np.random.default_rng(9)
    counts = np.bincount(ids, minlength=16)
    long_t = [k for k in range(T) if counts[ids[k]] >= PF_MIN]
    short_t = [k for k in range(T) if 0 < counts[ids[k]] < PF_MIN]
    toks = np.array(sorted({long_t[0], long_t[-1], short_t[len(short_t) // 2], int(rng.integers(0, T))}))
    for proj in (0, 4, 6):
        d_out, d_in = st.shapes[proj]
        rows = np.concatenate([np.arange(128) + 128 * int(rng.integers(0, d_out // 128)) for _ in range(2)])
        _, xv = host_activations(seed, 0, synth.PROJ_INPUT[proj], T, d_in)
        _, wv = synth.stream_base_weight(seed, 0, proj, d_out, d_in, rows=rows)
        wc, ws = ofp8.quantize_rows(np.asarray(wv, np.float32))
        x = np.asarray(xv, np.float32)[toks]
        ref_b = ofp8.backbone(wc, ws, x)
        xc, xs = ofp8.quantize_rows(x)
        bound = 2.0 * (d_in + 2) * 2.0 ** -24 * (np.abs(ofp8.dequantize_rows(xc, xs)) @ np.abs(ofp8.dequantize_rows(wc, ws)).T)
        got_b = base[proj][toks][:, rows]
        assert np.all(np.abs(got_b - ref_b) <= bound + 1e-30), f"fp8 backbone, proj {proj}"
        ref_d = _oracle(seed, s0, proj, d_out, d_in, T, ids, toks, rows, dc.DC_DELTA)
        assert_close(full[proj][toks][:, rows] - got_b, ref_d, f"13B fp8 prefill proj {proj} delta")
        assert_close(full[proj][toks][:, rows], ref_b + ref_d, f"13B fp8 prefill proj {proj}")
