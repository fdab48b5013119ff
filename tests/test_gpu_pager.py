"""Tenant paging on the GPU: the tenants of a resident stack served from fewer device slots.

Frequently used tenants stay resident and long-tail ones are loaded on demand (page
"Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", FAQ "多模型同机部署最该关注什么？").
A resident stack and a paged view of the same tenants (same weights, inputs, kernels) serve a
sequence of Zipf batches; the paged outputs must equal the resident ones bit for bit, including
for tenants that were evicted and loaded again, with the copies on their own stream.  A batch with
more tenants than slots is refused without touching the pager's state.
"""
import numpy as np
import pytest

import tenant_mixed_precision_b200 as dc
from tenant_mixed_precision_b200 import plans, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)


@pytest.fixture(scope="module")
def stacks():
    from tenant_mixed_precision_b200.stack import DeltaStack, PagedStack
    from tenant_mixed_precision_b200.synth_stack import populate

    def plan_fn(l, p, d_out, d_in, t):
        if t % 5 == 4 and p == 2:  # some tenants have no delta for one projection
            return None
        return plans.budget_plan(d_out, d_in, 1 / 16, plans.MIXED_1_16)

    T = 24
    ref = DeltaStack(512, 1024, 2, 14, T, plan_fn, out_dtype=torch.float32)
    populate(ref, 4242, s0=0.02 * np.sqrt(512.0))
    paged = PagedStack(ref, n_slots=4)
    yield ref, paged, T
    paged.pager.close()


def _outputs(st):
    return [[y.clone() for y in row] for row in st.y]


def test_paged_outputs_equal_resident(stacks):
    ref, paged, T = stacks
    compute = torch.cuda.Stream()
    copy = torch.cuda.Stream()
    rng = np.random.default_rng(99)
    was_evicted, reloaded = set(), set()
    for b in range(24):
        n = int(rng.integers(1, T + 1))
        ids = synth.zipf_tenants(rng, n, ref.n_tenants)
        if b % 6 == 5:
            ids[: n // 3] = -1  # some backbone-only tokens
        # at most 4 distinct tenants per batch (the slots); keep the draw's order
        keep = list(dict.fromkeys(int(t) for t in ids if t >= 0))[:4]
        ids = np.array([t if (t < 0 or t in keep) else keep[0] for t in ids], dtype=np.int32)
        ids_dev = torch.from_numpy(ids).cuda()
        with torch.cuda.stream(compute):
            ref.forward(ids_dev, n, stream=compute)
        compute.synchronize()
        assert dc.dc_read_device_status(ref.ws, compute) == 0
        want = _outputs(ref)
        for t in keep:
            if t in was_evicted and paged.pager.slot_of(t) < 0:
                reloaded.add(t)
        before = {t: paged.pager.slot_of(t) for t in range(ref.n_tenants)}
        with torch.cuda.stream(compute):
            paged.forward(ids, ids_dev, n, compute, copy)
        compute.synchronize()
        assert dc.dc_read_device_status(ref.ws, compute) == 0
        got = _outputs(ref)
        for l in range(ref.layers):
            for p in range(7):
                assert torch.equal(got[l][p][:n], want[l][p][:n]), (b, l, p)
        for t in range(ref.n_tenants):
            if before[t] >= 0 and paged.pager.slot_of(t) < 0:
                was_evicted.add(t)
        assert all(paged.pager.slot_of(t) >= 0 for t in keep)
    st = paged.pager.stats()
    assert st["batches"] == 24 and st["misses"] > 0 and st["evictions"] > 0 and st["hits"] > 0
    sizes = [paged.image_bytes(t) for t in range(ref.n_tenants)]
    assert st["misses"] * min(sizes) <= st["bytes_loaded"] <= st["misses"] * max(sizes)
    assert reloaded, "the Zipf sequence should evict a tenant and later load it again"


def test_batch_with_more_tenants_than_slots_is_refused(stacks):
    ref, paged, T = stacks
    before = [paged.pager.slot_of(t) for t in range(ref.n_tenants)]
    ids = np.arange(5, dtype=np.int32)
    s = torch.cuda.Stream()
    with pytest.raises(dc.DcError) as e:
        paged.pager.prepare(ids, s, s)
    assert e.value.status == dc.DC_ERR_UNSUPPORTED
    assert [paged.pager.slot_of(t) for t in range(ref.n_tenants)] == before
    with pytest.raises(dc.DcError) as e:
        paged.pager.prepare(np.array([0, ref.n_tenants], dtype=np.int32), s, s)
    assert e.value.status == dc.DC_ERR_TENANT
