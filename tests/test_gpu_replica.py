"""GPU parity of replica weight sync (bit copies) and replica gradient reduction (float32 sums in
replica order, against the oracle's float64 sums)."""
import numpy as np
import pytest
import torch

import oracle
from combine_get_dispatch_histogram_b200 import ep, inputs
from gpu_util import dev, i32_dev

pytestmark = pytest.mark.gpu


def _plan(E_log, extra, seed):
    rng = np.random.default_rng(seed)
    idx = inputs.zipf_topk(rng, 512, E_log, min(4, E_log), 1.5).reshape(1, 512, -1)
    return oracle.reroute(idx, E_log, extra)["phys_base"]


@pytest.mark.parametrize("E_log,extra,P", [(64, 16, 4096), (8, 5, 12), (3, 0, 1024), (1, 7, 64)])
def test_weight_sync_and_grad_reduce(E_log, extra, P):
    pb = _plan(E_log, extra, E_log + extra)
    E_phys = int(pb[-1])
    rng = np.random.default_rng(P)
    master = rng.standard_normal((E_log, P)).astype(np.float32)
    grads = (rng.standard_normal((E_phys, P)) * rng.choice([1e-3, 1.0, 1e3], (E_phys, 1))).astype(np.float32)
    pb_d = i32_dev(pb)
    reps = ep.ep_replica_weight_sync(torch.from_numpy(master).to(dev()), pb_d)
    mg = ep.ep_replica_grad_reduce(torch.from_numpy(grads).to(dev()), pb_d)
    torch.cuda.synchronize()
    assert np.array_equal(reps.cpu().numpy(), oracle.replica_weight_sync(master, pb))
    want = oracle.replica_grad_reduce(grads, pb)
    got = mg.cpu().numpy().astype(np.float64)
    # sequential float32 summation of n terms: |error| <= (n - 1) * 2^-24 * sum |g|
    n = np.diff(pb).astype(np.float64)[:, None]
    absum = np.zeros_like(want)
    for e in range(E_log):
        absum[e] = np.abs(grads[pb[e]:pb[e + 1]].astype(np.float64)).sum(axis=0)
    assert np.all(np.abs(got - want) <= np.maximum(n - 1, 0) * 2.0 ** -24 * absum + 1e-30)


def test_weight_sync_bf16_rows_and_bad_plan_flag():
    E_log, P = 4, 7168
    pb = np.array([0, 3, 5, 6, 7], np.int32)
    master = inputs.bf16_tokens(np.random.default_rng(1), E_log, P)
    m = torch.from_numpy(master.view(np.int16)).to(dev()).view(torch.bfloat16)
    reps = ep.ep_replica_weight_sync(m, i32_dev(pb))
    torch.cuda.synchronize()
    assert np.array_equal(reps.view(torch.int16).cpu().numpy().view(np.uint16), oracle.replica_weight_sync(master, pb))
    # a phys_base pointing past the replica buffer is refused by the kernel, not followed
    bad = i32_dev(np.array([0, 3, 5, 6, 99], np.int32))
    st = torch.zeros(1, dtype=torch.int32, device=dev())
    out = torch.zeros((7, P), dtype=torch.bfloat16, device=dev())
    ep.ep_replica_weight_sync(m, bad, replicas=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ep.EP_STATUS_BAD_EXPERT
