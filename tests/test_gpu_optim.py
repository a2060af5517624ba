"""The AdamW update kernel (nc_adamw_step) against the float64 oracle over
several steps: parameter groups with their own hyper-parameters, ragged
group boundaries, elements outside every group left alone, bf16 and fp32
compute copies of the weights."""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import NcError, adamw_step  # noqa: E402

GROUPS = [(0, 1000, 3e-3, 0.9, 0.95, 1e-8, 0.1),     # offset, count, lr, b1, b2, eps, wd
          (1000, 4097, 1e-2, 0.8, 0.99, 1e-6, 0.0),
          (5101, 333, 5e-4, 0.9, 0.999, 1e-8, 0.01)]  # 5097..5100 belong to no group
N = 5500


@pytest.mark.parametrize("wdtype", ["bf16", "fp32"])
def test_adamw_matches_oracle(wdtype):
    rng = np.random.default_rng(11)
    theta0 = rng.standard_normal(N).astype(np.float32)
    master = torch.from_numpy(theta0.copy()).cuda()
    weights = master.clone().to(torch.bfloat16 if wdtype == "bf16" else torch.float32)
    m = torch.zeros(N, device="cuda")
    v = torch.zeros(N, device="cuda")
    ref_t, ref_m, ref_v = theta0.astype(np.float64), np.zeros(N), np.zeros(N)
    for step in range(1, 5):
        g = (rng.standard_normal(N) * step).astype(np.float32)
        adamw_step(GROUPS, step, master, weights, torch.from_numpy(g).cuda(), m, v)
        for off, cnt, lr, b1, b2, eps, wd in GROUPS:
            sl = slice(off, off + cnt)
            t_, m_, v_ = ref_t[sl].copy(), ref_m[sl].copy(), ref_v[sl].copy()
            oracle.adamw_step(t_, g[sl].astype(np.float64), m_, v_, step, lr, b1, b2, eps, wd)
            ref_t[sl], ref_m[sl], ref_v[sl] = t_, m_, v_
    torch.cuda.synchronize()
    got = master.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref_t)) <= 1e-5 * np.max(np.abs(ref_t))
    np.testing.assert_allclose(m.cpu().numpy(), ref_m, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(v.cpu().numpy(), ref_v, rtol=1e-5, atol=1e-6)
    outside = np.r_[5097:5101, 5434:N]  # in no group: untouched
    assert np.array_equal(got[outside], theta0[outside].astype(np.float64))
    w = weights.float().cpu().numpy()
    expect = master.to(weights.dtype).float().cpu().numpy()  # the compute copy is the rounded master
    assert np.array_equal(w, expect)


def test_adamw_rejects_bad_arguments():
    t = torch.zeros(64, device="cuda")
    with pytest.raises(NcError):
        adamw_step([(0, 65, 1e-3, 0.9, 0.99, 1e-8, 0.0)], 1, t, t.clone(), t.clone(), t.clone(), t.clone())
    with pytest.raises(NcError):
        adamw_step([(0, 64, 1e-3, 0.9, 0.99, 1e-8, 0.0)], 0, t, t.clone(), t.clone(), t.clone(), t.clone())
    with pytest.raises(NcError):
        adamw_step([(0, 64, 1e-3, 1.0, 0.99, 1e-8, 0.0)], 1, t, t.clone(), t.clone(), t.clone(), t.clone())
