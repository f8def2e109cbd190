"""GPU parity of the mixed-radix butterfly (harp_mr_plan_*, HARP Sec. 2.1-2.2) against the
oracle's mr_butterfly_fwd/inv, which is pinned on the CPU (test_oracle_pins.py): its
all-radix-2 schedules equal the radix-2 butterfly, Theta = 0 gives Sylvester H_d or the
Kronecker product of the base mixers, and an independent stride-permutation
construction agrees with it.

The device builds every block once in fp64 (Cayley solve, QR mixer) and stores it fp32;
each stage is a b-term fp32 dot product per output, so the relative L2 error stays near
1e-7 per stage. The gate is 2e-5.
"""
import numpy as np
import pytest

import oracle
from harp_cases import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GATE = 2e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotated_bit_matmul_b200 import build_lib, _lib
    build_lib.build()
    _lib.load()
    yield
    torch.cuda.synchronize()


def _case(radices, seed, scale=0.2):
    """Seeded angles, signs and one Gaussian per stage (the QR mixer's fixed matrix)."""
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    th = rng.uniform(-scale, scale, oracle.mr_theta_size(radices)).astype(np.float32)
    sign = (rng.integers(0, 2, d) * 2 - 1).astype(np.int8)
    gauss = [rng.standard_normal((b, b)).astype(np.float32) for b in radices]
    return d, th, sign, gauss


@pytest.mark.parametrize("radices", [(8, 8, 8, 5, 2), (2, 2, 2, 2, 2, 2, 2, 2, 43), (3, 4, 5), (2,) * 8, (16, 4),
                                     (7, 64), (64, 64, 4), (2,) * 12, (2,) * 5])
@pytest.mark.parametrize("inverse", [False, True])
@pytest.mark.parametrize("rows", [3, 9])
def test_mixed_radix_matches_oracle(radices, inverse, rows):
    """3 rows: the stages run in runs of at most 4096 coordinates over many CTAs; 9 rows: one
    CTA per row holds the whole row."""
    import rotated_bit_matmul_b200 as rb
    d, th, sign, gauss = _case(radices, sum(radices))
    plan = rb.HarpMixedRadix(radices, torch.from_numpy(th).cuda(), torch.from_numpy(sign).cuda(),
                             torch.from_numpy(np.concatenate([g.reshape(-1) for g in gauss])).cuda())
    x = np.random.default_rng(d).standard_normal((rows, d)).astype(np.float32)
    f = plan.inv if inverse else plan.fwd
    got = f(torch.from_numpy(x).cuda()).cpu().numpy()
    torch.cuda.synchronize()
    plan.close()
    g64 = [g.astype(np.float64) for g in gauss]
    want = (oracle.mr_butterfly_inv if inverse else oracle.mr_butterfly_fwd)(x, radices, th, sign, g64)
    err = rel_l2(got, want)
    print(f"mixed radix {radices} inverse={inverse} rows={rows}: rel-L2 {err:.2e}")
    assert err < GATE


def test_mixed_radix_round_trip_and_bf16_input():
    """F^T F x = x on the device, and a bf16 input gives the fp32 transform of its values."""
    import rotated_bit_matmul_b200 as rb
    radices = (8, 8, 8, 5, 2)
    d, th, sign, gauss = _case(radices, 5)
    plan = rb.HarpMixedRadix(radices, torch.from_numpy(th).cuda(), torch.from_numpy(sign).cuda(),
                             torch.from_numpy(np.concatenate([g.reshape(-1) for g in gauss])).cuda())
    x = torch.randn(4, d, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    back = plan.inv(plan.fwd(x))
    assert rel_l2(back.cpu().numpy(), x.cpu().numpy()) < GATE
    xb = x.to(torch.bfloat16)
    y = plan.fwd(xb, out_dtype=torch.float32)
    y32 = plan.fwd(xb.float())
    assert torch.equal(y, y32)
    plan.close()
