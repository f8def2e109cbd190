"""GPU parity of the calibration objective (harp_calib_fit) against the oracle's
calib_fit: L_fit = L_diag + lambda_bd R_bd and its gradient in both butterflies' angles
(HARP page, Sec. 2.3). The oracle's calib_fit is pinned on the CPU in
test_oracle_pins.py, including its gradient against finite differences.

The gradient holds the code target T = deq(Q(W')) constant, so it jumps wherever a
rotated weight crosses a rounding boundary. The device rotates in fp32, the oracle in
fp64, and on realistic weights a few codes differ. Perturbing W by 1e-7 relative moves
the fp64 oracle's own gradient by 1.3e-3 to 3.2e-3 (relative L2) on these shapes, while
the loss moves by less than 1e-7. Hence:
  - the loss is compared at 1e-4 relative on realistic weights;
  - the gradient on realistic weights is compared at 2e-2, about ten times that gap;
  - the tight bar uses weights built so that every rotated weight sits at least 0.2 steps
    inside its code cell, with fp16-exact group minima and maxima. Both sides then take
    the same integer decisions, and only fp32 rounding separates them. The gradient is
    still ill-conditioned in W: the residual W' - T is about ten times smaller than W', so
    a 1e-6 relative perturbation of W moves the oracle's own gradient by up to 1.6e-4 on
    these shapes (most on the U side of the 4096 x 11008 layer). The device's fp32
    rotations stay below that perturbation, and the bar is 1e-3.
"""
import numpy as np
import pytest

import oracle
from rotated_bit_matmul_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LOSS_GATE = 1e-4
GRAD_GATE_EXACT = 1e-3
GRAD_GATE_REALISTIC = 2e-2
LAMBDA = 0.1


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rotated_bit_matmul_b200 import build_lib, _lib
    build_lib.build()
    _lib.load()
    yield
    import rotated_bit_matmul_b200 as rb
    torch.cuda.synchronize()
    rb.harp_device_status()


def _dev(a, dt):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype=dt)


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


def _params(n_out, n_in, w_in, w_out, linear):
    thV, sV = synth.butterfly_params(n_in, w_in, 11, 0, linear, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, 11, 0, linear, "U")
    return thV, sV, thU, sU


def _hessian(n_in, linear, samples=512):
    X = synth.calibration_inputs(samples, n_in, 11, 0, linear).astype(np.float64)
    return (X.T @ X / samples).astype(np.float32)


def _exact_decision_weights(n_out, n_in, w_in, w_out, bits, thV, sV, thU, sU, seed):
    """W = U^T W'_0 V for a rotated target W'_0 whose codes are unambiguous: per group of 64,
    fp16-exact scale s0 and zero z0, one weight at code 0 and one at code 2^b - 1 exactly
    (the group's min and max), and every other weight 0.3 steps or less from its cell
    centre. Returns (W fp32, the planned codes)."""
    rng = np.random.default_rng(seed)
    L = (1 << bits) - 1
    ng = n_in // 64
    s0 = 2.0 ** rng.integers(-9, -6, (n_out, ng)) * (1.0 + rng.integers(0, 8, (n_out, ng)) / 8.0)
    z0 = -s0 * rng.integers(0, L + 1, (n_out, ng))
    q = rng.integers(0, L + 1, (n_out, n_in))
    u = rng.uniform(-0.3, 0.3, (n_out, n_in))
    u = np.where(q == 0, np.abs(u), np.where(q == L, -np.abs(u), u))
    q[:, 0::64], u[:, 0::64] = 0, 0.0
    q[:, 1::64], u[:, 1::64] = L, 0.0
    Wp0 = np.repeat(z0, 64, axis=1) + np.repeat(s0, 64, axis=1) * (q + u)
    # W = U^T W'_0 V: columns through F_U, then rows through F_V^T
    A = oracle.butterfly_fwd(Wp0.T, thU, sU, w_out).T
    W = oracle.butterfly_inv(np.ascontiguousarray(A), thV, sV, w_in).astype(np.float32)
    return W, q


def _device(W, bits, w_in, w_out, thV, sV, thU, sU, H, lam, grad):
    import rotated_bit_matmul_b200 as rb
    r = rb.harp_calib_fit(_dev(W, torch.float32), bits, w_in, w_out, _dev(thV, torch.float32), _dev(sV, torch.int8),
                          _dev(thU, torch.float32), _dev(sU, torch.int8), _dev(H, torch.float32), lam, grad=grad)
    torch.cuda.synchronize()
    rb.harp_device_status()
    if grad:
        loss, gV, gU = r
        return loss.cpu().numpy(), gV.cpu().numpy(), gU.cpu().numpy()
    return r.cpu().numpy()


def _check_loss(got, want):
    for g, w in zip(got, want):
        assert abs(g - w) <= LOSS_GATE * abs(w) + 1e-30, (got, want)


SHAPES = [
    (4096, 4096, 4096, 4096, 2, True),     # attention projection, full-width blocks
    (11008, 4096, 4096, 256, 3, True),     # MLP up: 43 output blocks of 256
    (4096, 11008, 256, 4096, 4, False),    # MLP down (an 11008 x 11008 proxy is left out)
    (96, 256, 32, 32, 2, True),            # narrow blocks, ragged transpose tiles
]


@pytest.mark.parametrize("n_out,n_in,w_in,w_out,bits,hess", SHAPES)
def test_calib_loss_matches_oracle(n_out, n_in, w_in, w_out, bits, hess):
    thV, sV, thU, sU = _params(n_out, n_in, w_in, w_out, 0)
    W = synth.weights(n_out, n_in, 11, 0, 0)
    H = _hessian(n_in, 0) if hess else None
    got = _device(W, bits, w_in, w_out, thV, sV, thU, sU, H, LAMBDA, False)
    want = oracle.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=H, lambda_bd=LAMBDA)
    assert want[1] > 0 and (want[2] > 0) == hess
    _check_loss(got, want)


@pytest.mark.parametrize("n_out,n_in,w_in,w_out,bits,hess", SHAPES)
def test_calib_gradient_exact_decisions(n_out, n_in, w_in, w_out, bits, hess):
    thV, sV, thU, sU = _params(n_out, n_in, w_in, w_out, 1)
    W, q = _exact_decision_weights(n_out, n_in, w_in, w_out, bits, thV, sV, thU, sU, seed=n_out + bits)
    # the oracle's own codes are the planned ones
    Wr = oracle.rotate_weights(W, thV, sV, w_in, thU, sU, w_out)
    assert np.array_equal(oracle.quantize(Wr, bits)[0], q)
    H = _hessian(n_in, 1) if hess else None
    loss, gV, gU = _device(W, bits, w_in, w_out, thV, sV, thU, sU, H, LAMBDA, True)
    wl, wV, wU = oracle.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=H, lambda_bd=LAMBDA, grad=True)
    _check_loss(loss, wl)
    eV, eU = _rel(gV, wV), _rel(gU, wU)
    print(f"grad rel-L2 V {eV:.2e} U {eU:.2e}")
    assert eV < GRAD_GATE_EXACT and eU < GRAD_GATE_EXACT


def test_calib_gradient_realistic_weights():
    n_out, n_in, w_in, w_out, bits = 4096, 4096, 4096, 4096, 2
    thV, sV, thU, sU = _params(n_out, n_in, w_in, w_out, 2)
    W = synth.weights(n_out, n_in, 11, 0, 2)
    H = _hessian(n_in, 2)
    loss, gV, gU = _device(W, bits, w_in, w_out, thV, sV, thU, sU, H, LAMBDA, True)
    wl, wV, wU = oracle.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=H, lambda_bd=LAMBDA, grad=True)
    _check_loss(loss, wl)
    eV, eU = _rel(gV, wV), _rel(gU, wU)
    print(f"realistic grad rel-L2 V {eV:.2e} U {eU:.2e}")
    assert eV < GRAD_GATE_REALISTIC and eU < GRAD_GATE_REALISTIC


def test_calib_gradient_at_the_hadamard_start():
    """Null theta on both sides (Theta = 0, where calibration starts) against the oracle
    with explicit zero angles; the gradient is the first step's."""
    n_out, n_in, w_in, w_out, bits = 4096, 4096, 4096, 4096, 2
    _, sV, _, sU = _params(n_out, n_in, w_in, w_out, 3)
    zV = np.zeros((12, n_in // 2), np.float32)
    zU = np.zeros((12, n_out // 2), np.float32)
    W, _ = _exact_decision_weights(n_out, n_in, w_in, w_out, bits, zV, sV, zU, sU, seed=3)
    H = _hessian(n_in, 3)
    loss, gV, gU = _device(W, bits, w_in, w_out, None, sV, None, sU, H, LAMBDA, True)
    wl, wV, wU = oracle.calib_fit(W, bits, w_in, w_out, zV, sV, zU, sU, H=H, lambda_bd=LAMBDA, grad=True)
    _check_loss(loss, wl)
    assert _rel(gV, wV) < GRAD_GATE_EXACT and _rel(gU, wU) < GRAD_GATE_EXACT


def test_calib_is_reproducible_and_zero_for_zero_weights():
    n_out, n_in, w_in, w_out = 1024, 1024, 1024, 1024
    thV, sV, thU, sU = _params(n_out, n_in, w_in, w_out, 4)
    W = synth.weights(n_out, n_in, 11, 0, 4)
    H = _hessian(n_in, 4)
    a = _device(W, 2, w_in, w_out, thV, sV, thU, sU, H, LAMBDA, True)
    b = _device(W, 2, w_in, w_out, thV, sV, thU, sU, H, LAMBDA, True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    z = _device(np.zeros_like(W), 2, w_in, w_out, thV, sV, thU, sU, None, LAMBDA, True)
    assert np.all(z[0] == 0.0) and not np.any(z[1]) and not np.any(z[2])
