"""GPU parity of the calibration forward (harp_calib_error) against the oracle's
calib_error: L = sum_rj h_j (W - U^T deq(Q(U W V^T)) V)_rj^2.

The device rotates in fp32, the oracle in fp64, so a code may differ where a rotated
weight sits on a rounding boundary; either code is then about half a step away, which
moves L by a relative amount far below the 1e-4 gate. The oracle's calib_error is
pinned on the CPU (test_oracle_pins.py): h = 1 equals the rotated-domain error, h = e_j
equals column j of the linear's reconstruction error, and L is linear in h.
"""
import numpy as np
import pytest

import oracle
from rotated_bit_matmul_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GATE = 1e-4


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


def _case(n_out, n_in, w_in, w_out, linear=0):
    W = synth.weights(n_out, n_in, 11, 0, linear)
    thV, sV = synth.butterfly_params(n_in, w_in, 11, 0, linear, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, 11, 0, linear, "U")
    return W, thV, sV, thU, sU


def _run(W, bits, w_in, w_out, thV, sV, thU, sU, h):
    import rotated_bit_matmul_b200 as rb
    got = rb.harp_calib_error(_dev(W, torch.float32), bits, w_in, w_out, _dev(thV, torch.float32),
                              _dev(sV, torch.int8), _dev(thU, torch.float32), _dev(sU, torch.int8),
                              _dev(h, torch.float32)).item()
    torch.cuda.synchronize()
    rb.harp_device_status()
    return got


@pytest.mark.parametrize("n_out,n_in,w_in,w_out,bits", [
    (4096, 4096, 4096, 4096, 2),      # attention projection, full-width blocks
    (11008, 4096, 4096, 256, 3),      # MLP up: 43 output blocks of 256
    (4096, 11008, 256, 4096, 4),      # MLP down
    (96, 256, 32, 32, 2),             # several narrow blocks, a tile and a ragged transpose edge
])
@pytest.mark.parametrize("weighted", [False, True])
def test_calib_error_matches_oracle(n_out, n_in, w_in, w_out, bits, weighted):
    W, thV, sV, thU, sU = _case(n_out, n_in, w_in, w_out)
    h = np.random.default_rng(n_in + bits).gamma(2.0, 0.5, n_in).astype(np.float32) if weighted else None
    got = _run(W, bits, w_in, w_out, thV, sV, thU, sU, h)
    want = oracle.calib_error(W, bits, w_in, w_out, thV, sV, thU, sU, h)
    assert want > 0
    assert abs(got - want) <= GATE * want, (got, want)


def test_calib_error_rht_sides():
    """Null theta (Theta = 0) on both sides equals the oracle with explicit zero angles;
    the adapted angles of the synthetic case give a different error."""
    W, thV, sV, thU, sU = _case(4096, 4096, 4096, 4096, linear=3)
    got = _run(W, 2, 4096, 4096, None, sV, None, sU, None)
    want = oracle.calib_error(W, 2, 4096, 4096, np.zeros_like(thV), sV, np.zeros_like(thU), sU)
    assert abs(got - want) <= GATE * want, (got, want)
    learned = _run(W, 2, 4096, 4096, thV, sV, thU, sU, None)
    assert abs(learned - got) > GATE * want


def test_calib_error_is_reproducible_and_zero_for_zero_weights():
    W, thV, sV, thU, sU = _case(1024, 1024, 1024, 1024, linear=5)
    a = _run(W, 2, 1024, 1024, thV, sV, thU, sU, None)
    b = _run(W, 2, 1024, 1024, thV, sV, thU, sU, None)
    assert a == b
    assert _run(np.zeros_like(W), 2, 1024, 1024, thV, sV, thU, sU, None) == 0.0
