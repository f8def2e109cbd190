"""GPU parity of the fixed randomized Hadamard mode (Theta = 0, "RHT"): a null theta makes
a butterfly the Sylvester Hadamard transform H_w D / sqrt(w) per block. The kernels use
the constant 1/sqrt 2 blocks and load no per-stage parameters. The oracle computes the
same transform with explicit zero angles; its Theta = 0 case is pinned to
scipy.linalg.hadamard on the CPU (test_oracle_pins.py).
"""
import math

import numpy as np
import pytest

import oracle
from harp_cases import rel_l2
from rotated_bit_matmul_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

GATE = 2e-3


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
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype=dt)


@pytest.mark.parametrize("n,w,batch", [(4096, 4096, 3), (11008, 256, 2), (8192, 8192, 1), (1024, 1024, 4),
                                       (96, 32, 5)])
@pytest.mark.parametrize("inverse", [False, True])
def test_rht_butterfly(n, w, batch, inverse):
    import rotated_bit_matmul_b200 as rb
    rng = np.random.default_rng(n + w)
    sign = (rng.integers(0, 2, n) * 2 - 1).astype(np.int8)
    x = rng.standard_normal((batch, n)).astype(np.float32)
    f = rb.harp_butterfly_inv if inverse else rb.harp_butterfly_fwd
    got = f(_dev(x, torch.float32), None, _dev(sign, torch.int8), w).cpu().numpy()
    zero = np.zeros((int(math.log2(w)), n // 2), np.float32)
    want = (oracle.butterfly_inv if inverse else oracle.butterfly_fwd)(x, zero, sign, w)
    assert rel_l2(got, want) < 5e-6


def _rht_case(n_out, n_in, w_in, w_out, bits, V_rht=True, U_rht=True, workload=10, linear=0):
    """Seeded W and signs; the RHT sides get explicit zero angles for the oracle."""
    W = synth.weights(n_out, n_in, workload, 0, linear)
    thV, sV = synth.butterfly_params(n_in, w_in, workload, 0, linear, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, workload, 0, linear, "U")
    if V_rht:
        thV = np.zeros_like(thV)
    if U_rht:
        thU = np.zeros_like(thU)
    lay = oracle.prepare_layer(W, bits, w_in, w_out, thV, sV, thU, sU)[0]
    return dict(lay=lay, thV=None if V_rht else thV, sV=sV, thU=None if U_rht else thU, sU=sU, n_in=n_in,
                n_out=n_out, w_in=w_in, w_out=w_out, bits=bits)


def _device(case):
    import rotated_bit_matmul_b200 as rb
    lay = case["lay"]
    t = lambda a, dt: None if a is None else _dev(a, dt)
    return rb.HarpLayer(case["n_in"], case["n_out"], case["bits"], case["w_in"], case["w_out"],
                        t(case["thV"], torch.float32), t(case["sV"], torch.int8), t(case["thU"], torch.float32),
                        t(case["sU"], torch.int8), _dev(lay.packed.copy(), torch.uint8),
                        _dev(lay.sz.reshape(-1).view(np.int32).copy(), torch.int32))


@pytest.mark.parametrize("batch", [1, 16])
@pytest.mark.parametrize("shape,sides", [((4096, 4096, 4096, 4096), (True, True)),
                                         ((11008, 4096, 4096, 256), (True, True)),
                                         ((4096, 11008, 256, 4096), (True, False)),
                                         ((4096, 4096, 4096, 4096), (False, True))])
def test_rht_linear(shape, sides, batch):
    """Both sides, or one side, Theta = 0; dequant-GEMV (1 token) and tensor cores (16)."""
    case = _rht_case(*shape, 2, *sides)
    x = synth.activations(batch, case["n_in"], 10, step=batch)
    L = _device(case)
    got = L(_dev(x, torch.bfloat16), out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    L.close()
    want = oracle.linear_fwd(case["lay"], x.astype(np.float64))
    assert rel_l2(got, want) < GATE


def test_rht_fused_decode_step():
    """A 4096-wide block with every butterfly Theta = 0 runs the fused single-kernel step
    (no cos/sin tables loaded) and matches the oracle with zero angles."""
    import rotated_bit_matmul_b200 as rb
    hidden, ffn, nh, nkv, hd = 4096, 1024, 32, 2, 128
    shp = [(nh * hd, hidden), (nkv * hd, hidden), (nkv * hd, hidden), (hidden, nh * hd), (ffn, hidden),
           (ffn, hidden), (hidden, ffn)]
    cases = [_rht_case(o, i, 256 if i == ffn else i, 256 if o == ffn else o, 2, linear=k)
             for k, (o, i) in enumerate(shp)]
    layers = [_device(c) for c in cases]
    S = rb.HarpStack(layers, hidden, ffn, nh, nkv, hd)
    assert S.uses_fused_step(1)
    x = synth.activations(1, hidden, 10, step=5)
    got = S.step(_dev(x, torch.bfloat16)).cpu().numpy()
    torch.cuda.synchronize()
    rb.harp_device_status()
    S.close()
    for L in layers:
        L.close()
    want = oracle.stack_step([c["lay"] for c in cases], hidden, ffn, nh, nkv, hd, x.astype(np.float64))
    err = rel_l2(got, want)
    print(f"RHT fused rel-L2 {err:.3e}")
    assert err < GATE
