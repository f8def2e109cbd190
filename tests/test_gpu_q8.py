"""GPU parity of int8 angle storage (harp_quantize_angles, harp_create_layer_q8).

The HARP page stores its parameters in int8. This library keeps one symmetric step per
butterfly stage. A layer stored that way applies the dequantized angles
theta^ = delta_t q, so the oracle for it is the ordinary oracle layer built from theta^
(the oracle's quantize_angles and dequantize_angles are pinned on the CPU in
test_oracle_pins.py).
  - The device angle quantizer evaluates its rule in fp64 from the same fp32 angles, so
    its codes and steps must equal the oracle's bit for bit.
  - The per-linear butterflies evaluate cos/sin of pi/4 + delta_t q with sincosf; the
    fused decode step uses the fast sine/cosine unit (absolute error about 5e-7). Both
    are held to the same 2e-3 relative-L2 gate as the fp32-angle path.
"""
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
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype=dt)


@pytest.mark.parametrize("m,half", [(12, 2048), (8, 5504), (13, 4096), (1, 16), (5, 48)])
def test_angle_quantizer_matches_oracle(m, half):
    import rotated_bit_matmul_b200 as rb
    rng = np.random.default_rng(m * half)
    th = (rng.uniform(-0.05, 0.05, (m, half)) * rng.uniform(0.05, 4.0, (m, 1))).astype(np.float32)
    th[0, :7] = 0.0
    if m > 2:
        th[2] = 0.0  # an all-zero stage: step 0, codes 0
    q, d = rb.harp_quantize_angles(_dev(th, torch.float32))
    wq, wd = oracle.quantize_angles(th)
    assert np.array_equal(q.cpu().numpy(), wq)
    assert np.array_equal(d.cpu().numpy(), wd)


def _q8_case(n_out, n_in, w_in, w_out, bits, workload=12, layer=0, linear=0, rht=(False, False)):
    """Seeded W and angles; the angles pass through the oracle's int8 quantizer and the
    oracle layer is built from the angles they stand for."""
    W = synth.weights(n_out, n_in, workload, layer, linear)
    thV, sV = synth.butterfly_params(n_in, w_in, workload, layer, linear, "V")
    thU, sU = synth.butterfly_params(n_out, w_out, workload, layer, linear, "U")
    qV, dV = oracle.quantize_angles(thV)
    qU, dU = oracle.quantize_angles(thU)
    hV, hU = oracle.dequantize_angles(qV, dV), oracle.dequantize_angles(qU, dU)
    if rht[0]:
        qV, hV = None, np.zeros_like(hV)
    if rht[1]:
        qU, hU = None, np.zeros_like(hU)
    lay = oracle.prepare_layer(W, bits, w_in, w_out, hV, sV, hU, sU)[0]
    return dict(lay=lay, qV=qV, dV=dV, sV=sV, qU=qU, dU=dU, sU=sU, n_in=n_in, n_out=n_out, w_in=w_in, w_out=w_out,
                bits=bits, thV=thV, thU=thU)


def _device(c):
    import rotated_bit_matmul_b200 as rb
    lay = c["lay"]
    return rb.HarpLayer.int8_angles(c["n_in"], c["n_out"], c["bits"], c["w_in"], c["w_out"], _dev(c["qV"], torch.int8),
                                    _dev(c["dV"], torch.float32), _dev(c["sV"], torch.int8), _dev(c["qU"], torch.int8),
                                    _dev(c["dU"], torch.float32), _dev(c["sU"], torch.int8),
                                    _dev(lay.packed.copy(), torch.uint8),
                                    _dev(lay.sz.reshape(-1).view(np.int32).copy(), torch.int32))


@pytest.mark.parametrize("batch", [1, 3, 16])
@pytest.mark.parametrize("shape,bits", [((4096, 4096, 4096, 4096), 2), ((11008, 4096, 4096, 256), 3),
                                        ((4096, 11008, 256, 4096), 4), ((96, 256, 64, 32), 2)])
def test_q8_linear(shape, bits, batch):
    """int8-angle layers on the dequant-GEMV path (1 and 3 tokens) and the tensor-core
    path (16 tokens), against the oracle layer built from the dequantized angles."""
    c = _q8_case(*shape, bits)
    x = synth.activations(batch, c["n_in"], 12, step=batch)
    L = _device(c)
    got = L(_dev(x, torch.bfloat16), out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    L.close()
    want = oracle.linear_fwd(c["lay"], x.astype(np.float64))
    err = rel_l2(got, want)
    print(f"q8 linear {shape} b{bits} batch {batch}: rel-L2 {err:.2e}")
    assert err < GATE


def test_q8_linear_one_side_hadamard():
    """q NULL on one side makes it Theta = 0, as a null theta does."""
    c = _q8_case(4096, 4096, 4096, 4096, 2, rht=(True, False))
    x = synth.activations(1, 4096, 12, step=7)
    L = _device(c)
    got = L(_dev(x, torch.bfloat16), out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    L.close()
    assert rel_l2(got, oracle.linear_fwd(c["lay"], x.astype(np.float64))) < GATE


def test_q8_angles_differ_from_fp32_angles():
    """The int8 layer is the layer of the dequantized angles, not of the fp32 ones: the
    oracle's two layers differ by more than the gate, and the device matches the first."""
    c = _q8_case(4096, 4096, 4096, 4096, 2, linear=3)
    W = synth.weights(4096, 4096, 12, 0, 3)
    lay32 = oracle.prepare_layer(W, 2, 4096, 4096, c["thV"], c["sV"], c["thU"], c["sU"])[0]
    x = synth.activations(1, 4096, 12, step=9).astype(np.float64)
    y8, y32 = oracle.linear_fwd(c["lay"], x), oracle.linear_fwd(lay32, x)
    assert rel_l2(y8, y32) > 1e-2


def _stack_cases(hidden, ffn, nh, nkv, hd, wb, n_blocks, bits=2):
    shp = [(nh * hd, hidden, hidden, nh * hd), (nkv * hd, hidden, hidden, nkv * hd),
           (nkv * hd, hidden, hidden, nkv * hd), (hidden, nh * hd, nh * hd, hidden), (ffn, hidden, hidden, wb),
           (ffn, hidden, hidden, wb), (hidden, ffn, wb, hidden)]
    return [_q8_case(o, i, wi, wo, bits, layer=l, linear=k) for l in range(n_blocks)
            for k, (o, i, wi, wo) in enumerate(shp)]


@pytest.mark.parametrize("dims,n_blocks", [((4096, 1024, 32, 8, 128, 256), 1), ((4096, 11008, 32, 32, 128, 256), 2)])
def test_q8_fused_decode_step(dims, n_blocks):
    """A stack whose butterflies all keep int8 angles runs the fused single-kernel step
    (the int8 instantiation) and matches the oracle stack of the dequantized angles."""
    import rotated_bit_matmul_b200 as rb
    hidden, ffn, nh, nkv, hd, wb = dims
    cases = _stack_cases(hidden, ffn, nh, nkv, hd, wb, n_blocks)
    layers = [_device(c) for c in cases]
    S = rb.HarpStack(layers, hidden, ffn, nh, nkv, hd)
    assert S.uses_fused_step(1)
    for step in (1, 2):
        x = synth.activations(1, hidden, 12, step=step)
        got = S.step(_dev(x, torch.bfloat16)).cpu().numpy()
        torch.cuda.synchronize()
        rb.harp_device_status()
        want = oracle.stack_step([c["lay"] for c in cases], hidden, ffn, nh, nkv, hd, x.astype(np.float64))
        err = rel_l2(got, want)
        print(f"q8 fused {dims} x{n_blocks} step {step}: rel-L2 {err:.3e}")
        assert err < GATE
    S.close()
    for L in layers:
        L.close()
