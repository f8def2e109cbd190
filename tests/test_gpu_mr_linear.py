"""GPU parity of linears with mixed-radix sides (HARP page, Sec. 2.1, Suporte a Misto-Raiz):
harp_create_layer_mr against the oracle's mr_linear_fwd, which is pinned on the CPU
(exact change of basis, the all-radix-2 case equal to the radix-2 linear, its own codes).

The widths are the pages' non-power-of-two cases: 11008 = 2^8 * 43 (Llama-2-7B FFN) on the
output side (gate/up) and the input side (down), a radix-7 side of 14336 = 2^11 * 7 (the
70B FFN's 28672 = 2^12 * 7 exceeds the 16384 one mixed-radix row holds on the device), and
radix-8 Cayley sides. Gates as for the radix-2 layers: rel-L2 2e-3 on the GEMV path
(1 and 4 tokens) and on the tensor-core path (16 tokens).
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


def _side(radices, seed):
    """Seeded fp32 parameters, signs and one fp32 Gaussian per stage (the QR mixer's fixed
    matrix; read only for radices that are not powers of two)."""
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    theta = rng.uniform(-0.05, 0.05, oracle.mr_theta_size(radices)).astype(np.float32)
    sign = (rng.integers(0, 2, d) * 2 - 1).astype(np.int8)
    gauss = [rng.standard_normal((b, b)).astype(np.float32) for b in radices]
    return oracle.MixedRadixSide(radices, theta, sign, [g.astype(np.float64) for g in gauss])


def _device_plan(side):
    from rotated_bit_matmul_b200 import HarpMixedRadix
    dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype=dt)
    flat = np.concatenate([np.asarray(g, np.float32).reshape(-1) for g in side.gauss])
    return HarpMixedRadix(side.radices, dev(side.theta, torch.float32), dev(side.sign, torch.int8),
                          dev(flat, torch.float32))


CASES = [
    # (n_out radices, n_in radices): gate/up of 7B (11008 = 2^8 * 43 out), down of 7B
    # (11008 in), a radix-7 side (14336 = 2^11 * 7; 70B's 28672 = 2^12 * 7 is twice the
    # 16384 the mixed-radix kernel holds per row), radix-8 Cayley sides
    ((2, 2, 2, 2, 2, 2, 2, 2, 43), (16, 16, 16)),
    ((16, 16, 16), (43, 2, 2, 2, 2, 2, 2, 2, 2)),
    ((8, 8, 8, 4, 7), (8, 8, 8)),
    ((8, 8, 8), (8, 8, 8)),
    # all radices 2 on both sides: the plans run on the radix-2 butterfly kernels
    ((2,) * 9, (2,) * 12),
]


@pytest.mark.parametrize("out_r,in_r", CASES, ids=lambda r: "x".join(map(str, r)))
@pytest.mark.parametrize("bits", [2, 3])
def test_mr_linear_matches_oracle(out_r, in_r, bits):
    import rotated_bit_matmul_b200 as rb
    U, V = _side(out_r, 1), _side(in_r, 2)
    n_out, n_in = int(np.prod(out_r)), int(np.prod(in_r))
    W = synth.weights(n_out, n_in, 12, 0, bits)
    lay, _ = oracle.mr_prepare_layer(W, bits, V, U)
    pV, pU = _device_plan(V), _device_plan(U)
    codes = torch.from_numpy(lay["packed"].copy()).to("cuda")
    sz = torch.from_numpy(np.ascontiguousarray(lay["sz"]).reshape(-1).view(np.int32).copy()).to("cuda")
    L = rb.HarpLayer.mixed_radix(pV, pU, bits, codes, sz)
    for batch in (1, 4, 16):
        x = synth.activations(batch, n_in, 12, step=batch)
        got = L(torch.from_numpy(x).to("cuda", torch.bfloat16), out_dtype=torch.float32).cpu().numpy()
        want = oracle.mr_linear_fwd(lay, x.astype(np.float64))
        err = rel_l2(got, want)
        rows = max(rel_l2(got[b], want[b]) for b in range(batch))
        print(f"{n_out}x{n_in} {bits}-bit batch {batch}: rel-L2 {err:.3e}, worst row {rows:.3e}")
        assert err < GATE, (batch, err)
        assert rows < 2 * GATE, (batch, rows)
    L.close()
    pV.close()
    pU.close()


def test_mr_layer_rejects_mismatched_plans():
    """n_in must equal the input plan's length (checked before anything is launched)."""
    import ctypes
    from rotated_bit_matmul_b200 import _lib
    lib = _lib.load()
    V, U = _side((8, 8, 8), 3), _side((16, 16), 4)
    pV, pU = _device_plan(V), _device_plan(U)
    codes = torch.zeros(1024 * 256 // 4, dtype=torch.uint8, device="cuda")
    sz = torch.zeros(1024 * 256 // 64, dtype=torch.int32, device="cuda")
    h = ctypes.c_void_p()
    st = lib.harp_create_layer_mr(ctypes.byref(h), 1024, 256, 2, 64, pV.handle, pU.handle,
                                  ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(sz.data_ptr()), None)
    assert st == 1 and not h.value
    assert b"lengths" in lib.harp_last_error()
    pV.close()
    pU.close()
